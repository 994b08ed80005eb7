// Generic SIMT kernels of the LISA module: any supported shape, float32 or
// bfloat16 activations.  They serve every call the specialised sm_100a paths
// do not cover (the fp32 workloads, odd head counts and dimensions), and are
// written for clarity over speed.
//
// Operations follow "LISA: Linear-Indexed Sparse Attention for Efficient
// Long-Context Reasoning" (arXiv 2607.19358v1): indexer scores and top-M
// (Sec. 3.2), sparse softmax attention (Sec. 3.2 Eq. 1, Sec. 3.1), linear
// attention (Sec. 3.1, Sec. 3.3 Eq. 3-4) and the gate (Sec. 3.2 Eq. 1).
#include <math.h>

#include "lisa_internal.cuh"

namespace lisa {
namespace {

constexpr int kMaxDimChunks = 8;  // d <= 256 = 8 lanes-chunks of 32

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Exclusive prefix sum of `v` over the block; `total` receives the block sum.
// `scratch` holds one int per warp.  Every thread of the block must call it.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    int warp_off = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        int x = scratch[w];
        if (w < warp) warp_off += x;
        total += x;
    }
    __syncthreads();
    return warp_off + incl - v;
}

// ------------------------------------------------------------------ indexer
// One thread per (query row, key position).  scores: [B*T, L].
template <typename T>
__global__ void k_index_scores(Shape s, const T* __restrict__ q_I, const T* __restrict__ k_I,
                               const float* __restrict__ w, int64_t w_tok_stride,
                               float* __restrict__ scores) {
    extern __shared__ float sm[];
    float* qs = sm;                      // [H_I * d_I]
    float* ws = sm + s.H_I * s.d_I;      // [H_I]
    const int row = blockIdx.x;  // rows on x: B*T may exceed the 65535 limit of y
    const int b = row / s.T, t = row % s.T;
    const int p = s.n_past + t;
    const T* qrow = q_I + (int64_t)row * s.H_I * s.d_I;
    for (int i = threadIdx.x; i < s.H_I * s.d_I; i += blockDim.x) qs[i] = to_f32(qrow[i]);
    const int64_t wb = w_tok_stride ? (int64_t)s.T * w_tok_stride : s.H_I;
    for (int j = threadIdx.x; j < s.H_I; j += blockDim.x)
        ws[j] = w[b * wb + (int64_t)t * w_tok_stride + j];
    __syncthreads();
    const int key = blockIdx.y * blockDim.x + threadIdx.x;
    if (key >= s.L) return;
    float total = -INFINITY;
    if (key <= p) {
        total = 0.0f;
        const T* krow = k_I + ((int64_t)b * s.N_max + key) * s.H_Ik * s.d_I;
        for (int j = 0; j < s.H_I; ++j) {
            const T* kv = krow + (j % s.H_Ik) * s.d_I;
            const float* qv = qs + j * s.d_I;
            float dot = 0.0f;
            for (int c = 0; c < s.d_I; ++c) dot = fmaf(qv[c], to_f32(kv[c]), dot);
            total = fmaf(ws[j], fmaxf(dot, 0.0f), total);
        }
    }
    scores[(int64_t)row * s.L + key] = total;
}

// ------------------------------------------------------------------ top-M
// One block per query row.  Radix select (8 bits per pass, most significant
// first) finds the M-th largest key exactly; an order-preserving compaction
// then writes every key above it plus the lowest positions equal to it.
template <int NT>
__global__ void __launch_bounds__(NT) k_topm_rows(Shape s, const float* __restrict__ scores,
                                                  int32_t* __restrict__ idx,
                                                  int32_t* __restrict__ count) {
    __shared__ unsigned hist[256];
    __shared__ unsigned sh_prefix, sh_krem;
    __shared__ int scan_scratch[NT / 32];
    const int row = blockIdx.x;
    const int t = row % s.T;
    const int n_cand = s.n_past + t + 1;
    const float* sc = scores + (int64_t)row * s.L;
    int32_t* out = idx + (int64_t)row * s.M;
    if (n_cand <= s.M) {
        for (int i = threadIdx.x; i < s.M; i += NT) out[i] = i < n_cand ? i : -1;
        if (threadIdx.x == 0) count[row] = n_cand;
        return;
    }
    unsigned prefix = 0, mask = 0, krem = (unsigned)s.M;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n_cand; i += NT) {
            const unsigned key = order_key(sc[i]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            unsigned cum = 0;
            int bin = 255;
            for (; bin > 0; --bin) {
                if (cum + hist[bin] >= krem) break;
                cum += hist[bin];
            }
            sh_prefix = prefix | ((unsigned)bin << shift);
            sh_krem = krem - cum;
        }
        __syncthreads();
        prefix = sh_prefix;
        krem = sh_krem;
        mask |= 0xFFu << shift;
        __syncthreads();
    }
    // prefix is the M-th largest key; krem of the keys equal to it are kept.
    int base_out = 0, base_eq = 0;
    for (int i0 = 0; i0 < n_cand; i0 += NT) {
        const int i = i0 + threadIdx.x;
        const unsigned key = i < n_cand ? order_key(sc[i]) : 0u;
        const int gt = (i < n_cand) && key > prefix;
        const int eq = (i < n_cand) && key == prefix;
        int eq_total, sel_total;
        const int eq_rank = block_exclusive_scan<NT>(eq, scan_scratch, eq_total) + base_eq;
        const int sel = gt || (eq && eq_rank < (int)krem);
        const int pos = block_exclusive_scan<NT>(sel, scan_scratch, sel_total) + base_out;
        if (sel) out[pos] = i;
        base_out += sel_total;
        base_eq += eq_total;
    }
    if (threadIdx.x == 0) count[row] = s.M;
}

// ------------------------------------------------------------------ attention
// One block of 4 warps per (query row, query head).  Each warp runs an online
// softmax over a strided share of the positions; the warps are merged at the end.
template <typename T, typename TO>
__global__ void __launch_bounds__(128) k_attention(Shape s, const T* __restrict__ q,
                                                   const T* __restrict__ kc,
                                                   const T* __restrict__ vc,
                                                   const int32_t* __restrict__ idx,
                                                   const int32_t* __restrict__ count,
                                                   TO* __restrict__ o, unsigned* status) {
    __shared__ float qs[256];
    __shared__ float wm[4], wl[4];
    __shared__ float wacc[4][256];
    const int row = blockIdx.x, h = blockIdx.y;
    const int b = row / s.T, t = row % s.T;
    const int p = s.n_past + t;
    const int g = h / s.group;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const T* qrow = q + ((int64_t)row * s.H_q + h) * s.d;
    for (int c = threadIdx.x; c < s.d; c += 128) qs[c] = to_f32(qrow[c]);
    __syncthreads();
    const int n = idx ? min(count[row], s.M) : p + 1;
    float m = -INFINITY, l = 0.0f;
    float acc[kMaxDimChunks];
#pragma unroll
    for (int k = 0; k < kMaxDimChunks; ++k) acc[k] = 0.0f;
    for (int i = warp; i < n; i += 4) {
        const int pos = idx ? idx[(int64_t)row * s.M + i] : i;
        if (pos < 0 || pos > p) {
            if (lane == 0) record_error(status, kDevBounds);
            continue;
        }
        const int64_t base = (((int64_t)b * s.N_max + pos) * s.H_kv + g) * s.d;
        float dot = 0.0f;
#pragma unroll
        for (int k = 0; k < kMaxDimChunks; ++k) {
            const int c = lane + 32 * k;
            if (c < s.d) dot = fmaf(qs[c], to_f32(kc[base + c]), dot);
        }
        const float logit = warp_sum(dot) * s.sm_scale;
        const float m_new = fmaxf(m, logit);
        const float corr = expf(m - m_new);
        const float e = expf(logit - m_new);
        l = l * corr + e;
#pragma unroll
        for (int k = 0; k < kMaxDimChunks; ++k) {
            const int c = lane + 32 * k;
            if (c < s.d) acc[k] = fmaf(e, to_f32(vc[base + c]), acc[k] * corr);
        }
        m = m_new;
    }
    if (lane == 0) { wm[warp] = m; wl[warp] = l; }
#pragma unroll
    for (int k = 0; k < kMaxDimChunks; ++k) {
        const int c = lane + 32 * k;
        if (c < s.d) wacc[warp][c] = acc[k];
    }
    __syncthreads();
    float mt = -INFINITY;
    for (int w = 0; w < 4; ++w) mt = fmaxf(mt, wm[w]);
    float lt = 0.0f;
    float sc[4];
    for (int w = 0; w < 4; ++w) {
        sc[w] = (wl[w] > 0.0f) ? expf(wm[w] - mt) : 0.0f;
        lt += wl[w] * sc[w];
    }
    TO* orow = o + ((int64_t)row * s.H_q + h) * s.d;
    for (int c = threadIdx.x; c < s.d; c += 128) {
        float v = 0.0f;
        for (int w = 0; w < 4; ++w) v += wacc[w][c] * sc[w];
        orow[c] = from_f32<TO>(lt > 0.0f ? v / lt : 0.0f);
    }
}

// ------------------------------------------------------------------ linear attention
__device__ __forceinline__ double feature(int phi, double x) {
    if (phi == LISA_PHI_IDENTITY) return x;
    return x > 0.0 ? x + 1.0 : exp(x);
}

// One block per (sequence, KV head, slice of 32 value columns); 8 row groups x
// 32 columns.  The state slice is kept in fp64 in shared memory for the whole
// token loop (the fp32 workload's tolerance needs it: identity-feature outputs
// grow like sqrt(d * n) with N(0,1) inputs), and written back as float32.
template <typename T, typename TO>
__global__ void __launch_bounds__(256) k_linear(Shape s, const T* __restrict__ q_L,
                                                const T* __restrict__ k_L,
                                                const T* __restrict__ v_L, float* __restrict__ S,
                                                float* __restrict__ z, TO* __restrict__ o) {
    extern __shared__ double dsm[];
    const int d = s.d;
    double* Ss = dsm;                 // [d][32]
    double* fk = Ss + d * 32;         // [d]
    double* fq = fk + d;              // [d]
    double* zs = fq + d;              // [d]
    double* red = zs + d;             // [8][32]
    double* vv = red + 8 * 32;        // [32]
    double* den = vv + 32;            // [1]
    const int b = blockIdx.x, g = blockIdx.y;
    const int col0 = blockIdx.z * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int col = col0 + tx;
    const bool col_ok = col < d;
    float* Sg = S + ((int64_t)b * s.H_kv + g) * d * d;
    float* zg = z ? z + ((int64_t)b * s.H_kv + g) * d : nullptr;
    const bool norm = s.phi == LISA_PHI_ELU1_NORM;
    for (int i = ty; i < d; i += 8) Ss[i * 32 + tx] = col_ok ? (double)Sg[(int64_t)i * d + col] : 0.0;
    for (int i = threadIdx.x; i < d; i += 256) zs[i] = norm ? (double)zg[i] : 0.0;
    __syncthreads();
    for (int t = 0; t < s.T; ++t) {
        const T* kt = k_L + (((int64_t)b * s.T + t) * s.H_kv + g) * d;
        const T* vt = v_L + (((int64_t)b * s.T + t) * s.H_kv + g) * d;
        for (int i = threadIdx.x; i < d; i += 256) fk[i] = feature(s.phi, (double)to_f32(kt[i]));
        if (threadIdx.x < 32) vv[tx] = col_ok ? (double)to_f32(vt[col]) : 0.0;
        __syncthreads();
        for (int i = ty; i < d; i += 8) Ss[i * 32 + tx] += fk[i] * vv[tx];
        if (norm)
            for (int i = threadIdx.x; i < d; i += 256) zs[i] += fk[i];
        __syncthreads();
        for (int hh = 0; hh < s.group; ++hh) {
            const int h = g * s.group + hh;
            const T* qt = q_L + (((int64_t)b * s.T + t) * s.H_q + h) * d;
            for (int i = threadIdx.x; i < d; i += 256) fq[i] = feature(s.phi, (double)to_f32(qt[i]));
            __syncthreads();
            double part = 0.0;
            for (int i = ty; i < d; i += 8) part += fq[i] * Ss[i * 32 + tx];
            red[ty * 32 + tx] = part;
            if (norm && ty == 0) {
                double dz = 0.0;
                for (int i = tx; i < d; i += 32) dz += fq[i] * zs[i];
                for (int off = 16; off > 0; off >>= 1) dz += __shfl_xor_sync(0xffffffffu, dz, off);
                if (tx == 0) den[0] = dz;
            }
            __syncthreads();
            if (ty == 0 && col_ok) {
                double num = 0.0;
                for (int r = 0; r < 8; ++r) num += red[r * 32 + tx];
                const double val = norm ? num / den[0] : num;
                o[(((int64_t)b * s.T + t) * s.H_q + h) * d + col] = from_f32<TO>((float)val);
            }
            __syncthreads();
        }
    }
    for (int i = ty; i < d; i += 8)
        if (col_ok) Sg[(int64_t)i * d + col] = (float)Ss[i * 32 + tx];
    if (norm && blockIdx.z == 0)
        for (int i = threadIdx.x; i < d; i += 256) zg[i] = (float)zs[i];
}

// ------------------------------------------------------------------ gate, append
template <typename TL, typename TA, typename TB, typename TO>
__global__ void k_gate(int64_t n_out, int d, const TL* __restrict__ logit,
                       const TA* __restrict__ o_lin, const TB* __restrict__ o_sp,
                       TO* __restrict__ o) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_out) return;
    const float x = to_f32(logit[i / d]);
    const float g = 1.0f / (1.0f + expf(-x));
    const float a = to_f32(o_lin[i]), c = to_f32(o_sp[i]);
    o[i] = from_f32<TO>(g * a + (1.0f - g) * c);
}

template <typename T>
__global__ void k_append(int B, int n_past, int N_max, int width_kv, int width_kI,
                         const T* __restrict__ k_new, const T* __restrict__ v_new,
                         const T* __restrict__ kI_new, T* __restrict__ kc, T* __restrict__ vc,
                         T* __restrict__ kIc) {
    const int b = blockIdx.x;
    const int64_t dst_kv = ((int64_t)b * N_max + n_past) * width_kv;
    const int64_t dst_kI = ((int64_t)b * N_max + n_past) * width_kI;
    for (int i = threadIdx.x; i < width_kv; i += blockDim.x) {
        kc[dst_kv + i] = k_new[(int64_t)b * width_kv + i];
        vc[dst_kv + i] = v_new[(int64_t)b * width_kv + i];
    }
    for (int i = threadIdx.x; i < width_kI; i += blockDim.x)
        kIc[dst_kI + i] = kI_new[(int64_t)b * width_kI + i];
}

// Sliding-window rows (Sec. 3.2, Stage 1): token t at position p = n_past + t
// keeps [max(0, p-M+1), p] in ascending order, -1 padded.
__global__ void k_window_indices(int64_t rows, int T, int n_past, int M, int32_t* __restrict__ idx,
                                 int32_t* __restrict__ count) {
    const int64_t row = blockIdx.x;
    if (row >= rows) return;
    const int p = n_past + (int)(row % T);
    const int first = max(0, p - M + 1);
    const int c = p - first + 1;
    for (int i = threadIdx.x; i < M; i += blockDim.x) idx[row * M + i] = i < c ? first + i : -1;
    if (threadIdx.x == 0) count[row] = c;
}

}  // namespace

cudaError_t generic_window_indices(const Shape& s, int32_t* idx, int32_t* count, cudaStream_t st) {
    const int64_t rows = (int64_t)s.B * s.T;
    if (rows == 0) return cudaSuccess;
    k_window_indices<<<(unsigned)rows, 128, 0, st>>>(rows, s.T, s.n_past, s.M, idx, count);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ launchers
cudaError_t generic_index_scores(const Shape& s, const void* q_I, const void* k_I, const float* w,
                                 int64_t w_tok_stride, float* scores, cudaStream_t st) {
    const int rows = s.B * s.T;
    if (rows == 0 || s.L == 0) return cudaSuccess;
    if ((s.L + 127) / 128 > 65535) return cudaErrorInvalidValue;  // key blocks on y
    dim3 grid(rows, (s.L + 127) / 128);
    const size_t smem = sizeof(float) * (s.H_I * s.d_I + s.H_I);
    if (s.dtype == LISA_BF16)
        k_index_scores<__nv_bfloat16><<<grid, 128, smem, st>>>(
            s, (const __nv_bfloat16*)q_I, (const __nv_bfloat16*)k_I, w, w_tok_stride, scores);
    else
        k_index_scores<float><<<grid, 128, smem, st>>>(s, (const float*)q_I, (const float*)k_I, w,
                                                       w_tok_stride, scores);
    return cudaGetLastError();
}

cudaError_t generic_topm_from_scores(const Shape& s, const float* scores, int32_t* idx,
                                     int32_t* count, cudaStream_t st) {
    const int rows = s.B * s.T;
    if (rows == 0) return cudaSuccess;
    k_topm_rows<1024><<<rows, 1024, 0, st>>>(s, scores, idx, count);
    return cudaGetLastError();
}

cudaError_t generic_attention(const Shape& s, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* idx, const int32_t* count,
                              void* o, bool o_f32, unsigned* status, cudaStream_t st) {
    const int rows = s.B * s.T;
    if (rows == 0 || s.H_q == 0) return cudaSuccess;
    dim3 grid(rows, s.H_q);
    if (s.dtype == LISA_BF16) {
        using T = __nv_bfloat16;
        if (o_f32)
            k_attention<T, float><<<grid, 128, 0, st>>>(s, (const T*)q, (const T*)k_cache,
                                                        (const T*)v_cache, idx, count, (float*)o,
                                                        status);
        else
            k_attention<T, T><<<grid, 128, 0, st>>>(s, (const T*)q, (const T*)k_cache,
                                                    (const T*)v_cache, idx, count, (T*)o, status);
    } else {
        k_attention<float, float><<<grid, 128, 0, st>>>(s, (const float*)q, (const float*)k_cache,
                                                        (const float*)v_cache, idx, count,
                                                        (float*)o, status);
    }
    return cudaGetLastError();
}

cudaError_t generic_linear(const Shape& s, const void* q_L, const void* k_L, const void* v_L,
                           float* S, float* z, void* o, bool o_f32, cudaStream_t st) {
    if (s.B == 0 || s.T == 0) return cudaSuccess;
    dim3 grid(s.B, s.H_kv, (s.d + 31) / 32);
    const size_t smem = sizeof(double) * (s.d * 32 + 3 * s.d + 8 * 32 + 32 + 1);
    if (s.dtype == LISA_BF16) {
        using T = __nv_bfloat16;
        if (o_f32) {
            auto kern = k_linear<T, float>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            kern<<<grid, 256, smem, st>>>(s, (const T*)q_L, (const T*)k_L, (const T*)v_L, S, z,
                                          (float*)o);
        } else {
            auto kern = k_linear<T, T>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            kern<<<grid, 256, smem, st>>>(s, (const T*)q_L, (const T*)k_L, (const T*)v_L, S, z,
                                          (T*)o);
        }
    } else {
        auto kern = k_linear<float, float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<grid, 256, smem, st>>>(s, (const float*)q_L, (const float*)k_L, (const float*)v_L,
                                      S, z, (float*)o);
    }
    return cudaGetLastError();
}

cudaError_t generic_gate(const Shape& s, const void* logit, const void* o_lin, bool lin_f32,
                         const void* o_sp, bool sp_f32, void* o, cudaStream_t st) {
    const int64_t n = (int64_t)s.B * s.T * s.H_q * s.d;
    if (n == 0) return cudaSuccess;
    const int blocks = (int)((n + 255) / 256);
    if (s.dtype == LISA_BF16) {
        using T = __nv_bfloat16;
        const T* lg = (const T*)logit;
        if (lin_f32 && sp_f32)
            k_gate<<<blocks, 256, 0, st>>>(n, s.d, lg, (const float*)o_lin, (const float*)o_sp, (T*)o);
        else if (!lin_f32 && !sp_f32)
            k_gate<<<blocks, 256, 0, st>>>(n, s.d, lg, (const T*)o_lin, (const T*)o_sp, (T*)o);
        else if (lin_f32)
            k_gate<<<blocks, 256, 0, st>>>(n, s.d, lg, (const float*)o_lin, (const T*)o_sp, (T*)o);
        else
            k_gate<<<blocks, 256, 0, st>>>(n, s.d, lg, (const T*)o_lin, (const float*)o_sp, (T*)o);
    } else {
        k_gate<<<blocks, 256, 0, st>>>(n, s.d, (const float*)logit, (const float*)o_lin,
                                       (const float*)o_sp, (float*)o);
    }
    return cudaGetLastError();
}

cudaError_t generic_append(const Shape& s, const void* k_new, const void* v_new,
                           const void* k_I_new, void* k_cache, void* v_cache, void* k_I_cache,
                           cudaStream_t st) {
    if (s.B == 0) return cudaSuccess;
    const int wkv = s.H_kv * s.d, wkI = (k_I_new && k_I_cache) ? s.H_Ik * s.d_I : 0;
    if (s.dtype == LISA_BF16) {
        using T = __nv_bfloat16;
        k_append<T><<<s.B, 256, 0, st>>>(s.B, s.n_past, s.N_max, wkv, wkI, (const T*)k_new,
                                         (const T*)v_new, (const T*)k_I_new, (T*)k_cache,
                                         (T*)v_cache, (T*)k_I_cache);
    } else {
        k_append<float><<<s.B, 256, 0, st>>>(s.B, s.n_past, s.N_max, wkv, wkI,
                                             (const float*)k_new, (const float*)v_new,
                                             (const float*)k_I_new, (float*)k_cache,
                                             (float*)v_cache, (float*)k_I_cache);
    }
    return cudaGetLastError();
}

}  // namespace lisa
