// Sparse softmax attention over given index lists (lisa_sparse_attn) for many
// query rows, bf16, head dim 128: one CTA per query row runs the gather (K rows
// by 1-D bulk copies, V rows by 16-byte cp.async) and tensor-core online
// softmax of attend_core.cuh over the row's count[b,t] positions and writes
// the normalised output (LISA, arXiv 2607.19358v1,
// Sec. 3.2 Eq. 1, the SA_M branch).  Positions outside [0, p] are masked out
// and reported as LISA_ERR_DEVICE_BOUNDS through the status word.
#include <algorithm>

#include "attend_core.cuh"
#include "lisa_fast.cuh"
#include "lisa_internal.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;
struct SpParams {
    int B, T, n_past, N_max, H_q, group, M;
    float scale_log2;
    const bf16* q;
    const bf16* k;
    const bf16* v;
    const int32_t* idx;
    const int32_t* count;
    bf16* o;
    unsigned* status;
};

template <int HKV>
struct SpSmem {
    static constexpr int spos = 0;                                     // int[stages][keys]
    static constexpr int ring = (kAttStages * AttGeo<HKV>::keys * 4 + 127) / 128 * 128;
    static constexpr int kbar = ring + AttGeo<HKV>::ring_bytes;        // uint64[kAttStages]
    static constexpr int total = kbar + kAttStages * 8;
    static_assert(total <= 227 * 1024, "shared memory per CTA");
};

template <int HKV>
__global__ void __launch_bounds__(kAttThreads, 1) k_sparse_rows(const SpParams P) {
    using L = SpSmem<HKV>;
    extern __shared__ __align__(128) uint8_t sp_raw[];
    int* spos = reinterpret_cast<int*>(sp_raw + L::spos);
    const int row = blockIdx.x;
    const int b = row / P.T, t = row % P.T;
    const int p = P.n_past + t;
    const int cnt = max(0, min(P.count[row], P.M));
    const int* pos = P.idx + (int64_t)row * P.M;  // read through L1 by the gather
    const AttQ q = attn_load_q<HKV>(P.q + (int64_t)row * P.H_q * 128, P.group);
    AttOut r;
    const AttSrc kv{P.k, P.v, (int64_t)b * P.N_max, p, -1, nullptr, nullptr};
    attn_core<HKV, true>(q, sp_raw + L::ring, spos, pos, cnt, kv, P.scale_log2, P.status, r,
                         reinterpret_cast<uint64_t*>(sp_raw + L::kbar));
    // normalised output of each KV head's query heads (group rows of 128 dims,
    // contiguous in o), staged by the head's first warp in its own slot of the
    // ring and stored with 16-byte writes
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp % AttGeo<HKV>::wph != 0) return;
    const int g = warp / AttGeo<HKV>::wph, gid = lane >> 2, tq = lane & 3;
    bf16* stage = reinterpret_cast<bf16*>(sp_raw + L::ring) + warp * 36 * 32 * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int slot = 2 * tq + h;
        if (slot >= P.group) continue;
        const float inv = r.l[h] > 0.0f ? 1.0f / r.l[h] : 0.0f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            stage[slot * 128 + t * 16 + gid] = __float2bfloat16_rn(r.o[t][h] * inv);
            stage[slot * 128 + t * 16 + gid + 8] = __float2bfloat16_rn(r.o[t][h + 2] * inv);
        }
    }
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(P.o + ((int64_t)row * P.H_q + g * P.group) * 128);
    const uint4* src = reinterpret_cast<const uint4*>(stage);
    for (int c = lane; c < P.group * 16; c += 32) dst[c] = src[c];
}

// Dense causal attention (the O(n) reference line): the causal range [0, p]
// of each query row is split over `nsplit` CTAs; each runs the attention core
// over its run of positions and writes the partial state (base-2 max, sum,
// un-normalised output) of every query head; k_dense_combine merges them.
struct DenseParams {
    int T, n_past, N_max, H_q, group, nsplit;
    float scale_log2;
    const bf16* q;
    const bf16* k;
    const bf16* v;
    float* part;  // [rows][nsplit][H_q][130]
    bf16* o;
    unsigned* status;
};

template <int HKV>
__global__ void __launch_bounds__(kAttThreads, 1) k_dense_split(const DenseParams P) {
    using L = SpSmem<HKV>;
    extern __shared__ __align__(128) uint8_t sp_raw[];
    int* spos = reinterpret_cast<int*>(sp_raw + L::spos);
    const int row = blockIdx.x / P.nsplit, sp = blockIdx.x % P.nsplit;
    const int b = row / P.T, t = row % P.T;
    const int p = P.n_past + t;
    const int per = (p + 1 + P.nsplit - 1) / P.nsplit;
    const int k0 = min(p + 1, sp * per);
    const int cnt = min(p + 1, k0 + per) - k0;
    const AttQ q = attn_load_q<HKV>(P.q + (int64_t)row * P.H_q * 128, P.group);
    AttOut r;
    const AttSrc kv{P.k, P.v, (int64_t)b * P.N_max, p, -1, nullptr, nullptr};
    attn_core<HKV, true>(q, sp_raw + L::ring, spos, nullptr, cnt, kv, P.scale_log2, P.status, r,
                         reinterpret_cast<uint64_t*>(sp_raw + L::kbar), k0);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp % AttGeo<HKV>::wph != 0) return;
    const int g = warp / AttGeo<HKV>::wph, gid = lane >> 2, tq = lane & 3;
    float* prow = P.part + (((int64_t)row * P.nsplit + sp) * P.H_q + g * P.group) * 130;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int slot = 2 * tq + h;
        if (slot >= P.group) continue;
        float* rec = prow + (int64_t)slot * 130;
        if (gid == 0) {
            rec[0] = r.m[h];
            rec[1] = r.l[h];
        }
#pragma unroll
        for (int t8 = 0; t8 < 8; ++t8) {
            rec[2 + t8 * 16 + gid] = r.o[t8][h];
            rec[2 + t8 * 16 + gid + 8] = r.o[t8][h + 2];
        }
    }
}

// One CTA of 128 threads (one per dim) per (row, query head).
__global__ void __launch_bounds__(128) k_dense_combine(const DenseParams P) {
    const int row = blockIdx.x / P.H_q, h = blockIdx.x % P.H_q, c = threadIdx.x;
    float Mx = -INFINITY, Ls = 0.0f, O = 0.0f;
    for (int sp = 0; sp < P.nsplit; ++sp) {
        const float* rec = P.part + (((int64_t)row * P.nsplit + sp) * P.H_q + h) * 130;
        const float m = rec[0];
        if (m == -INFINITY) continue;  // an empty split
        const float nm = fmaxf(Mx, m);
        const float a = Mx == -INFINITY ? 0.0f : exp2f(Mx - nm);
        const float w = exp2f(m - nm);
        Ls = Ls * a + rec[1] * w;
        O = O * a + rec[2 + c] * w;
        Mx = nm;
    }
    P.o[((int64_t)row * P.H_q + h) * 128 + c] = __float2bfloat16_rn(Ls > 0.0f ? O / Ls : 0.0f);
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

// Splits of each row's causal range: enough CTAs for two per SM, at least 256
// positions each.
int dense_nsplit(const Shape& s) {
    const int rows = std::max(1, s.B * s.T);
    const int by_sm = (2 * 148 + rows - 1) / rows;
    const int by_len = std::max(1, (s.L + 255) / 256);
    return std::max(1, std::min(by_sm, by_len));
}

}  // namespace

namespace {

cudaError_t dense_attention(const Shape& s, const void* q, const void* k, const void* v, void* o,
                            void* ws, cudaStream_t st) {
    DenseParams P;
    P.T = s.T; P.n_past = s.n_past; P.N_max = s.N_max; P.H_q = s.H_q; P.group = s.group;
    P.nsplit = dense_nsplit(s);
    P.scale_log2 = s.sm_scale * 1.4426950408889634f;
    P.q = (const bf16*)q; P.k = (const bf16*)k; P.v = (const bf16*)v;
    P.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kStatusBytes);
    P.o = (bf16*)o; P.status = (unsigned*)ws;
    static bool attrs[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_dense_split<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<1>::total);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_dense_split<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<2>::total);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_dense_split<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<4>::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    const dim3 grid(s.B * s.T * P.nsplit);
    switch (s.H_kv) {
        case 1: k_dense_split<1><<<grid, kAttThreads, SpSmem<1>::total, st>>>(P); break;
        case 2: k_dense_split<2><<<grid, kAttThreads, SpSmem<2>::total, st>>>(P); break;
        default: k_dense_split<4><<<grid, kAttThreads, SpSmem<4>::total, st>>>(P); break;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_dense_combine<<<s.B * s.T * s.H_q, 128, 0, st>>>(P);
    return cudaGetLastError();
}

}  // namespace

size_t fast_attention_ws_bytes(const Shape& s, bool dense) {
    if (dense)
        return kStatusBytes + sizeof(float) * (size_t)s.B * s.T * dense_nsplit(s) * s.H_q * 130;
    if (sparse_mask_preferred(s)) return std::max(kStatusBytes, sparse_mask_ws_bytes(s));
    return kStatusBytes;
}

bool fast_attention_supported(const Shape& s, const void* q, const void* k, const void* v,
                              bool dense) {
    (void)dense;  // the dense line runs on the same attention core (split over CTAs)
    if (s.dtype != LISA_BF16 || s.d != 128) return false;
    if (!(s.H_kv == 1 || s.H_kv == 2 || s.H_kv == 4) || s.group > 8) return false;
    return aligned16(q) && aligned16(k) && aligned16(v);
}

cudaError_t fast_attention(const Shape& s, const void* q, const void* k, const void* v,
                           const int32_t* idx, const int32_t* count, void* o, void* ws,
                           cudaStream_t st) {
    if (idx && sparse_mask_supported(s, q, k, v))
        return sparse_mask_attention(s, q, k, v, idx, count, o, ws, st);
    if (!idx) return dense_attention(s, q, k, v, o, ws, st);
    SpParams P;
    P.B = s.B; P.T = s.T; P.n_past = s.n_past; P.N_max = s.N_max; P.H_q = s.H_q;
    P.group = s.group; P.M = s.M; P.scale_log2 = s.sm_scale * 1.4426950408889634f;
    P.q = (const bf16*)q; P.k = (const bf16*)k; P.v = (const bf16*)v;
    P.idx = idx; P.count = count; P.o = (bf16*)o; P.status = (unsigned*)ws;
    static bool attrs[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_sparse_rows<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<1>::total);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_sparse_rows<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<2>::total);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_sparse_rows<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<4>::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    const dim3 grid(s.B * s.T);
    switch (s.H_kv) {
        case 1: k_sparse_rows<1><<<grid, kAttThreads, SpSmem<1>::total, st>>>(P); break;
        case 2: k_sparse_rows<2><<<grid, kAttThreads, SpSmem<2>::total, st>>>(P); break;
        default: k_sparse_rows<4><<<grid, kAttThreads, SpSmem<4>::total, st>>>(P); break;
    }
    return cudaGetLastError();
}

}  // namespace lisa
