// Chunked linear-attention prefill on B200 tensor cores (LISA, arXiv
// 2607.19358v1: the linear branch of Sec. 3.1 and Sec. 3.3 Eq. 3-4, inclusive
// of the current token).  With chunks of C = 64 tokens and S_{c-1} the state
// before chunk c:
//   O_c = phi(Q_c) S_{c-1} + tril(phi(Q_c) phi(K_c)^T) V_c
//   S_c = S_{c-1} + phi(K_c)^T V_c
// (elu+1 mode: the same for the normaliser, z_c = z_{c-1} + sum phi(K_c), and
// O_c is divided row-wise by phi(Q_c) z_{c-1} + rowsum(tril(phi(Q_c) phi(K_c)^T)).)
//
// k_la_chunk_sums  (B x H_kv x chunks CTAs): U_c = phi(K_c)^T V_c in fp32
//                   (mma m16n8k16, bf16 operands), and sum_t phi(K_c) for z.
// k_la_prefix      (one thread per state element): U_c <- S_0 + sum_{c'<c} U_c'
//                   in place; the final state goes to S (and z).
// k_la_chunk_out   (B x H_kv x chunks CTAs, two query heads at a time): the
//                   inter-chunk term uses the fp32 prefix state split into two
//                   bf16 halves (hi + lo), so it keeps ~16 bits of mantissa;
//                   the intra-chunk term applies the inclusive causal mask.
#include <math.h>

#include "lisa_fast.cuh"
#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kD = 128;
constexpr int kC = 64;                 // chunk length of this path
constexpr int kRow = kD * 2 + 16;      // padded shared-memory row (bytes) of 128 bf16

struct LaParams {
    int B, T, H_q, H_kv, group, phi, nch;
    const bf16* q;
    const bf16* k;
    const bf16* v;
    float* S;
    float* z;
    bf16* o;
    float* U;      // workspace [B][H_kv][nch][128][128]
    float* Z;      // workspace [B][H_kv][nch][128]
};

__device__ __forceinline__ float feat(int phi, float x) {
    if (phi == LISA_PHI_IDENTITY) return x;
    return x > 0.0f ? x + 1.0f : __expf(x);
}

// Loads rows [t0, t0 + 64) of one head (row stride `stride` elements) into
// padded shared memory as bf16 (rows past T are zero).  mode 0: values as
// given; 1: phi(x); 2: phi(x) - 1, which bf16 holds far more accurately than
// phi(x) itself in the elu+1 map (phi(x) is close to 1 for small x).
__device__ __forceinline__ void load_rows(uint8_t* dst, const bf16* src, int64_t stride, int t0,
                                          int T, int phi, int mode, int nthreads) {
    for (int e = threadIdx.x; e < kC * (kD / 8); e += nthreads) {
        const int r = e / (kD / 8), c8 = e % (kD / 8);
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        const bool valid = t0 + r < T;
        if (valid) u = *reinterpret_cast<const uint4*>(src + (int64_t)(t0 + r) * stride + c8 * 8);
        if (mode != 0 && phi != LISA_PHI_IDENTITY && valid) {
            const float sub = mode == 2 ? 1.0f : 0.0f;
            __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const float2 f = __bfloat1622float2(h2[x]);
                const float a = f.x > 0.0f ? f.x + (1.0f - sub) : (mode == 2 ? expm1f(f.x) : __expf(f.x));
                const float c = f.y > 0.0f ? f.y + (1.0f - sub) : (mode == 2 ? expm1f(f.y) : __expf(f.y));
                h2[x] = __floats2bfloat162_rn(a, c);
            }
        }
        *reinterpret_cast<uint4*>(dst + r * kRow + c8 * 16) = u;
    }
}

// ---------------------------------------------------------------- chunk sums
__global__ void __launch_bounds__(256) k_la_chunk_sums(const LaParams P) {
    __shared__ __align__(128) uint8_t ks[kC * kRow];
    __shared__ __align__(128) uint8_t vs[kC * kRow];
    const int c = blockIdx.x % P.nch, g = (blockIdx.x / P.nch) % P.H_kv, b = blockIdx.x / (P.nch * P.H_kv);
    const int t0 = c * kC;
    const int64_t rs = (int64_t)P.H_kv * kD;
    const bool norm = P.phi == LISA_PHI_ELU1_NORM;
    // elu+1: the tensor cores see phi(K) - 1; U = (phi(K) - 1)^T V + 1 (x) sum_t V[t]
    load_rows(ks, P.k + ((int64_t)b * P.T * P.H_kv + g) * kD, rs, t0, P.T, P.phi, 2, 256);
    load_rows(vs, P.v + ((int64_t)b * P.T * P.H_kv + g) * kD, rs, t0, P.T, P.phi, 0, 256);
    __shared__ float vsum[kD];
    __syncthreads();
    if (norm && threadIdx.x < kD) {
        float a = 0.0f;
        for (int t = 0; t < kC; ++t)
            a += __bfloat162float(*reinterpret_cast<const bf16*>(vs + t * kRow + threadIdx.x * 2));
        vsum[threadIdx.x] = a;
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const int m0 = warp * 16;  // key-feature rows of this warp
    float acc[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] = 0.0f;
    const uint32_t kb = ptx::smem_u32(ks), vb = ptx::smem_u32(vs);
#pragma unroll
    for (int kt = 0; kt < kC / 16; ++kt) {
        // A = phi(K)^T (rows = features, cols = tokens) from K rows via transposed ldmatrix
        uint32_t a[4];
        {
            const int j = lane >> 3;
            const int t = kt * 16 + (j >> 1) * 8 + (lane & 7);
            const int f = m0 + (j & 1) * 8;
            ptx::ldmatrix_x4_trans(a, kb + t * kRow + f * 2);
        }
#pragma unroll
        for (int n = 0; n < 16; n += 2) {
            uint32_t vr[4];
            const int t = kt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
            const int f = (n + (lane >> 4)) * 8;
            ptx::ldmatrix_x4_trans(vr, vb + t * kRow + f * 2);
            ptx::mma_bf16(acc[n], a, vr[0], vr[1]);
            ptx::mma_bf16(acc[n + 1], a, vr[2], vr[3]);
        }
    }
    float* U = P.U + (((int64_t)b * P.H_kv + g) * P.nch + c) * kD * kD;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const int col = n * 8 + 2 * tq;
        const float r0 = norm ? vsum[col] : 0.0f, r1 = norm ? vsum[col + 1] : 0.0f;
        *reinterpret_cast<float2*>(U + (m0 + gid) * kD + col) = make_float2(acc[n][0] + r0, acc[n][1] + r1);
        *reinterpret_cast<float2*>(U + (m0 + gid + 8) * kD + col) = make_float2(acc[n][2] + r0, acc[n][3] + r1);
    }
    if (norm && threadIdx.x < kD) {
        // sum_t phi(k_t) = sum_t (phi(k_t) - 1) + (valid tokens of the chunk)
        float zs = (float)min(kC, P.T - t0);
        for (int t = 0; t < kC; ++t)
            zs += __bfloat162float(*reinterpret_cast<const bf16*>(ks + t * kRow + threadIdx.x * 2));
        P.Z[(((int64_t)b * P.H_kv + g) * P.nch + c) * kD + threadIdx.x] = zs;
    }
}

// ---------------------------------------------------------------- prefix over chunks
__global__ void __launch_bounds__(256) k_la_prefix(const LaParams P) {
    const int64_t per = (int64_t)kD * kD;
    const int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const int64_t nstate = (int64_t)P.B * P.H_kv * per;
    if (e < nstate) {
        const int64_t bg = e / per, el = e % per;
        float run = P.S[e];
        float* U = P.U + bg * P.nch * per + el;
        int c = 0;
        for (; c + 8 <= P.nch; c += 8) {
            float u[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) u[x] = U[(int64_t)(c + x) * per];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                U[(int64_t)(c + x) * per] = run;
                run += u[x];
            }
        }
        for (; c < P.nch; ++c) {
            const float u = U[(int64_t)c * per];
            U[(int64_t)c * per] = run;
            run += u;
        }
        P.S[e] = run;
    }
    if (P.phi == LISA_PHI_ELU1_NORM && e < (int64_t)P.B * P.H_kv * kD) {
        const int64_t bg = e / kD, el = e % kD;
        float run = P.z[e];
        float* Z = P.Z + bg * P.nch * kD + el;
        for (int c = 0; c < P.nch; ++c) {
            const float u = Z[(int64_t)c * kD];
            Z[(int64_t)c * kD] = run;
            run += u;
        }
        P.z[e] = run;
    }
}

// ---------------------------------------------------------------- chunk outputs
struct OutSmem {
    static constexpr int shi = 0;                      // S_{c-1} high half, bf16 [128][128]
    static constexpr int slo = shi + kD * kRow;        // low half
    static constexpr int k = slo + kD * kRow;          // phi(K_c) [64][128]
    static constexpr int v = k + kC * kRow;            // V_c
    static constexpr int q = v + kC * kRow;            // phi(Q_c) of two heads [2][64][128]
    static constexpr int zc = q + 2 * kC * kRow;       // z_{c-1} float[128]
    static constexpr int total = zc + kD * 4;
};

__global__ void __launch_bounds__(256, 1) k_la_chunk_out(const LaParams P) {
    extern __shared__ __align__(128) uint8_t la_raw[];
    const int c = blockIdx.x % P.nch, g = (blockIdx.x / P.nch) % P.H_kv, b = blockIdx.x / (P.nch * P.H_kv);
    const int t0 = c * kC;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const bool norm = P.phi == LISA_PHI_ELU1_NORM;
    // prefix state of this chunk, split into bf16 hi + lo
    const float* Sp = P.U + (((int64_t)b * P.H_kv + g) * P.nch + c) * kD * kD;
    for (int e = tid; e < kD * kD / 2; e += 256) {
        const int r = e / (kD / 2), c2 = (e % (kD / 2)) * 2;
        const float2 f = *reinterpret_cast<const float2*>(Sp + r * kD + c2);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(f.x, f.y);
        const float2 hf = __bfloat1622float2(hi);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(f.x - hf.x, f.y - hf.y);
        *reinterpret_cast<__nv_bfloat162*>(la_raw + OutSmem::shi + r * kRow + c2 * 2) = hi;
        *reinterpret_cast<__nv_bfloat162*>(la_raw + OutSmem::slo + r * kRow + c2 * 2) = lo;
    }
    const int64_t rs_kv = (int64_t)P.H_kv * kD;
    load_rows(la_raw + OutSmem::k, P.k + ((int64_t)b * P.T * P.H_kv + g) * kD, rs_kv, t0, P.T, P.phi, 1, 256);
    load_rows(la_raw + OutSmem::v, P.v + ((int64_t)b * P.T * P.H_kv + g) * kD, rs_kv, t0, P.T, P.phi, 0, 256);
    float* zc = reinterpret_cast<float*>(la_raw + OutSmem::zc);
    if (norm && tid < kD) zc[tid] = P.Z[(((int64_t)b * P.H_kv + g) * P.nch + c) * kD + tid];
    const uint32_t shi = ptx::smem_u32(la_raw + OutSmem::shi), slo = ptx::smem_u32(la_raw + OutSmem::slo);
    const uint32_t kbase = ptx::smem_u32(la_raw + OutSmem::k), vbase = ptx::smem_u32(la_raw + OutSmem::v);
    const int half = warp >> 2;          // which of the two heads
    const int r0 = (warp & 3) * 16;      // query rows of this warp within the chunk
    const int64_t rs_q = (int64_t)P.H_q * kD;
    for (int hp = 0; hp < P.group; hp += 2) {
        __syncthreads();  // previous pair finished with the query buffer
        for (int x = 0; x < 2; ++x)
            if (hp + x < P.group)
                load_rows(la_raw + OutSmem::q + x * kC * kRow,
                          P.q + ((int64_t)b * P.T * P.H_q + g * P.group + hp + x) * kD, rs_q, t0,
                          P.T, P.phi, 1, 256);
        __syncthreads();
        const int h = hp + half;
        if (h >= P.group) continue;
        const uint32_t qb = ptx::smem_u32(la_raw + OutSmem::q + half * kC * kRow);
        float o[16][4];
#pragma unroll
        for (int n = 0; n < 16; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[n][e] = 0.0f;
        float sc[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[n][e] = 0.0f;
        float qz[2] = {0.0f, 0.0f};  // phi(q) . z_{c-1} of rows gid, gid + 8
#pragma unroll 2
        for (int ks = 0; ks < kD / 16; ++ks) {
            uint32_t a[4];
            {
                const int row = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = ks * 16 + (lane >> 4) * 8;
                ptx::ldmatrix_x4(a, qb + row * kRow + col * 2);
            }
            // inter-chunk: phi(Q) S_{c-1}, both halves of S
#pragma unroll
            for (int n = 0; n < 16; n += 2) {
                uint32_t br[4];
                const int kr = ks * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                const int col = (n + (lane >> 4)) * 8;
                ptx::ldmatrix_x4_trans(br, shi + kr * kRow + col * 2);
                ptx::mma_bf16(o[n], a, br[0], br[1]);
                ptx::mma_bf16(o[n + 1], a, br[2], br[3]);
                ptx::ldmatrix_x4_trans(br, slo + kr * kRow + col * 2);
                ptx::mma_bf16(o[n], a, br[0], br[1]);
                ptx::mma_bf16(o[n + 1], a, br[2], br[3]);
            }
            // intra-chunk scores: phi(Q) phi(K)^T over the chunk's 64 keys
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                uint32_t kr2[2];
                {
                    uint32_t kr4[4];
                    const int key = n * 8 + (lane & 7);
                    const int col = ks * 16 + ((lane >> 3) & 1) * 8;
                    ptx::ldmatrix_x4(kr4, kbase + key * kRow + col * 2);
                    kr2[0] = kr4[0];
                    kr2[1] = kr4[1];
                }
                ptx::mma_bf16(sc[n], a, kr2[0], kr2[1]);
            }
        }
        if (norm) {
            // phi(q) . z_{c-1} for rows r0 + gid and r0 + gid + 8, from shared memory
            const uint8_t* qrow0 = la_raw + OutSmem::q + half * kC * kRow + (r0 + gid) * kRow;
            const uint8_t* qrow1 = qrow0 + 8 * kRow;
            for (int f = tq; f < kD; f += 4) {
                qz[0] = fmaf(__bfloat162float(*reinterpret_cast<const bf16*>(qrow0 + f * 2)), zc[f], qz[0]);
                qz[1] = fmaf(__bfloat162float(*reinterpret_cast<const bf16*>(qrow1 + f * 2)), zc[f], qz[1]);
            }
            qz[0] += __shfl_xor_sync(0xffffffffu, qz[0], 1);
            qz[0] += __shfl_xor_sync(0xffffffffu, qz[0], 2);
            qz[1] += __shfl_xor_sync(0xffffffffu, qz[1], 1);
            qz[1] += __shfl_xor_sync(0xffffffffu, qz[1], 2);
        }
        // inclusive causal mask inside the chunk, row sums for the normaliser
        float rsum[2] = {0.0f, 0.0f};
        uint32_t pa[4][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int qi = r0 + gid + 8 * (e >> 1);
                const int kj = n * 8 + 2 * tq + (e & 1);
                if (kj > qi) sc[n][e] = 0.0f;
                rsum[e >> 1] += sc[n][e];
            }
            const int kk = n >> 1, hi2 = n & 1;
            pa[kk][0 + 2 * hi2] = ptx::pack_bf16(sc[n][0], sc[n][1]);
            pa[kk][1 + 2 * hi2] = ptx::pack_bf16(sc[n][2], sc[n][3]);
        }
        // + tril(phi(Q) phi(K)^T) V
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk) {
#pragma unroll
            for (int n = 0; n < 16; n += 2) {
                uint32_t vr[4];
                const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                const int col = (n + (lane >> 4)) * 8;
                ptx::ldmatrix_x4_trans(vr, vbase + key * kRow + col * 2);
                ptx::mma_bf16(o[n], pa[kk], vr[0], vr[1]);
                ptx::mma_bf16(o[n + 1], pa[kk], vr[2], vr[3]);
            }
        }
        float inv[2] = {1.0f, 1.0f};
        if (norm) {
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                rsum[x] += __shfl_xor_sync(0xffffffffu, rsum[x], 1);
                rsum[x] += __shfl_xor_sync(0xffffffffu, rsum[x], 2);
                inv[x] = 1.0f / (qz[x] + rsum[x]);
            }
        }
        const int hq = g * P.group + h;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int t = t0 + r0 + gid + 8 * x;
            if (t >= P.T) continue;
            bf16* orow = P.o + (((int64_t)b * P.T + t) * P.H_q + hq) * kD;
#pragma unroll
            for (int n = 0; n < 16; ++n)
                *reinterpret_cast<__nv_bfloat162*>(orow + n * 8 + 2 * tq) =
                    __floats2bfloat162_rn(o[n][2 * x] * inv[x], o[n][2 * x + 1] * inv[x]);
        }
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

size_t fast_linear_prefill_ws_bytes(const Shape& s) {
    const size_t nch = (size_t)((s.T + kC - 1) / kC);
    return kStatusBytes + sizeof(float) * (size_t)s.B * s.H_kv * nch * (kD * kD + kD) + 512;
}

bool fast_linear_prefill_supported(const Shape& s, const void* q, const void* k, const void* v) {
    if (s.dtype != LISA_BF16 || s.d != kD || s.chunk != kC) return false;
    if (s.T < 1 || s.group > 64) return false;
    return aligned16(q) && aligned16(k) && aligned16(v);
}

cudaError_t fast_linear_prefill(const Shape& s, const void* q, const void* k, const void* v,
                                float* S, float* z, void* o, void* ws, cudaStream_t st) {
    LaParams P;
    P.B = s.B; P.T = s.T; P.H_q = s.H_q; P.H_kv = s.H_kv; P.group = s.group; P.phi = s.phi;
    P.nch = (s.T + kC - 1) / kC;
    P.q = (const bf16*)q; P.k = (const bf16*)k; P.v = (const bf16*)v;
    P.S = S; P.z = z; P.o = (bf16*)o;
    char* w8 = (char*)ws + kStatusBytes;
    P.U = (float*)w8;
    P.Z = P.U + (size_t)s.B * s.H_kv * P.nch * kD * kD;
    static bool attrs[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_la_chunk_out, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             OutSmem::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    const int ctas = s.B * s.H_kv * P.nch;
    k_la_chunk_sums<<<ctas, 256, 0, st>>>(P);
    const int64_t nstate = (int64_t)s.B * s.H_kv * kD * kD;
    k_la_prefix<<<(unsigned)((nstate + 255) / 256), 256, 0, st>>>(P);
    k_la_chunk_out<<<ctas, 256, OutSmem::total, st>>>(P);
    return cudaGetLastError();
}

}  // namespace lisa
