// Chunked linear-attention prefill on B200 tensor cores (LISA, arXiv
// 2607.19358v1: the linear branch of Sec. 3.1 and Sec. 3.3 Eq. 3-4, inclusive
// of the current token).  With chunks of C = 64 tokens and S_{c-1} the state
// before chunk c:
//   O_c = phi(Q_c) S_{c-1} + tril(phi(Q_c) phi(K_c)^T) V_c
//   S_c = S_{c-1} + phi(K_c)^T V_c
// (elu+1 mode: the same for the normaliser, z_c = z_{c-1} + sum phi(K_c), and
// O_c is divided row-wise by phi(Q_c) z_{c-1} + rowsum(tril(phi(Q_c) phi(K_c)^T)).)
//
// k_la_sums_tc  (B x H_kv x chunks CTAs): U_c = phi(K_c)^T V_c on tcgen05,
//               operands by TMA, accumulator in TMEM; sum_t phi(K_c) for z.
// k_la_prefix   (one thread per state element): U_c <- S_0 + sum_{c'<c} U_c'
//               in place; the final state goes to S (and z).
// k_la_out_tc   (B x H_kv x chunks CTAs): every product of the chunk's query
//               heads on tcgen05, the inter-chunk term through the fp32 prefix
//               state split into two bf16 halves (hi + lo, ~16 bits kept).
// Every wait is bounded; one that gives up records LISA_ERR_TIMEOUT.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include "lisa_fast.cuh"
#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kD = 128;
constexpr int kC = 64;                 // chunk length of this path
constexpr uint32_t kTries = 1u << 22;  // polls of a bounded wait

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
    unsigned* status;
};

// ---------------------------------------------------------------- chunk sums
// One CTA per (sequence, KV head, chunk): U_c = phi(K_c)^T V_c on the tensor
// cores, M = 128 key features x N = 128 value dims x K = 64 tokens, both
// operands MN-major straight from their TMA tiles (128-byte swizzle).  In the
// elu+1 mode the tile holds phi(K) - 1 (bf16 keeps it far more accurately
// than phi(K), which is near 1 for small keys) and the rank-one rest,
// 1 (x) sum_t V[t], is added in the epilogue; the chunk's sum of phi(k) goes
// to Z.  Thread i reads TMEM lane i (key feature i) and writes row i of U_c.
constexpr int kSumThreads = 128;

__device__ __forceinline__ float elu1_minus1(float x) { return x > 0.0f ? x : expm1f(x); }

// Element (t, c) of a [64 rows][128 cols] bf16 tile held as two TMA boxes of
// 64 columns (128-byte rows, 128-byte swizzle), box b at byte b * 8192.
__device__ __forceinline__ int sw_off64(int t, int c) {
    const int box = c >> 6, cc = c & 63;
    return box * 8192 + t * 128 + ((((cc >> 3) ^ (t & 7)) << 4) | ((cc & 7) << 1));
}

__global__ void __launch_bounds__(kSumThreads, 1)
    k_la_sums_tc(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                 const LaParams P) {
    __shared__ __align__(1024) uint8_t ks[16384];
    __shared__ __align__(1024) uint8_t vs[16384];
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ uint32_t tmem_slot;
    __shared__ float vsum[kD];
    const int c = blockIdx.x % P.nch, g = (blockIdx.x / P.nch) % P.H_kv, b = blockIdx.x / (P.nch * P.H_kv);
    const int t0 = c * kC;
    const int tid = threadIdx.x, warp = tid >> 5;
    const bool norm = P.phi == LISA_PHI_ELU1_NORM;
    if (tid == 0) {
        ptx::mbar_init(&bars[0], 1);
        ptx::mbar_init(&bars[1], 1);
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&tmem_slot, 128);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (tid == 0) {
        ptx::mbar_arrive_expect_tx(&bars[0], 32768);
        ptx::tma_load_3d(ks, &tmap_k, g * kD, t0, b, &bars[0]);
        ptx::tma_load_3d(ks + 8192, &tmap_k, g * kD + 64, t0, b, &bars[0]);
        ptx::tma_load_3d(vs, &tmap_v, g * kD, t0, b, &bars[0]);
        ptx::tma_load_3d(vs + 8192, &tmap_v, g * kD + 64, t0, b, &bars[0]);
    }
    bool ok = __syncthreads_and(ptx::mbar_wait_bounded(&bars[0], 0, kTries));
    const int nvalid = min(kC, P.T - t0);
    float zsum = 0.0f;
    if (ok && norm) {
        // phi(K) - 1 in place (rows past T stay zero), the sum of V per value
        // dim and of phi(k) per key feature (thread = column)
        __nv_bfloat162* kw = reinterpret_cast<__nv_bfloat162*>(ks);
        for (int e = tid; e < 16384 / 4; e += kSumThreads) {
            const int t = ((e * 4) & 8191) >> 7;  // the token row of this word
            if (t < nvalid) {
                const float2 f = __bfloat1622float2(kw[e]);
                kw[e] = __floats2bfloat162_rn(elu1_minus1(f.x), elu1_minus1(f.y));
            }
        }
        float vs_acc = 0.0f;
        for (int t = 0; t < nvalid; ++t)
            vs_acc += __bfloat162float(*reinterpret_cast<const bf16*>(vs + sw_off64(t, tid)));
        vsum[tid] = vs_acc;
        __syncthreads();
        for (int t = 0; t < nvalid; ++t)
            zsum += __bfloat162float(*reinterpret_cast<const bf16*>(ks + sw_off64(t, tid)));
        zsum += (float)nvalid;
        ptx::fence_proxy_async_shared();
    }
    __syncthreads();
    if (tid == 0 && ok) {
        ptx::tc_fence_after();
        // A = phi(K)^T: M = features (contiguous within a box), K = tokens;
        // B = V: N = value dims (contiguous), K = tokens
        const uint32_t idesc = ptx::idesc_bf16_f32_bmn(kD, kD) | (1u << 15);
        const uint64_t ad = ptx::sdesc_mnmajor_sw128(ks, 8192, 1024);
        const uint64_t bd = ptx::sdesc_mnmajor_sw128(vs, 8192, 1024);
#pragma unroll
        for (int kk = 0; kk < kC / 16; ++kk)
            ptx::umma_f16(tmem, ad + (uint64_t)(128 * kk), bd + (uint64_t)(128 * kk), idesc, kk > 0);
        ptx::umma_commit(&bars[1]);
    }
    ok = ok && __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&bars[1], 0, kTries));
    if (!ok) {
        if ((tid & 31) == 0) record_error(P.status, kDevTimeout);
    } else {
        ptx::tc_fence_after();
        const int lb = warp * 32, i = lb + (tid & 31);
        float* U = P.U + (((int64_t)b * P.H_kv + g) * P.nch + c) * kD * kD + (int64_t)i * kD;
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + ((uint32_t)lb << 16) + (uint32_t)c0, r);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                float4 u;
                u.x = __uint_as_float(r[e]) + (norm ? vsum[c0 + e] : 0.0f);
                u.y = __uint_as_float(r[e + 1]) + (norm ? vsum[c0 + e + 1] : 0.0f);
                u.z = __uint_as_float(r[e + 2]) + (norm ? vsum[c0 + e + 2] : 0.0f);
                u.w = __uint_as_float(r[e + 3]) + (norm ? vsum[c0 + e + 3] : 0.0f);
                *reinterpret_cast<float4*>(U + c0 + e) = u;
            }
        }
        if (norm) P.Z[(((int64_t)b * P.H_kv + g) * P.nch + c) * kD + tid] = zsum;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 0) ptx::tmem_dealloc(tmem, 128);
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
        for (; c + 16 <= P.nch; c += 16) {  // 16 loads in flight per thread
            float u[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) u[x] = __ldcg(U + (int64_t)(c + x) * per);
#pragma unroll
            for (int x = 0; x < 16; ++x) {
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
// One CTA per (sequence, KV head, chunk).  The group's query heads go two at a
// time through 128-row tiles (rows 0-63: the chunk's tokens of head 2m, rows
// 64-127: of head 2m + 1), all products on the tensor cores with the
// accumulators in TMEM:
//   O  = phi(Q) S_hi + phi(Q) S_lo       (M = 128, N = 128, K = 128 features;
//                                          S_{c-1} split into two bf16 halves,
//                                          MN-major, so ~16 bits are kept)
//   Si = phi(Q) phi(K_c)^T                (N = 64 tokens)
//   O += tril(Si) V_c                     (K = 64 tokens, V MN-major from TMA)
// Warp 0 brings K_c, V_c and the query tiles by TMA (two query buffers);
// warp 1 owns TMEM (two O and two Si buffers) and issues the MMAs; warps 2-5
// (thread = tile row = TMEM lane) write the two halves of S_{c-1}, apply phi
// in the elu+1 mode, mask Si causally into P (bf16, shared memory), and
// write O (divided by phi(q) . z_{c-1} + the row sum of tril(Si) in the elu+1
// mode) as bf16.
constexpr int kOutThreads = 192;

struct OutSmem {
    static constexpr int shi = 0;                 // 2 blocks of 128 features x 64 dims (MN-major)
    static constexpr int slo = shi + 32768;
    static constexpr int k = slo + 32768;         // K_c: 2 boxes of 64 features x 64 tokens
    static constexpr int v = k + 16384;           // V_c
    static constexpr int q = v + 16384;           // 2 buffers x 2 feature halves x 2 heads x 64 rows
    static constexpr int p = q + 2 * 32768;       // tril(Si): 128 rows x 64 tokens bf16
    static constexpr int zc = p + 16384;          // z_{c-1}: float[128]
    static constexpr int bars = zc + 512;
    static constexpr int misc = bars + 24 * 8;
    static constexpr int total = misc + 16 + 1024;
};
static_assert(OutSmem::total <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ void phi_inplace(uint8_t* buf, int bytes, int lt, int nt) {
    __nv_bfloat162* w = reinterpret_cast<__nv_bfloat162*>(buf);
    for (int e = lt; e < bytes / 4; e += nt) {
        const float2 f = __bfloat1622float2(w[e]);
        w[e] = __floats2bfloat162_rn(f.x > 0.0f ? f.x + 1.0f : __expf(f.x),
                                     f.y > 0.0f ? f.y + 1.0f : __expf(f.y));
    }
}

__global__ void __launch_bounds__(kOutThreads, 1)
    k_la_out_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                const __grid_constant__ CUtensorMap tmap_v, const LaParams P) {
    extern __shared__ uint8_t la_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(la_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* shi = base + OutSmem::shi;
    uint8_t* slo = base + OutSmem::slo;
    uint8_t* kt = base + OutSmem::k;
    uint8_t* vt = base + OutSmem::v;
    uint8_t* qb = base + OutSmem::q;
    uint8_t* pt = base + OutSmem::p;
    float* zc = reinterpret_cast<float*>(base + OutSmem::zc);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + OutSmem::bars);
    uint64_t* kv_full = bars;        // K_c and V_c landed
    uint64_t* q_full = bars + 1;     // [2]
    uint64_t* q_empty = bars + 3;    // [2]
    uint64_t* s_ready = bars + 5;    // S halves written, phi applied to K_c (4 warps)
    uint64_t* q_ready = bars + 6;    // [2] phi applied to the query tile (4 warps)
    uint64_t* si_full = bars + 8;    // [2]
    uint64_t* p_full = bars + 10;    // 4 warps
    uint64_t* o_full = bars + 11;    // [2]
    uint64_t* o_empty = bars + 13;   // [2] (4 warps)
    uint64_t* mma_all = bars + 15;
    uint32_t* misc = reinterpret_cast<uint32_t*>(base + OutSmem::misc);

    const int c = blockIdx.x % P.nch, g = (blockIdx.x / P.nch) % P.H_kv, b = blockIdx.x / (P.nch * P.H_kv);
    const int t0 = c * kC;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool norm = P.phi == LISA_PHI_ELU1_NORM;
    const int n_mt = (P.group + 1) / 2;  // 128-row tiles (two heads each)

    if (tid == 0) {
        ptx::mbar_init(kv_full, 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&q_full[i], 1);
            ptx::mbar_init(&q_empty[i], 1);
            ptx::mbar_init(&q_ready[i], 4);
            ptx::mbar_init(&si_full[i], 1);
            ptx::mbar_init(&o_full[i], 1);
            ptx::mbar_init(&o_empty[i], 4);
        }
        ptx::mbar_init(s_ready, 4);
        ptx::mbar_init(p_full, 4);
        ptx::mbar_init(mma_all, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(misc, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc[0];

    auto heads_of = [&](int m) { return min(2, P.group - 2 * m); };
    if (warp == 0) {
        if (lane == 0) {
            // ---- producer
            ptx::mbar_arrive_expect_tx(kv_full, 32768);
            ptx::tma_load_3d(kt, &tmap_k, g * kD, t0, b, kv_full);
            ptx::tma_load_3d(kt + 8192, &tmap_k, g * kD + 64, t0, b, kv_full);
            ptx::tma_load_3d(vt, &tmap_v, g * kD, t0, b, kv_full);
            ptx::tma_load_3d(vt + 8192, &tmap_v, g * kD + 64, t0, b, kv_full);
            bool ok = true;
            for (int m = 0; m < n_mt && ok; ++m) {
                const int qi = m & 1;
                if (m >= 2) ok = ptx::mbar_wait_bounded(&q_empty[qi], ((m >> 1) - 1) & 1, kTries);
                if (!ok) break;
                const int nh = heads_of(m);
                uint8_t* dst = qb + qi * 32768;
                ptx::mbar_arrive_expect_tx(&q_full[qi], (uint32_t)nh * 16384);
                for (int hh = 0; hh < nh; ++hh) {
                    const int x = (g * P.group + 2 * m + hh) * kD;
                    ptx::tma_load_3d(dst + hh * 8192, &tmap_q, x, t0, b, &q_full[qi]);
                    ptx::tma_load_3d(dst + 16384 + hh * 8192, &tmap_q, x + 64, t0, b, &q_full[qi]);
                }
            }
            if (!ok) record_error(P.status, kDevTimeout);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer
            const uint32_t id_qs = ptx::idesc_bf16_f32_bmn(128, kD);
            const uint32_t id_qk = ptx::idesc_bf16_f32(128, kC);
            const uint32_t id_pv = ptx::idesc_bf16_f32_bmn(128, kD);
            const uint64_t shd = ptx::sdesc_mnmajor_sw128(shi, 16384, 1024);
            const uint64_t sld = ptx::sdesc_mnmajor_sw128(slo, 16384, 1024);
            const uint64_t kd0 = ptx::sdesc_kmajor_sw128(kt), kd1 = ptx::sdesc_kmajor_sw128(kt + 8192);
            const uint64_t vd = ptx::sdesc_mnmajor_sw128(vt, 8192, 1024);
            const uint64_t pd = ptx::sdesc_kmajor_sw128(pt);
            bool ok = ptx::mbar_wait_bounded(s_ready, 0, kTries);
            for (int m = 0; m < n_mt && ok; ++m) {
                const int qi = m & 1, ob = m & 1;
                ok = ptx::mbar_wait_bounded(norm ? &q_ready[qi] : &q_full[qi], (m >> 1) & 1, kTries);
                if (ok && m >= 2) ok = ptx::mbar_wait_bounded(&o_empty[ob], ((m >> 1) - 1) & 1, kTries);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint64_t qd0 = ptx::sdesc_kmajor_sw128(qb + qi * 32768);
                const uint64_t qd1 = ptx::sdesc_kmajor_sw128(qb + qi * 32768 + 16384);
                const uint32_t t_o = tmem + (uint32_t)(ob * 128), t_si = tmem + 256 + (uint32_t)(ob * 64);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t a = (kk < 4 ? qd0 : qd1) + 2 * (kk & 3);
                    ptx::umma_f16(t_o, a, shd + (uint64_t)(128 * kk), id_qs, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t a = (kk < 4 ? qd0 : qd1) + 2 * (kk & 3);
                    ptx::umma_f16(t_o, a, sld + (uint64_t)(128 * kk), id_qs, 1u);
                }
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t a = (kk < 4 ? qd0 : qd1) + 2 * (kk & 3);
                    const uint64_t bd = (kk < 4 ? kd0 : kd1) + 2 * (kk & 3);
                    ptx::umma_f16(t_si, a, bd, id_qk, kk > 0);
                }
                ptx::umma_commit(&q_empty[qi]);
                ptx::umma_commit(&si_full[ob]);
                ok = ptx::mbar_wait_bounded(p_full, m & 1, kTries);
                if (!ok) break;
                ptx::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    ptx::umma_f16(t_o, pd + 2 * kk, vd + (uint64_t)(128 * kk), id_pv, 1u);
                ptx::umma_commit(&o_full[ob]);
            }
            if (!ok) record_error(P.status, kDevTimeout);
            ptx::umma_commit(mma_all);
            ptx::mbar_wait_bounded(mma_all, 0, kTries);
        }
    } else {
        // ---- warps 2-5: thread = tile row (TMEM lane)
        const int lb = (warp & 3) * 32, r = lb + lane, et = tid - 64;  // et: 0..127
        // S_{c-1} (fp32, row = key feature) into bf16 hi + lo, MN-major: row i of
        // value block jb at jb * 16384 + i * 128, chunk of 8 dims swizzled by i % 8
        const float* Sp = P.U + (((int64_t)b * P.H_kv + g) * P.nch + c) * kD * kD;
        // eight rows in flight per warp (warp w % 4 takes rows w - 2, w + 2, ...)
#pragma unroll 1
        for (int r0 = warp - 2; r0 < kD; r0 += 4 * 8) {
            float4 f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                f[u] = __ldcg(reinterpret_cast<const float4*>(Sp + (int64_t)(r0 + 4 * u) * kD + lane * 4));
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int rr = r0 + 4 * u;
                const int j = lane * 4, jb = j >> 6, cc = (j & 63) >> 3;
                const int off = jb * 16384 + rr * 128 + (((cc ^ (rr & 7)) << 4) | ((j & 7) << 1));
                const __nv_bfloat162 h0 = __floats2bfloat162_rn(f[u].x, f[u].y);
                const __nv_bfloat162 h1 = __floats2bfloat162_rn(f[u].z, f[u].w);
                const float2 g0 = __bfloat1622float2(h0), g1 = __bfloat1622float2(h1);
                const __nv_bfloat162 l0 = __floats2bfloat162_rn(f[u].x - g0.x, f[u].y - g0.y);
                const __nv_bfloat162 l1 = __floats2bfloat162_rn(f[u].z - g1.x, f[u].w - g1.y);
                *reinterpret_cast<uint2*>(shi + off) = make_uint2(*reinterpret_cast<const uint32_t*>(&h0),
                                                                  *reinterpret_cast<const uint32_t*>(&h1));
                *reinterpret_cast<uint2*>(slo + off) = make_uint2(*reinterpret_cast<const uint32_t*>(&l0),
                                                                  *reinterpret_cast<const uint32_t*>(&l1));
            }
        }
        if (norm) zc[et] = P.Z[(((int64_t)b * P.H_kv + g) * P.nch + c) * kD + et];
        asm volatile("bar.sync 1, 128;" ::: "memory");  // warps 2-5, unconditionally: z is in
        bool ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(kv_full, 0, kTries));
        // phi(K_c) for the intra-chunk scores (rows past T: phi(0) = 1, but
        // they are masked: a key past T is past every valid query)
        if (ok && norm) phi_inplace(kt, 16384, et, 128);
        ptx::fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(s_ready);
        // elu+1 mode: each thread applies phi to its own row of query tile m in
        // place and takes phi(q) . z_{c-1} of it at once (the producer reuses
        // the buffer as soon as the tile's MMAs have read it)
        float qz_next = 0.0f;
        auto prep_q = [&](int m) {
            const int qi = m & 1;
            const bool w = __all_sync(0xffffffffu,
                                      ptx::mbar_wait_bounded(&q_full[qi], (m >> 1) & 1, kTries));
            float acc = 0.0f;
            if (w) {
                uint8_t* qrow = qb + qi * 32768 + r * 128;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        uint4* chunk = reinterpret_cast<uint4*>(qrow + half * 16384 + ((cc ^ (r & 7)) << 4));
                        uint4 u = *chunk;
                        __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const float2 f = __bfloat1622float2(h2[x]);
                            h2[x] = __floats2bfloat162_rn(f.x > 0.0f ? f.x + 1.0f : __expf(f.x),
                                                          f.y > 0.0f ? f.y + 1.0f : __expf(f.y));
                            const float2 pf = __bfloat1622float2(h2[x]);
                            const int f0 = half * 64 + cc * 8 + 2 * x;
                            acc = fmaf(pf.x, zc[f0], fmaf(pf.y, zc[f0 + 1], acc));
                        }
                        *chunk = u;
                    }
                }
            }
            qz_next = acc;
            ptx::fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&q_ready[qi]);
            return w;
        };
        if (norm && ok && n_mt > 0) ok = prep_q(0);
        const int tl = r & 63;              // token of this row within the chunk
        const bool tok_ok = t0 + tl < P.T;
        for (int m = 0; m < n_mt && ok; ++m) {
            const int ob = m & 1;
            const int hh = r >> 6;          // which head of the pair
            const bool row_ok = tok_ok && 2 * m + hh < P.group;
            if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&si_full[ob], (m >> 1) & 1, kTries))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            uint32_t sr[64];
            ptx::tmem_ld32(tmem + ((uint32_t)lb << 16) + 256 + (uint32_t)(ob * 64), *reinterpret_cast<uint32_t(*)[32]>(sr));
            ptx::tmem_ld32(tmem + ((uint32_t)lb << 16) + 256 + (uint32_t)(ob * 64 + 32),
                           *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
            ptx::tmem_ld_wait();
            // tril: keys j <= this row's token (inclusive), row sum for the normaliser
            float rsum = 0.0f;
            uint32_t pk[32];
#pragma unroll
            for (int j = 0; j < kC; j += 2) {
                const float a0 = j <= tl ? __uint_as_float(sr[j]) : 0.0f;
                const float a1 = j + 1 <= tl ? __uint_as_float(sr[j + 1]) : 0.0f;
                rsum += a0 + a1;
                pk[j >> 1] = ptx::pack_bf16(a0, a1);
            }
            // the P tile is free once the previous tile's P.V has completed
            if (m > 0 && !__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&o_full[(m - 1) & 1], ((m - 1) >> 1) & 1, kTries))) {
                ok = false;
                break;
            }
            uint8_t* prow = pt + r * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
                *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) =
                    make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
            ptx::fence_proxy_async_shared();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(p_full);
            const float qz = qz_next;  // phi(q) . z_{c-1} of this row (elu+1)
            if (norm && m + 1 < n_mt && !prep_q(m + 1)) {
                ok = false;
                break;
            }
            if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&o_full[ob], (m >> 1) & 1, kTries))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            const float inv = norm ? 1.0f / (qz + rsum) : 1.0f;
            bf16* orow = P.o + (((int64_t)b * P.T + t0 + tl) * P.H_q + g * P.group + 2 * m + hh) * kD;
#pragma unroll 1
            for (int c0 = 0; c0 < kD; c0 += 32) {
                uint32_t ov[32];
                ptx::tmem_ld32(tmem + ((uint32_t)lb << 16) + (uint32_t)(ob * 128 + c0), ov);
                ptx::tmem_ld_wait();
                if (row_ok) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(ptx::pack_bf16(__uint_as_float(ov[8 * e]) * inv, __uint_as_float(ov[8 * e + 1]) * inv),
                                            ptx::pack_bf16(__uint_as_float(ov[8 * e + 2]) * inv, __uint_as_float(ov[8 * e + 3]) * inv),
                                            ptx::pack_bf16(__uint_as_float(ov[8 * e + 4]) * inv, __uint_as_float(ov[8 * e + 5]) * inv),
                                            ptx::pack_bf16(__uint_as_float(ov[8 * e + 6]) * inv, __uint_as_float(ov[8 * e + 7]) * inv));
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&o_empty[ob]);
        }
        if (!ok && lane == 0) record_error(P.status, kDevTimeout);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, 512);
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
    return aligned16(q) && aligned16(k) && aligned16(v) && tma_encode_fn() != nullptr;
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
    P.status = (unsigned*)ws;
    CUtensorMap tq, tk, tv;
    memset(&tq, 0, sizeof(tq));
    memset(&tk, 0, sizeof(tk));
    memset(&tv, 0, sizeof(tv));
    const uint64_t qrow = (uint64_t)s.H_q * kD, kvrow = (uint64_t)s.H_kv * kD;
    if (!make_tmap_bf16_3d(&tq, q, qrow, s.T, s.B, qrow, (uint64_t)s.T * qrow, 64, kC) ||
        !make_tmap_bf16_3d(&tk, k, kvrow, s.T, s.B, kvrow, (uint64_t)s.T * kvrow, 64, kC) ||
        !make_tmap_bf16_3d(&tv, v, kvrow, s.T, s.B, kvrow, (uint64_t)s.T * kvrow, 64, kC))
        return cudaErrorInvalidValue;
    static bool attrs[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_la_out_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             OutSmem::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    const int ctas = s.B * s.H_kv * P.nch;
    k_la_sums_tc<<<ctas, kSumThreads, 0, st>>>(tk, tv, P);
    const int64_t nstate = (int64_t)s.B * s.H_kv * kD * kD;
    k_la_prefix<<<(unsigned)((nstate + 255) / 256), 256, 0, st>>>(P);
    k_la_out_tc<<<ctas, kOutThreads, OutSmem::total, st>>>(tq, tk, tv, P);
    return cudaGetLastError();
}

}  // namespace lisa
