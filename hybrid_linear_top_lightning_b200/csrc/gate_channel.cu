// Per-channel gate of the two branches (LISA, arXiv 2607.19358v1, Sec. 3.3
// Eq. 5: g = sigmoid(W_g h), one gate per output channel, mixing the branches
// as in Eq. 1: o = g * o_lin + (1 - g) * o_sparse).  The gate logits are a
// dense contraction, C[m][n] = sum_k h[m][k] W_g[n][k] over the M = B*T tokens,
// N = H_q*d channels and K = D_h hidden features.
//
// k_gate_channel_tc (more than 64 tokens): persistent, one CTA per SM walking
//   128 x 256 tiles of C (the channel tile varies fastest, so the CTAs at work
//   share their h rows and all of W_g stays in L2); tcgen05.mma kind::f16
//   (M=128, N=256, K=16) accumulating in TMEM over K in steps of 64, h and W_g
//   tiles brought by TMA (128-byte swizzle) through a 4-stage ring.  Warp 0
//   issues TMA, warp 1 owns TMEM and issues the MMAs, warps 2-5 (one TMEM lane
//   = one token each) apply the sigmoid and mix the branches while the next
//   tile accumulates in the other TMEM buffer.
// k_gate_channel_rows (up to 64 tokens, decode): W_g streamed once from HBM
//   onto the warp MMA (m16n8k16) straight from registers; HBM-bound on W_g.
#include <cuda.h>

#include "lisa_fast.cuh"
#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kGM = 128;        // tokens per tile (MMA M)
constexpr int kGN = 256;        // channels per tile (MMA N)
constexpr int kGK = 64;         // hidden features per stage (128 bytes of bf16)
constexpr int kGStages = 4;
constexpr int kGThreads = 192;
constexpr uint32_t kGTries = 1u << 22;

struct GcParams {
    int M, N, K;
    int tiles_n, tiles;     // channel tiles per token tile; all tiles
    const bf16* o_lin;
    const bf16* o_sp;
    bf16* o;
    unsigned* status;
};

struct GcSmem {
    static constexpr int a = 0;                                    // kGStages x 16 KB
    static constexpr int b = a + kGStages * kGM * 128;             // kGStages x 32 KB
    static constexpr int bars = b + kGStages * kGN * 128;          // full, empty, tfull, tempty
    static constexpr int tmem = bars + 16 * 8;
    static constexpr int total = tmem + 16 + 1024;                 // + base alignment slack
};

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __bfloat1622float2(h[e]);
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}

// Persistent: CTA c takes tiles c, c + gridDim.x, ...; tile i -> (token tile
// i / tiles_n, channel tile i % tiles_n).  The accumulator is double-buffered
// in TMEM (2 x 256 columns), so the epilogue of one tile runs under the
// mainloop of the next.
__global__ void __launch_bounds__(kGThreads, 1)
    k_gate_channel_tc(const __grid_constant__ CUtensorMap tmap_h,
                      const __grid_constant__ CUtensorMap tmap_w, const GcParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* as = base + GcSmem::a;
    uint8_t* bs = base + GcSmem::b;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + GcSmem::bars);
    uint64_t* full = bars;
    uint64_t* empty = bars + kGStages;
    uint64_t* tfull = bars + 2 * kGStages;       // [2] accumulator ready
    uint64_t* tempty = bars + 2 * kGStages + 2;  // [2] accumulator drained
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + GcSmem::tmem);
    __shared__ int s_fail;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nk = P.K / kGK;
    const uint32_t idesc = ptx::idesc_bf16_f32(kGM, kGN);

    if (tid == 0) {
        for (int s = 0; s < kGStages; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int j = 0; j < 2; ++j) {
            ptx::mbar_init(&tfull[j], 1);
            ptx::mbar_init(&tempty[j], 4);  // one arrival per epilogue warp
        }
        ptx::fence_mbar_init();
        s_fail = 0;
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, 2u * kGN);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- producer: one continuous ring over every k step of every tile
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x) {
                const int m0 = (tile / P.tiles_n) * kGM, n0 = (tile % P.tiles_n) * kGN;
                for (int ks = 0; ks < nk; ++ks, ++it) {
                    const uint32_t s = it % kGStages, use = it / kGStages;
                    if (use > 0 && !ptx::mbar_wait_bounded(&empty[s], (use - 1) & 1, kGTries)) {
                        ok = false;
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&full[s], (kGM + kGN) * 128);
                    ptx::tma_load_2d(as + s * kGM * 128, &tmap_h, ks * kGK, m0, &full[s]);
                    ptx::tma_load_2d(bs + s * kGN * 128, &tmap_w, ks * kGK, n0, &full[s]);
                }
            }
            if (!ok) {
                s_fail = 1;
                record_error(P.status, kDevTimeout);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer
            uint32_t it = 0, local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++local) {
                const uint32_t buf = local & 1, use = local >> 1;
                if (use > 0 && !ptx::mbar_wait_bounded(&tempty[buf], (use - 1) & 1, kGTries)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t acc = tmem + buf * kGN;
                for (int ks = 0; ks < nk; ++ks, ++it) {
                    const uint32_t s = it % kGStages;
                    if (!ptx::mbar_wait_bounded(&full[s], (it / kGStages) & 1, kGTries)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint64_t adesc = ptx::sdesc_kmajor_sw128(as + s * kGM * 128);
                    const uint64_t bdesc = ptx::sdesc_kmajor_sw128(bs + s * kGN * 128);
#pragma unroll
                    for (int kk = 0; kk < kGK / 16; ++kk)
                        ptx::umma_f16(acc, adesc + 2 * kk, bdesc + 2 * kk, idesc, ks > 0 || kk > 0);
                    ptx::umma_commit(&empty[s]);
                }
                if (ok) ptx::umma_commit(&tfull[buf]);
            }
            if (!ok) {
                s_fail = 1;
                record_error(P.status, kDevTimeout);
            }
        }
    } else {
        // ---- epilogue: thread = token (TMEM lane), 32 channels at a time
        const int lg = (warp & 3) * 32;
        uint32_t local = 0;
        for (int tile = blockIdx.x; tile < P.tiles; tile += gridDim.x, ++local) {
            const uint32_t buf = local & 1, use = local >> 1;
            if (!ptx::mbar_wait_bounded(&tfull[buf], use & 1, kGTries)) {
                s_fail = 1;
                if (lane == 0) record_error(P.status, kDevTimeout);
                break;
            }
            ptx::tc_fence_after();
            const int m = (tile / P.tiles_n) * kGM + lg + lane, n0 = (tile % P.tiles_n) * kGN;
            const uint32_t acc = tmem + buf * kGN + ((uint32_t)lg << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < kGN; c0 += 32) {
                uint32_t r[32];
                ptx::tmem_ld32(acc + (uint32_t)c0, r);
                ptx::tmem_ld_wait();
                if (c0 + 32 == kGN) {
                    // the whole accumulator is in registers: hand the buffer back
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
                }
                if (m < P.M) {
                    const int64_t off = (int64_t)m * P.N + n0 + c0;
                    const uint4* la = reinterpret_cast<const uint4*>(P.o_lin + off);
                    const uint4* sa = reinterpret_cast<const uint4*>(P.o_sp + off);
                    uint4* oa = reinterpret_cast<uint4*>(P.o + off);
                    uint4 lv[4], sv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        lv[u] = __ldcs(la + u);
                        sv[u] = __ldcs(sa + u);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        float a8[8], c8[8];
                        unpack8(lv[u], a8);
                        unpack8(sv[u], c8);
                        uint4 res;
                        __nv_bfloat162* rh = reinterpret_cast<__nv_bfloat162*>(&res);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float x0 = __uint_as_float(r[8 * u + 2 * e]);
                            const float x1 = __uint_as_float(r[8 * u + 2 * e + 1]);
                            const float g0 = 1.0f / (1.0f + __expf(-x0));
                            const float g1 = 1.0f / (1.0f + __expf(-x1));
                            rh[e] = __floats2bfloat162_rn(fmaf(g0, a8[2 * e] - c8[2 * e], c8[2 * e]),
                                                          fmaf(g1, a8[2 * e + 1] - c8[2 * e + 1],
                                                               c8[2 * e + 1]));
                        }
                        __stcs(oa + u, res);
                    }
                }
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (s_fail && tid == 0) {
        // let copies still in flight land before the shared memory is released
        for (int s = 0; s < kGStages; ++s)
            for (uint32_t par = 0; par < 2; ++par) ptx::mbar_wait_bounded(&full[s], par, 1u << 16);
    }
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 2u * kGN);
    }
}

// Up to 64 tokens (decode): W_g streamed from HBM once, on the warp MMA.
// A CTA owns 16 channels; its warps split K in 32-column chunks (warp w of WN
// takes chunks w, w+WN, ...).  Per chunk a lane reads 16 bytes of W_g row g and of row
// g+8 (g = lane/4, t = lane%4: columns 8t..8t+7 of the chunk) and 16 bytes of
// token g's h at the same columns.  The 32 columns are fed to two m16n8k16
// MMAs in a column order that A and B share (MMA j takes columns 8t+4j..8t+4j+3
// of lane (g, t) as its k = 2t, 2t+1, 2t+8, 2t+9), which leaves the sum over k
// unchanged, so neither operand needs shared memory.  NT tiles of 8 tokens.
template <int NT>
struct RowCfg {
    // warps per CTA and chunks in flight per warp: at D_h = 3584 (112 chunks)
    // one token tile reads its whole W_g share in a single round of loads
    static constexpr int warps = NT <= 2 ? 16 : 8;
    static constexpr int unroll = NT == 1 ? 7 : NT == 2 ? 4 : NT == 4 ? 4 : 2;
};

template <int NT>
__global__ void __launch_bounds__(RowCfg<NT>::warps * 32) k_gate_channel_rows(
    const bf16* __restrict__ h, const bf16* __restrict__ W, int M, int N, int K,
    const bf16* __restrict__ o_lin, const bf16* __restrict__ o_sp, bf16* __restrict__ o) {
    constexpr int kRowWarps = RowCfg<NT>::warps;
    constexpr int kRowUnroll = RowCfg<NT>::unroll;
    __shared__ float red[kRowWarps][NT][16][8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int n0 = blockIdx.x * 16;
    const uint4* w0 = reinterpret_cast<const uint4*>(W + (int64_t)(n0 + g) * K) + t;
    const uint4* w1 = reinterpret_cast<const uint4*>(W + (int64_t)(n0 + g + 8) * K) + t;
    const uint4* hr[NT];
    bool hv[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        hv[j] = 8 * j + g < M;
        hr[j] = reinterpret_cast<const uint4*>(h + (int64_t)(hv[j] ? 8 * j + g : 0) * K) + t;
    }
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.0f;
    const int nchunk = K / 32;
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int c0 = warp; c0 < nchunk; c0 += kRowWarps * kRowUnroll) {
        uint4 a0[kRowUnroll], a1[kRowUnroll], bv[kRowUnroll][NT];
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            const int c = c0 + u * kRowWarps;
            const bool in = c < nchunk;
            a0[u] = in ? __ldcs(w0 + 4 * c) : zero;
            a1[u] = in ? __ldcs(w1 + 4 * c) : zero;
#pragma unroll
            for (int j = 0; j < NT; ++j) bv[u][j] = (in && hv[j]) ? __ldg(hr[j] + 4 * c) : zero;
        }
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            const uint32_t fa0[4] = {a0[u].x, a1[u].x, a0[u].y, a1[u].y};
            const uint32_t fa1[4] = {a0[u].z, a1[u].z, a0[u].w, a1[u].w};
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                ptx::mma_bf16(acc[j], fa0, bv[u][j].x, bv[u][j].y);
                ptx::mma_bf16(acc[j], fa1, bv[u][j].z, bv[u][j].w);
            }
        }
    }
    // D fragment: acc[j][0..1] = channel g, tokens 8j+2t, +1; acc[j][2..3] = channel g+8
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        red[warp][j][g][2 * t] = acc[j][0];
        red[warp][j][g][2 * t + 1] = acc[j][1];
        red[warp][j][g + 8][2 * t] = acc[j][2];
        red[warp][j][g + 8][2 * t + 1] = acc[j][3];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < NT * 128; i += kRowWarps * 32) {
        const int ch = i & 15, tok = i >> 4;  // tok = 8 * j + column
        if (tok >= M) continue;
        float x = 0.0f;
#pragma unroll
        for (int w = 0; w < kRowWarps; ++w) x += red[w][tok >> 3][ch][tok & 7];
        const float gt = 1.0f / (1.0f + __expf(-x));
        const int64_t off = (int64_t)tok * N + n0 + ch;
        const float a = __bfloat162float(o_lin[off]), c = __bfloat162float(o_sp[off]);
        o[off] = __float2bfloat16_rn(fmaf(gt, a - c, c));
    }
}

template <int NT>
void launch_rows(int M, int N, int K, const void* h, const void* W, const void* o_lin,
                 const void* o_sp, void* o, cudaStream_t st) {
    k_gate_channel_rows<NT><<<N / 16, RowCfg<NT>::warps * 32, 0, st>>>(
        (const bf16*)h, (const bf16*)W, M, N, K, (const bf16*)o_lin, (const bf16*)o_sp, (bf16*)o);
}

constexpr int kRowMax = 64;  // tokens up to which W_g is streamed on the warp MMA

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Any size and either activation type: one warp per (token, channel).
template <typename T>
__global__ void __launch_bounds__(256) k_gate_channel_generic(const T* __restrict__ h,
                                                              const T* __restrict__ W, int M, int N,
                                                              int K, const T* __restrict__ o_lin,
                                                              const T* __restrict__ o_sp,
                                                              T* __restrict__ o) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (wid >= (int64_t)M * N) return;
    const int m = (int)(wid / N), n = (int)(wid % N);
    const T* hr = h + (int64_t)m * K;
    const T* wr = W + (int64_t)n * K;
    float x = 0.0f;
    for (int k = lane; k < K; k += 32) x = fmaf(to_f32(wr[k]), to_f32(hr[k]), x);
#pragma unroll
    for (int o_ = 16; o_ > 0; o_ >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o_);
    if (lane == 0) {
        const float g = 1.0f / (1.0f + __expf(-x));
        const float a = to_f32(o_lin[wid]), c = to_f32(o_sp[wid]);
        o[wid] = from_f32<T>(fmaf(g, a - c, c));
    }
}

}  // namespace

cudaError_t generic_gate_channel(const Shape& s, int D_h, const void* h, const void* W,
                                 const void* o_lin, const void* o_sp, void* o, cudaStream_t st) {
    const int M = s.B * s.T, N = s.H_q * s.d;
    const int64_t warps = (int64_t)M * N;
    if (warps == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((warps + 7) / 8);
    if (s.dtype == LISA_BF16)
        k_gate_channel_generic<bf16><<<blocks, 256, 0, st>>>(
            (const bf16*)h, (const bf16*)W, M, N, D_h, (const bf16*)o_lin, (const bf16*)o_sp, (bf16*)o);
    else
        k_gate_channel_generic<float><<<blocks, 256, 0, st>>>(
            (const float*)h, (const float*)W, M, N, D_h, (const float*)o_lin, (const float*)o_sp,
            (float*)o);
    return cudaGetLastError();
}

bool fast_gate_channel_supported(const Shape& s, int D_h, const void* h, const void* W,
                                 const void* o_lin, const void* o_sp, const void* o) {
    if (s.dtype != LISA_BF16) return false;
    const int N = s.H_q * s.d;
    if (D_h % kGK != 0 || N % kGN != 0) return false;
    const int M = s.B * s.T;
    if (M > kRowMax && !tma_encode_fn()) return false;
    return aligned16(h) && aligned16(W) && aligned16(o_lin) && aligned16(o_sp) && aligned16(o);
}

cudaError_t fast_gate_channel(const Shape& s, int D_h, const void* h, const void* W,
                              const void* o_lin, const void* o_sp, void* o, void* ws,
                              cudaStream_t st) {
    const int M = s.B * s.T, N = s.H_q * s.d;
    if (M == 0) return cudaSuccess;
    if (M <= kRowMax) {
        switch ((M + 7) / 8) {
            case 1: launch_rows<1>(M, N, D_h, h, W, o_lin, o_sp, o, st); break;
            case 2: launch_rows<2>(M, N, D_h, h, W, o_lin, o_sp, o, st); break;
            case 3:
            case 4: launch_rows<4>(M, N, D_h, h, W, o_lin, o_sp, o, st); break;
            default: launch_rows<8>(M, N, D_h, h, W, o_lin, o_sp, o, st); break;
        }
        return cudaGetLastError();
    }
    static bool attrs[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(
            k_gate_channel_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, GcSmem::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    CUtensorMap th, tw;
    if (!make_tmap_bf16_box(&th, h, (uint64_t)D_h, (uint64_t)M, kGK, kGM) ||
        !make_tmap_bf16_box(&tw, W, (uint64_t)D_h, (uint64_t)N, kGK, kGN))
        return cudaErrorInvalidValue;
    GcParams P;
    P.M = M; P.N = N; P.K = D_h;
    P.tiles_n = N / kGN;
    P.tiles = P.tiles_n * ((M + kGM - 1) / kGM);
    P.o_lin = (const bf16*)o_lin; P.o_sp = (const bf16*)o_sp; P.o = (bf16*)o;
    P.status = (unsigned*)ws;
    int sms = 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        sms = 148;
    const int grid = P.tiles < sms ? P.tiles : sms;
    k_gate_channel_tc<<<grid, kGThreads, GcSmem::total, st>>>(th, tw, P);
    return cudaGetLastError();
}

}  // namespace lisa
