// Lightning Indexer over many query rows (prefill) on B200: tcgen05 score GEMM
// into a workspace, then an exact top-M per row (LISA, arXiv 2607.19358v1,
// Sec. 3.2: per-head ReLU dot-product scores, weighted and summed over the
// indexer heads, the M highest kept).
//
// k_index_scores_tc: one CTA per (sequence, tile of 32 query rows), looping
//   over the key tiles of 128 keys that are causally visible to the tile.
//   D[key, (query, head)] = K_I[key] . Q_I[query, head] is one tcgen05.mma
//   chain of shape M=128 (keys) x N=32*H_I (query x head) x K=d_I=64, operands
//   brought into shared memory by TMA (128-byte swizzle), accumulator in TMEM.
//   Roles: warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs, warps 2-9
//   read the accumulator (one TMEM lane = one key per thread; the two warps of
//   a lane quarter take alternate 32-column chunks) and reduce over the heads
//   inside the thread: score = sum_h w[q,h] * ReLU(D[key, (q,h)]).
//   Stores are coalesced along keys.  Two CTAs share an SM, so one's epilogue
//   overlaps the other's MMAs.
// k_topm_rows_fast: one CTA per query row; the row comes into shared memory by
//   TMA bulk copies, then the exact radix select of select_row.cuh writes the
//   selected positions in ascending order.
//
// All waits are bounded; a wait that gives up records LISA_ERR_TIMEOUT and the
// kernel releases its TMEM and returns.
#include <cuda.h>

#include <algorithm>

#include "lisa_fast.cuh"
#include "lisa_internal.cuh"
#include "select_row.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kDI = 64;
constexpr int kQT = 32;        // query rows per tile
constexpr int kKT = 128;       // keys per tile (MMA M)
constexpr int kKStages = 4;    // key tiles in flight
constexpr int kScoreThreads = 192;      // the paper-form kernel: warp 0 TMA, 1 MMA, 2-5 epilogue
constexpr int kScoreMainThreads = 320;  // k_index_scores_tc: warp 0 TMA, 1 MMA, 2-9 epilogue
constexpr uint32_t kTries = 1u << 22;

struct ScoreParams {
    int B, T, n_past, L, Lpad, N_max, H_I, nqt;
    int64_t w_tok_stride;
    const float* w;
    uint32_t* keys;  // [B*T][Lpad]: order-preserving keys of the causal scores
    unsigned* status;
};

struct ScoreSmem {
    static constexpr int q = 0;                                   // N x 128 B (<= 32 KB)
    static constexpr int k = q + 256 * 128;                       // kKStages x 16 KB
    static constexpr int w = k + kKStages * kKT * 128;             // float[32][8]
    static constexpr int bars = w + kQT * 8 * 4;                   // q_full, k_full[4], k_empty[4], t_full, t_empty
    static constexpr int tmem = bars + 16 * 8;                     // u32
    static constexpr int total = tmem + 16 + 1024;                 // + base alignment slack
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    return ptx::mbar_wait_bounded(bar, parity, kTries);
}

template <int HI>
__global__ void __launch_bounds__(kScoreMainThreads, 2)
    k_index_scores_tc(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_k, const ScoreParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* qs = base + ScoreSmem::q;
    uint8_t* ks = base + ScoreSmem::k;
    float* ws = reinterpret_cast<float*>(base + ScoreSmem::w);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + ScoreSmem::bars);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = bars + 1 + kKStages;
    uint64_t* t_full = bars + 1 + 2 * kKStages;
    uint64_t* t_empty = bars + 2 + 2 * kKStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + ScoreSmem::tmem);
    __shared__ int s_fail;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lin = gridDim.x - 1 - blockIdx.x;  // the longest tiles (last queries) first
    const int b = lin / P.nqt, qt = lin % P.nqt;
    const int q0 = qt * kQT;
    const int qrows = min(kQT, P.T - q0);
    constexpr int N = kQT * HI;  // MMA N: 32..256
    const int kt_causal = (P.n_past + q0 + qrows - 1) / kKT + 1;
    const int n_kt = min((P.L + kKT - 1) / kKT, kt_causal);
    const uint32_t idesc = ptx::idesc_bf16_f32(kKT, N);

    if (tid == 0) {
        ptx::mbar_init(q_full, 1);
        for (int s = 0; s < kKStages; ++s) {
            ptx::mbar_init(&k_full[s], 1);
            ptx::mbar_init(&k_empty[s], 1);
        }
        ptx::mbar_init(t_full, 1);
        ptx::mbar_init(t_empty, 256);
        ptx::fence_mbar_init();
        s_fail = 0;
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, (uint32_t)N);
        ptx::tmem_relinquish();
    }
    if (warp >= 2) {
        // head weights of this tile's queries
        const int e = tid - 64;  // 0..255
        for (int i = e; i < kQT * P.H_I; i += 256) {
            const int ql = i / P.H_I, h = i % P.H_I;
            float v = 0.0f;
            if (ql < qrows) {
                const int64_t bs = P.w_tok_stride ? (int64_t)P.T * P.w_tok_stride : P.H_I;
                v = P.w[b * bs + (int64_t)(q0 + ql) * P.w_tok_stride + h];
            }
            ws[ql * 8 + h] = v;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- producer
            ptx::mbar_arrive_expect_tx(q_full, (uint32_t)N * 128);
            ptx::tma_load_2d(qs, &tmap_q, 0, (b * P.T + q0) * P.H_I, q_full);
            for (int kt = 0; kt < n_kt; ++kt) {
                const int s = kt % kKStages, use = kt / kKStages;
                if (use > 0 && !wait_bar(&k_empty[s], (use - 1) & 1)) {
                    s_fail = 1;
                    record_error(P.status, kDevTimeout);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&k_full[s], kKT * 128);
                ptx::tma_load_2d(ks + s * kKT * 128, &tmap_k, 0, b * P.N_max + kt * kKT, &k_full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer
            bool ok = wait_bar(q_full, 0);
            const uint64_t bdesc = ptx::sdesc_kmajor_sw128(qs);
            for (int kt = 0; ok && kt < n_kt; ++kt) {
                const int s = kt % kKStages;
                ok = wait_bar(&k_full[s], (kt / kKStages) & 1);
                if (ok && kt > 0) ok = wait_bar(t_empty, (kt - 1) & 1);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint64_t adesc = ptx::sdesc_kmajor_sw128(ks + s * kKT * 128);
#pragma unroll
                for (int kk = 0; kk < kDI / 16; ++kk)
                    ptx::umma_f16(tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0);
                ptx::umma_commit(&k_empty[s]);
                ptx::umma_commit(t_full);
            }
            if (!ok) {
                s_fail = 1;
                record_error(P.status, kDevTimeout);
            }
        }
    } else {
        // ---- epilogue: thread = key (TMEM lane), columns = (query, head); the
        // two warps of a lane quarter take alternate 32-column chunks
        const int lg = (warp & 3) * 32;
        const int half = (warp - 2) >> 2;
        const int key_l = lg + lane;
        constexpr int qpc = 32 / HI;  // queries per 32-column chunk
        for (int kt = 0; kt < n_kt; ++kt) {
            if (!wait_bar(t_full, kt & 1)) {
                s_fail = 1;
                if (lane == 0) record_error(P.status, kDevTimeout);
                break;
            }
            ptx::tc_fence_after();
            const int key = kt * kKT + key_l;
#pragma unroll 1
            for (int c0 = half * 32; c0 < N; c0 += 64) {
                uint32_t r[32];
                ptx::tmem_ld32(tmem + ((uint32_t)lg << 16) + (uint32_t)c0, r);
                ptx::tmem_ld_wait();
                const int qb = c0 / HI;
#pragma unroll
                for (int u = 0; u < qpc; ++u) {
                    const int ql = qb + u;
                    float sc = 0.0f;
#pragma unroll
                    for (int h = 0; h < HI; ++h)
                        sc = fmaf(ws[ql * 8 + h], fmaxf(__uint_as_float(r[u * HI + h]), 0.0f), sc);
                    const int t = q0 + ql;
                    if (ql < qrows && key < P.L && key <= P.n_past + t)
                        P.keys[((int64_t)b * P.T + t) * P.Lpad + key] = order_key(sc);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(t_empty);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (s_fail && tid == 0) {
        // let copies still in flight land before the shared memory is released
        ptx::mbar_wait_bounded(q_full, 0, 1u << 16);
        for (int s = 0; s < kKStages; ++s)
            for (uint32_t par = 0; par < 2; ++par) ptx::mbar_wait_bounded(&k_full[s], par, 1u << 16);
    }
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, (uint32_t)N);
    }
}

// ---------------------------------------------------------------- the paper's form
// A key per indexer head (H_Ik = H_I = 8; LISA Sec. 3.2: head j scores its own
// keys).  One CTA per (sequence, 32 query rows) as above, but the product is a
// batch of eight: for every key tile and head j, D[key, 32 j + q] =
// K_I[key, j] . Q_I[q, j] (tcgen05, M = 128 keys x N = 32 queries x K = 64),
// the operands brought by TMA from 3-D maps [rows][head][64] whose boxes take
// one head of 128 keys (or 32 queries); the key ring holds one (key tile, head)
// item per stage.  The epilogue sums w[q, j] * ReLU(D) over the heads per query.
struct HeadsSmem {
    static constexpr int q = 0;                                   // 8 heads x 32 rows x 128 B
    static constexpr int k = q + 8 * kQT * 128;                   // kKStages x 128 rows x 128 B
    static constexpr int w = k + kKStages * kKT * 128;            // float[32][8]
    static constexpr int bars = w + kQT * 8 * 4;
    static constexpr int tmem = bars + 16 * 8;
    static constexpr int total = tmem + 16 + 1024;
};

__global__ void __launch_bounds__(kScoreThreads, 2)
    k_index_scores_heads_tc(const __grid_constant__ CUtensorMap tmap_q,
                            const __grid_constant__ CUtensorMap tmap_k, const ScoreParams P) {
    constexpr int HI = 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* qs = base + HeadsSmem::q;
    uint8_t* ks = base + HeadsSmem::k;
    float* ws = reinterpret_cast<float*>(base + HeadsSmem::w);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + HeadsSmem::bars);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = bars + 1 + kKStages;
    uint64_t* t_full = bars + 1 + 2 * kKStages;
    uint64_t* t_empty = bars + 2 + 2 * kKStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + HeadsSmem::tmem);
    __shared__ int s_fail;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lin = gridDim.x - 1 - blockIdx.x;  // the longest tiles (last queries) first
    const int b = lin / P.nqt, qt = lin % P.nqt;
    const int q0 = qt * kQT;
    const int qrows = min(kQT, P.T - q0);
    constexpr int N = kQT * HI;  // 256 columns: head j owns 32 j .. 32 j + 31
    const int kt_causal = (P.n_past + q0 + qrows - 1) / kKT + 1;
    const int n_kt = min((P.L + kKT - 1) / kKT, kt_causal);
    const uint32_t idesc = ptx::idesc_bf16_f32(kKT, kQT);

    if (tid == 0) {
        ptx::mbar_init(q_full, 1);
        for (int s = 0; s < kKStages; ++s) {
            ptx::mbar_init(&k_full[s], 1);
            ptx::mbar_init(&k_empty[s], 1);
        }
        ptx::mbar_init(t_full, 1);
        ptx::mbar_init(t_empty, 128);
        ptx::fence_mbar_init();
        s_fail = 0;
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_slot, (uint32_t)N);
        ptx::tmem_relinquish();
    }
    if (warp >= 2) {
        const int e = tid - 64;  // 0..127: head weights of this tile's queries
        for (int i = e; i < kQT * HI; i += 128) {
            const int ql = i / HI, h = i % HI;
            float v = 0.0f;
            if (ql < qrows) {
                const int64_t bs = P.w_tok_stride ? (int64_t)P.T * P.w_tok_stride : HI;
                v = P.w[b * bs + (int64_t)(q0 + ql) * P.w_tok_stride + h];
            }
            ws[ql * 8 + h] = v;
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- producer: the query tile (8 heads), then one (key tile, head) per stage
            ptx::mbar_arrive_expect_tx(q_full, (uint32_t)HI * kQT * 128);
            for (int h = 0; h < HI; ++h)
                ptx::tma_load_3d(qs + h * kQT * 128, &tmap_q, 0, h, b * P.T + q0, q_full);
            for (int it = 0; it < n_kt * HI; ++it) {
                const int s = it % kKStages, use = it / kKStages;
                const int kt = it / HI, h = it % HI;
                if (use > 0 && !wait_bar(&k_empty[s], (use - 1) & 1)) {
                    s_fail = 1;
                    record_error(P.status, kDevTimeout);
                    break;
                }
                ptx::mbar_arrive_expect_tx(&k_full[s], kKT * 128);
                ptx::tma_load_3d(ks + s * kKT * 128, &tmap_k, 0, h, b * P.N_max + kt * kKT, &k_full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer
            bool ok = wait_bar(q_full, 0);
            for (int kt = 0; ok && kt < n_kt; ++kt) {
                if (kt > 0) ok = wait_bar(t_empty, (kt - 1) & 1);
                for (int h = 0; ok && h < HI; ++h) {
                    const int it = kt * HI + h, s = it % kKStages;
                    ok = wait_bar(&k_full[s], (it / kKStages) & 1);
                    if (!ok) break;
                    ptx::tc_fence_after();
                    const uint64_t adesc = ptx::sdesc_kmajor_sw128(ks + s * kKT * 128);
                    const uint64_t bdesc = ptx::sdesc_kmajor_sw128(qs + h * kQT * 128);
#pragma unroll
                    for (int kk = 0; kk < kDI / 16; ++kk)
                        ptx::umma_f16(tmem + (uint32_t)(h * kQT), adesc + 2 * kk, bdesc + 2 * kk, idesc, kk > 0);
                    ptx::umma_commit(&k_empty[s]);
                }
                if (ok) ptx::umma_commit(t_full);
            }
            if (!ok) {
                s_fail = 1;
                record_error(P.status, kDevTimeout);
            }
        }
    } else {
        // ---- epilogue: thread = key (TMEM lane); per query, the weighted sum of
        // the heads' ReLU scores
        const int lg = (warp & 3) * 32;
        const int key_l = lg + lane;
        for (int kt = 0; kt < n_kt; ++kt) {
            if (!wait_bar(t_full, kt & 1)) {
                s_fail = 1;
                if (lane == 0) record_error(P.status, kDevTimeout);
                break;
            }
            ptx::tc_fence_after();
            const int key = kt * kKT + key_l;
            // 16 queries at a time (few registers live)
#pragma unroll 1
            for (int qh = 0; qh < kQT; qh += 16) {
                float acc[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) acc[q] = 0.0f;
#pragma unroll 1
                for (int h = 0; h < HI; ++h) {
                    uint32_t r[16];
                    ptx::tmem_ld16(tmem + ((uint32_t)lg << 16) + (uint32_t)(h * kQT + qh), r);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        acc[q] = fmaf(ws[(qh + q) * 8 + h], fmaxf(__uint_as_float(r[q]), 0.0f), acc[q]);
                }
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const int t = q0 + qh + q;
                    if (qh + q < qrows && key < P.L && key <= P.n_past + t)
                        P.keys[((int64_t)b * P.T + t) * P.Lpad + key] = order_key(acc[q]);
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(t_empty);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (s_fail && tid == 0) {
        // let copies still in flight land before the shared memory is released
        ptx::mbar_wait_bounded(q_full, 0, 1u << 16);
        for (int s = 0; s < kKStages; ++s)
            for (uint32_t par = 0; par < 2; ++par) ptx::mbar_wait_bounded(&k_full[s], par, 1u << 16);
    }
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, (uint32_t)N);
    }
}

// ---------------------------------------------------------------- per-row selection
constexpr int kRowCap = 16384;  // scores of a row held in shared memory
constexpr int kRowThreads = 256;

struct RowParams {
    int B, T, n_past, Lpad, M;
    const uint32_t* keys;
    int32_t* idx;
    int32_t* count;
    unsigned* status;
};

struct RowSmem {
    static constexpr int row = 0;                         // float[kRowCap + 32]
    static constexpr int hist = row + (kRowCap + 32) * 4; // u32[4096]
    static constexpr int cand = hist + 4096 * 4;          // uint2[kCandTotal]
    static constexpr int bc = cand + kCandTotal * 8;
    static constexpr int bar = bc + 128 * 4;
    static constexpr int total = bar + 16;
};

__global__ void __launch_bounds__(kRowThreads) k_topm_rows_fast(const RowParams P) {
    extern __shared__ __align__(128) uint8_t row_raw[];
    const int row = blockIdx.x;
    const int t = row % P.T;
    const int nc = P.n_past + t + 1;
    int32_t* out = P.idx + (int64_t)row * P.M;
    ptx::pdl_wait_prior();
    if (nc <= P.M) {
        for (int i = threadIdx.x; i < P.M; i += kRowThreads) out[i] = i < nc ? i : -1;
        if (threadIdx.x == 0) P.count[row] = nc;
        return;
    }
    uint32_t* rs = reinterpret_cast<uint32_t*>(row_raw + RowSmem::row);
    uint64_t* bar = reinterpret_cast<uint64_t*>(row_raw + RowSmem::bar);
    const uint32_t* gr = P.keys + (int64_t)row * P.Lpad;
    const bool resident = nc <= kRowCap;
    if (resident && threadIdx.x == 0) {
        ptx::mbar_init(bar, 1);
        ptx::fence_mbar_init();
        const int bytes = ((nc + 3) / 4) * 16;
        ptx::mbar_arrive_expect_tx(bar, bytes);
        for (int off = 0; off < bytes; off += 16384)
            ptx::bulk_load(row_raw + RowSmem::row + off, gr + off / 4, min(16384, bytes - off), bar);
    }
    __syncthreads();
    SelectSmem sel;
    sel.hist = reinterpret_cast<unsigned*>(row_raw + RowSmem::hist);
    sel.bc = reinterpret_cast<int*>(row_raw + RowSmem::bc);
    sel.cand = reinterpret_cast<uint2*>(row_raw + RowSmem::cand);
    row_topm<kRowThreads>(resident ? rs : gr, resident, nc, P.M, nullptr, sel, 0, P.M, out,
             resident ? bar : nullptr, P.status);
    if (threadIdx.x == 0) P.count[row] = P.M;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

size_t fast_topm_ws_bytes(const Shape& s) {
    const size_t Lpad = (size_t)((s.L + 31) / 32 * 32);
    return kStatusBytes + sizeof(float) * (size_t)s.B * s.T * Lpad + 256;
}

bool fast_topm_supported(const Shape& s, const void* q_I, const void* k_I, const float* w,
                         int64_t w_tok_stride) {
    if (s.dtype != LISA_BF16 || s.d_I != kDI) return false;
    if (!(s.H_I == 1 || s.H_I == 2 || s.H_I == 4 || s.H_I == 8)) return false;
    if (!(s.H_Ik == 1 || (s.H_Ik == 8 && s.H_I == 8))) return false;
    if (s.T < 1 || s.L < 1) return false;
    if ((int64_t)s.B * s.T * s.H_I >= (1ll << 31) || (int64_t)s.B * s.N_max >= (1ll << 31)) return false;
    if (!aligned16(q_I) || !aligned16(k_I) || !w) return false;
    (void)w_tok_stride;
    return tma_encode_fn() != nullptr;
}

cudaError_t fast_topm(const Shape& s, const void* q_I, const void* k_I, const float* w,
                      int64_t w_tok_stride, int32_t* idx, int32_t* count, void* ws,
                      cudaStream_t st) {
    ScoreParams P;
    P.B = s.B; P.T = s.T; P.n_past = s.n_past; P.L = s.L; P.Lpad = (s.L + 31) / 32 * 32;
    P.N_max = s.N_max; P.H_I = s.H_I; P.nqt = (s.T + kQT - 1) / kQT;
    P.w_tok_stride = w_tok_stride; P.w = w;
    P.keys = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(ws) + kStatusBytes);
    P.status = reinterpret_cast<unsigned*>(ws);
    CUtensorMap tq, tk;
    const int N = kQT * s.H_I;
    const bool heads = s.H_Ik > 1;  // the paper's form: a key per indexer head
    if (heads) {
        // [rows][head][64] views: a box is one head of 32 queries or 128 keys
        if (!make_tmap_bf16_3d(&tq, q_I, kDI, 8, (uint64_t)s.B * s.T, kDI, 8 * kDI, kDI, 1, kQT) ||
            !make_tmap_bf16_3d(&tk, k_I, kDI, 8, (uint64_t)s.B * s.N_max, kDI, 8 * kDI, kDI, 1, kKT))
            return cudaErrorInvalidValue;
    } else if (!make_tmap_bf16_rows(&tq, q_I, kDI, (uint64_t)s.B * s.T * s.H_I, (uint32_t)N) ||
               !make_tmap_bf16_rows(&tk, k_I, kDI, (uint64_t)s.B * s.N_max, kKT)) {
        return cudaErrorInvalidValue;
    }
    static bool attrs[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        cudaError_t e = cudaSuccess;
        const int sm = ScoreSmem::total;
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_index_scores_tc<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_index_scores_tc<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_index_scores_tc<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_index_scores_tc<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_index_scores_heads_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     HeadsSmem::total);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_topm_rows_fast, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     RowSmem::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    const dim3 grid(s.B * P.nqt);
    if (heads) k_index_scores_heads_tc<<<grid, kScoreThreads, HeadsSmem::total, st>>>(tq, tk, P);
    else switch (s.H_I) {
        case 1: k_index_scores_tc<1><<<grid, kScoreMainThreads, ScoreSmem::total, st>>>(tq, tk, P); break;
        case 2: k_index_scores_tc<2><<<grid, kScoreMainThreads, ScoreSmem::total, st>>>(tq, tk, P); break;
        case 4: k_index_scores_tc<4><<<grid, kScoreMainThreads, ScoreSmem::total, st>>>(tq, tk, P); break;
        default: k_index_scores_tc<8><<<grid, kScoreMainThreads, ScoreSmem::total, st>>>(tq, tk, P); break;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    RowParams R;
    R.B = s.B; R.T = s.T; R.n_past = s.n_past; R.Lpad = P.Lpad; R.M = s.M;
    R.keys = P.keys; R.idx = idx; R.count = count; R.status = P.status;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(s.B * s.T);
    cfg.blockDim = dim3(kRowThreads);
    cfg.dynamicSmemBytes = RowSmem::total;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_topm_rows_fast, R);
}

}  // namespace lisa
