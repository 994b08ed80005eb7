// Sparse softmax attention SA_M over given index rows (lisa_sparse_attn) for
// many query rows, on the tcgen05 tensor cores (LISA, arXiv 2607.19358v1,
// Sec. 3.2 Eq. 1: each query head attends over the positions its token's
// indexer selected; GQA: head h reads KV head h / group).
//
// When the rows of a call select a sizeable share of their causal range (a
// prefill: row t keeps min(M, t+1) of its t+1 positions), gathering every
// selected row for every query moves the same K/V rows through the SMs over
// and over.  Here the selections become a bit mask instead, and the attention
// runs as a flash-attention loop over 128-query x 64-key tiles in which the
// scores of unselected keys are dropped before the softmax:
//
//  k_sel_mask:       one CTA per query row writes the row's selection as bits
//                    (position s -> bit s) and marks, per 128-row query tile,
//                    the 64-key tiles that any of its rows selects from.
//  k_sparse_mask_tc: one CTA per two (query tile, query head) units of one
//                    KV head, normally two heads of the same query tile (the
//                    same selections, the same K/V tiles), so every K/V tile
//                    brought into shared memory feeds 256 query rows.  Warp 0
//                    brings both units' Q tiles (once) and the K tiles, warp 10
//                    the V tiles, of the key tiles either unit marks (TMA,
//                    128-byte swizzle, 4-stage rings); warp 1 owns TMEM, and
//                    warps 1 and 11 each issue one unit's products, per key
//                    tile S_u = Q_u K^T
//                    (M = 128 queries, N = 64 keys, K = 128 dims) into one of
//                    the unit's two TMEM score buffers and O_u += P_u V
//                    (M = 128, N = 128 dims, K = 64 keys; P read from TMEM, V
//                    MN-major straight from its TMA tile) into the unit's TMEM
//                    output; warps 2-5 (unit 0) and 6-9 (unit 1), one query row
//                    per thread (the row's TMEM lane), read S, keep only the
//                    selected keys, update the row's running reference and sum
//                    (the output is rescaled in TMEM only when a selected score
//                    exceeds the reference by more than 2^64, which leaves the
//                    result exact), write P as bf16 over the first half of the
//                    scores it came from, and at the end normalise O and store
//                    it.
//
// Every wait is bounded; one that gives up records LISA_ERR_TIMEOUT, and the
// kernel waits (bounded) for its own copies and MMAs in flight, releases its
// TMEM and returns.  Positions outside [0, p] are skipped by k_sel_mask and
// reported as LISA_ERR_DEVICE_BOUNDS.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include <algorithm>

#include "lisa_fast.cuh"
#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kQT = 128;          // query rows per tile (MMA M)
constexpr int kKT = 64;           // keys per tile
constexpr int kD = 128;           // head dimension of this path
constexpr int kStages = 4;        // K (and V) tiles in flight
constexpr int kThreads = 384;     // warp 0 TMA (Q, K), 1 TMEM + MMA unit 0, 2-9 softmax (one group per unit),
                                  // 10 TMA (V), 11 MMA unit 1
constexpr int kVWarp = 10;
constexpr int kMma1Warp = 11;
constexpr int kMaxTiles = 2048;   // key tiles of a context this path takes (keys <= 131072)
constexpr uint32_t kTries = 1u << 22;  // polls of a wait
constexpr float kLazyP = 1.8446744e19f;  // 2^64: a tile sum above this moves the softmax reference
constexpr uint32_t kTmemCols = 512;  // score buffers (2 per unit) at columns 0-255, the units' outputs at 256, 384
constexpr uint32_t kOCol = 4 * kKT;

struct MaskParams {
    int T, n_past, M, Lw, nqt, nkw;
    const int32_t* idx;
    const int32_t* count;
    uint32_t* mask;  // [B*T][Lw]: bit s of row (b, t) = position s selected
    uint32_t* occ;   // [B*nqt][nkw]: bit k = some row of the query tile selects in key tile k
    unsigned* status;
};

__global__ void __launch_bounds__(256) k_sel_mask(const MaskParams P) {
    extern __shared__ uint32_t wbits[];  // the row's Lw words
    const int row = blockIdx.x, tid = threadIdx.x;
    const int b = row / P.T, t = row % P.T, p = P.n_past + t;
    for (int i = tid; i < P.Lw; i += 256) wbits[i] = 0u;
    __syncthreads();
    const int cnt = max(0, min(P.count[row], P.M));
    const int32_t* ix = P.idx + (int64_t)row * P.M;
    bool bad = false;
    for (int i = tid; i < cnt; i += 256) {
        const int pos = ix[i];
        if (pos < 0 || pos > p) {
            bad = true;
            continue;
        }
        atomicOr(wbits + (pos >> 5), 1u << (pos & 31));
    }
    if (bad) record_error(P.status, kDevBounds);
    __syncthreads();
    // the row out, two words (one 64-key tile) per thread and step; the
    // tiles that hold a selection are OR-ed into the query tile's marks
    const int ntile = P.Lw / 2;
    uint2* dst = reinterpret_cast<uint2*>(P.mask + (int64_t)row * P.Lw);
    const uint2* src = reinterpret_cast<const uint2*>(wbits);
    uint32_t* occ = P.occ + ((int64_t)b * P.nqt + t / kQT) * P.nkw;
    for (int i0 = 0; i0 < ntile; i0 += 256) {
        const int i = i0 + tid;
        bool any = false;
        if (i < ntile) {
            const uint2 v = src[i];
            dst[i] = v;
            any = (v.x | v.y) != 0u;
        }
        const unsigned bal = __ballot_sync(0xffffffffu, any);
        if ((tid & 31) == 0 && bal) atomicOr(occ + (i0 + (tid & ~31)) / 32, bal);
    }
}

struct AttnParams {
    int B, T, H_q, H_kv, group, nqt, Lw, nkw, slots;
    float scale_log2;
    const uint32_t* mask;
    const uint32_t* occ;
    bf16* o;
    unsigned* status;
};

struct Smem {
    static constexpr int q = 0;                                  // 2 units x 2 boxes of 64 dims x 128 rows
    static constexpr int k = q + 2 * 2 * 16384;                  // kStages x (2 x 64 dims x 64 keys)
    static constexpr int v = k + kStages * 16384;                // the same for V
    static constexpr int bars = v + kStages * 16384;             // mbarriers
    static constexpr int misc = bars + 32 * 8;                   // tmem base, tile count, fail
    static constexpr int total = misc + 64 + 1024;               // + base alignment slack
};
static_assert(Smem::total <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    return ptx::mbar_wait_bounded(bar, parity, kTries);
}

// Walks the key tiles that either unit of the CTA visits (the OR of the two
// query tiles' marks), in ascending order.
struct TileCursor {
    const uint32_t* a;
    const uint32_t* b;
    int nkw, w;
    uint32_t bits;
    __device__ TileCursor(const uint32_t* a_, const uint32_t* b_, int nkw_)
        : a(a_), b(b_), nkw(nkw_), w(-1), bits(0u) {}
    __device__ __forceinline__ int next() {
        while (bits == 0u && w + 1 < nkw) {
            ++w;
            bits = __ldg(a + w) | __ldg(b + w);
        }
        if (bits == 0u) return 0;  // past the last mark (callers stop at the count)
        const int t = w * 32 + __ffs(bits) - 1;
        bits &= bits - 1u;
        return t;
    }
};

// The two (query tile, query head) units of a CTA.  Per (sequence, KV head g,
// query tile) there are `slots` CTAs: slot j < group/2 takes heads 2j and
// 2j+1 of the group on that query tile; with an odd group the last slot
// takes the group's last head on two neighbouring query tiles (qt, qt-1),
// counted down from the last tile, so that slot is empty on every other
// tile; a lone first tile pairs with itself and its second copy stores
// nothing.
struct Units {
    int b, g, qt[2], h[2];
    bool live, dup;
};

__device__ __forceinline__ Units cta_units(const AttnParams& P) {
    Units u;
    const int slot = blockIdx.x % P.slots;
    int rest = blockIdx.x / P.slots;
    u.g = rest % P.H_kv;
    rest /= P.H_kv;
    u.b = rest % P.B;
    const int qt = P.nqt - 1 - rest / P.B;  // longest query tiles first
    const int npair = P.group / 2;
    u.live = true;
    u.dup = false;
    if (slot < npair) {
        u.qt[0] = u.qt[1] = qt;
        u.h[0] = u.g * P.group + 2 * slot;
        u.h[1] = u.h[0] + 1;
    } else {
        u.h[0] = u.h[1] = u.g * P.group + P.group - 1;
        u.live = ((P.nqt - 1 - qt) & 1) == 0;
        u.qt[0] = qt;
        u.qt[1] = qt > 0 ? qt - 1 : qt;
        u.dup = qt == 0;
    }
    return u;
}

__global__ void __launch_bounds__(kThreads, 1)
    k_sparse_mask_tc(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const AttnParams P) {
    const Units U = cta_units(P);
    if (!U.live) return;  // (uniform over the CTA: nothing initialised yet)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* qs = base + Smem::q;
    uint8_t* ks = base + Smem::k;
    uint8_t* vs = base + Smem::v;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + Smem::bars);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* k_empty = k_full + kStages;
    uint64_t* v_full = k_empty + kStages;
    uint64_t* v_empty = v_full + kStages;
    // per unit u and score buffer b (index u * 2 + b; key tile i uses buffer i % 2)
    uint64_t* s_full = v_empty + kStages;   // scores written
    uint64_t* p_full = s_full + 4;          // P written over the scores it came from
    uint64_t* pv_done = p_full + 4;         // the P.V product that read it has completed
    uint64_t* mma_all = pv_done + 4;        // every MMA of both issuers has completed
    uint32_t* misc = reinterpret_cast<uint32_t*>(base + Smem::misc);  // [0] tmem, [1] tiles, [2] fail

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = U.b, g = U.g;
    const uint32_t* occ0 = P.occ + ((int64_t)b * P.nqt + U.qt[0]) * P.nkw;
    const uint32_t* occ1 = P.occ + ((int64_t)b * P.nqt + U.qt[1]) * P.nkw;

    if (tid == 0) {
        ptx::mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&k_full[s], 1);
            ptx::mbar_init(&k_empty[s], 2);  // one commit per unit's issuer
            ptx::mbar_init(&v_full[s], 1);
            ptx::mbar_init(&v_empty[s], 2);
        }
        for (int s = 0; s < 4; ++s) {
            ptx::mbar_init(&s_full[s], 1);
            ptx::mbar_init(&p_full[s], 4);
            ptx::mbar_init(&pv_done[s], 1);
        }
        ptx::mbar_init(mma_all, 2);
        ptx::fence_mbar_init();
        misc[2] = 0u;
    }
    if (warp == 1) {
        ptx::tmem_alloc(misc, kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 0) {
        // how many key tiles the CTA visits
        int c = 0;
        for (int w = lane; w < P.nkw; w += 32) c += __popc(__ldg(occ0 + w) | __ldg(occ1 + w));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if (lane == 0) misc[1] = (uint32_t)c;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = misc[0];
    const int n = (int)misc[1];

    if (warp == 0) {
        if (lane == 0 && n > 0) {
            // ---- producer of both units' Q tiles and the K tiles (V has its
            // own warp, so a K load never waits behind a V slot in use)
            bool ok = true;
            ptx::mbar_arrive_expect_tx(q_full, 4 * 16384);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                ptx::tma_load_3d(qs + u * 32768, &tmap_q, U.h[u] * kD, U.qt[u] * kQT, b, q_full);
                ptx::tma_load_3d(qs + u * 32768 + 16384, &tmap_q, U.h[u] * kD + 64, U.qt[u] * kQT, b, q_full);
            }
            TileCursor cur(occ0, occ1, P.nkw);
            int issued = 0;
            for (int i = 0; i < n && ok; ++i) {
                const int s = i % kStages, use = i / kStages;
                const int kt = cur.next();
                if (use > 0) ok = wait_bar(&k_empty[s], (use - 1) & 1);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(&k_full[s], 16384);
                ptx::tma_load_3d(ks + s * 16384, &tmap_k, g * kD, kt * kKT, b, &k_full[s]);
                ptx::tma_load_3d(ks + s * 16384 + 8192, &tmap_k, g * kD + 64, kt * kKT, b, &k_full[s]);
                issued = i + 1;
            }
            if (!ok) {
                misc[2] = 1u;
                record_error(P.status, kDevTimeout);
                // copies still in flight land before the shared memory is released
                for (int i = max(0, issued - kStages); i < issued; ++i)
                    ptx::mbar_wait_bounded(&k_full[i % kStages], (i / kStages) & 1, 1u << 16);
            }
        }
    } else if (warp == kVWarp) {
        if (lane == 0 && n > 0) {
            // ---- producer of the V tiles
            bool ok = true;
            TileCursor cur(occ0, occ1, P.nkw);
            int issued = 0;
            for (int i = 0; i < n && ok; ++i) {
                const int s = i % kStages, use = i / kStages;
                const int kt = cur.next();
                if (use > 0) ok = wait_bar(&v_empty[s], (use - 1) & 1);
                if (!ok) break;
                ptx::mbar_arrive_expect_tx(&v_full[s], 16384);
                ptx::tma_load_3d(vs + s * 16384, &tmap_v, g * kD, kt * kKT, b, &v_full[s]);
                ptx::tma_load_3d(vs + s * 16384 + 8192, &tmap_v, g * kD + 64, kt * kKT, b, &v_full[s]);
                issued = i + 1;
            }
            if (!ok) {
                misc[2] = 1u;
                record_error(P.status, kDevTimeout);
                for (int i = max(0, issued - kStages); i < issued; ++i)
                    ptx::mbar_wait_bounded(&v_full[i % kStages], (i / kStages) & 1, 1u << 16);
            }
        }
    } else if (warp == 1 || warp == kMma1Warp) {
        if (lane == 0 && n > 0) {
            // ---- MMA issuer of unit u (one thread per unit: every tcgen05
            // instruction costs its issuing thread tens of cycles, so one thread
            // for both units would pace the tensor pipe).  Per key tile:
            //   S_u(j) = Q_u K_j^T into score buffer j % 2, once K_j has landed
            //          and the product that read P_u(j-2) from that buffer has
            //          completed;
            //   O_u += P_u(i) V_i, with P_u(i) read from TMEM where the unit's
            //          softmax wrote it over the first half of S_u(i), once P_u(i)
            //          is written and V_i has landed.
            // A K (V) slot is released when both issuers' products that read it
            // have completed (one commit from each).
            const int u = warp == 1 ? 0 : 1;
            const uint32_t idesc_s = ptx::idesc_bf16_f32(kQT, kKT);
            const uint32_t idesc_pv = ptx::idesc_bf16_f32_bmn(kQT, kD);
            const uint64_t qd0 = ptx::sdesc_kmajor_sw128(qs + u * 32768);
            const uint64_t qd1 = ptx::sdesc_kmajor_sw128(qs + u * 32768 + 16384);
            const uint32_t o_col = tmem + kOCol + (uint32_t)(u * kD);
            bool ok = wait_bar(q_full, 0);
            auto issue_s = [&](int j) {
                const int s = j % kStages, bi = u * 2 + (j & 1);
                ok = ok && wait_bar(&k_full[s], (j / kStages) & 1);
                if (j >= 2) ok = ok && wait_bar(&pv_done[bi], ((j >> 1) - 1) & 1);
                if (!ok) return;
                ptx::tc_fence_after();
                const uint64_t kd0 = ptx::sdesc_kmajor_sw128(ks + s * 16384);
                const uint64_t kd1 = ptx::sdesc_kmajor_sw128(ks + s * 16384 + 8192);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint64_t a = (kk < 4 ? qd0 : qd1) + 2 * (kk & 3);
                    const uint64_t bd = (kk < 4 ? kd0 : kd1) + 2 * (kk & 3);
                    ptx::umma_f16(tmem + (uint32_t)(bi * kKT), a, bd, idesc_s, kk > 0);
                }
                ptx::umma_commit(&s_full[bi]);
                ptx::umma_commit(&k_empty[s]);
            };
            issue_s(0);
            if (n > 1) issue_s(1);
            for (int i = 0; i < n && ok; ++i) {
                const int s = i % kStages, bi = u * 2 + (i & 1);
                ok = ok && wait_bar(&v_full[s], (i / kStages) & 1);
                ok = ok && wait_bar(&p_full[bi], (i >> 1) & 1);
                if (!ok) break;
                ptx::tc_fence_after();
                const uint64_t vd = ptx::sdesc_mnmajor_sw128(vs + s * 16384, 8192, 1024);
                const uint32_t pt = tmem + (uint32_t)(bi * kKT);
#pragma unroll
                for (int kk = 0; kk < kKT / 16; ++kk)
                    ptx::umma_f16_ts(o_col, pt + (uint32_t)(8 * kk), vd + (uint64_t)((2048 >> 4) * kk),
                                     idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
                ptx::umma_commit(&pv_done[bi]);
                ptx::umma_commit(&v_empty[s]);
                if (i + 2 < n) issue_s(i + 2);
            }
            if (!ok) {
                misc[2] = 1u;
                record_error(P.status, kDevTimeout);
            }
            // every MMA issued has completed before TMEM is released
            ptx::umma_commit(mma_all);
            ptx::mbar_wait_bounded(mma_all, 0, kTries);
        }
    } else {
        // ---- softmax: group u (four warps) takes unit u over every key
        // tile, with the row's running reference and sum; thread = query row
        const int u = (warp - 2) >> 2;
        const int lb = (warp & 3) * 32;
        const int r = lb + lane;
        const int t = (u == 0 ? U.qt[0] : U.qt[1]) * kQT + r;
        const int h = u == 0 ? U.h[0] : U.h[1];
        const bool valid = t < P.T;
        const uint2* mrow = reinterpret_cast<const uint2*>(P.mask + ((int64_t)b * P.T + (valid ? t : 0)) * P.Lw);
        const uint32_t t_row = tmem + ((uint32_t)lb << 16);
        const uint32_t t_out = t_row + kOCol + (uint32_t)(u * kD);
        float m_used = -INFINITY, l = 0.0f;
        // the row's mask words of the next two tiles
        TileCursor cur(occ0, occ1, P.nkw);
        uint2 mk_a = make_uint2(0u, 0u), mk_b = make_uint2(0u, 0u);
        if (n > 0) {
            const int t0 = cur.next();
            if (valid) mk_a = __ldg(mrow + t0);
        }
        if (n > 1) {
            const int t1 = cur.next();
            if (valid) mk_b = __ldg(mrow + t1);
        }
        bool ok = true;
        for (int i = 0; i < n; ++i) {
            const uint2 mk = mk_a;
            mk_a = mk_b;
            if (i + 2 < n) {
                const int tn = cur.next();
                if (valid) mk_b = __ldg(mrow + tn);
            }
            const int sb = i & 1;
            const uint32_t t_s = t_row + (uint32_t)((u * 2 + sb) * kKT);  // this tile's score buffer
            // (waits agree across the warp: the TMEM accesses that follow are collective)
            if (!__all_sync(0xffffffffu, wait_bar(&s_full[u * 2 + sb], (i >> 1) & 1))) {
                ok = false;
                break;
            }
            ptx::tc_fence_after();
            // the tile's 64 scores, both loads in flight before the one wait
            uint32_t sr[64];
            ptx::tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(sr));
            ptx::tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
            ptx::tmem_ld_wait();
            // The reference m_used only has to keep every selected p = 2^(s - m_used)
            // far from overflow.  So P is computed against the current reference
            // and the tile's sum checked: only when it exceeds 2^64 (some
            // selected score grew past the reference by about that much; +inf
            // included) or the row meets its first selected keys is the masked
            // maximum taken, the reference moved, and P computed again.  A row
            // whose reference moves rescales its output and sum by alpha.
            const uint32_t wlo = mk.x, whi = mk.y;
            const float2 sc2 = make_float2(P.scale_log2, P.scale_log2);
            uint32_t pk[32];
            float lt = 0.0f;
            auto probs = [&](float ref) {
                const float2 nm2 = make_float2(-ref, -ref);
                float2 l2[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
#pragma unroll
                for (int k = 0; k < 64; k += 2) {
                    const uint32_t w = k < 32 ? wlo : whi;
                    const bool s0 = (w & (1u << (k & 31))) != 0u, s1 = (w & (1u << ((k + 1) & 31))) != 0u;
                    const float2 x = ptx::fma2(make_float2(__uint_as_float(sr[k]), __uint_as_float(sr[k + 1])), sc2, nm2);
                    const float p0 = s0 ? ptx::ex2(x.x) : 0.0f;
                    const float p1 = s1 ? ptx::ex2(x.y) : 0.0f;
                    l2[(k >> 1) & 1] = ptx::add2(l2[(k >> 1) & 1], make_float2(p0, p1));
                    pk[k >> 1] = ptx::pack_bf16(p0, p1);
                }
                lt = (l2[0].x + l2[1].x) + (l2[0].y + l2[1].y);
            };
            const bool any_sel = (wlo | whi) != 0u;
            if (m_used != -INFINITY) probs(m_used);
            // (the comparison is false for a NaN sum: NaN scores stay NaN)
            const bool redo = any_sel && (m_used == -INFINITY || lt > kLazyP);
            float alpha = 1.0f;
            bool grow = false;
            if (__any_sync(0xffffffffu, redo)) {
                if (redo) {
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int k = 0; k < 64; ++k) {
                        const uint32_t w = k < 32 ? wlo : whi;
                        if (w & (1u << (k & 31))) m4[k & 3] = fmaxf(m4[k & 3], __uint_as_float(sr[k]));
                    }
                    const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * P.scale_log2;
                    grow = m_used != -INFINITY && mx > m_used;
                    if (grow) alpha = exp2f(m_used - mx);
                    if (m_used == -INFINITY || grow) m_used = mx;
                }
                // (every lane of the warp, with its own reference)
                if (m_used != -INFINITY) probs(m_used);
            }
            if (m_used == -INFINITY) {  // nothing selected in the row so far
                lt = 0.0f;
#pragma unroll
                for (int k = 0; k < 32; ++k) pk[k] = 0u;
            }
            l = l * alpha + lt;
            // P(i) as bf16 pairs over the first 32 columns of the score buffer
            // (the A operand of the P.V product)
            ptx::tmem_st32(t_s, *reinterpret_cast<const uint32_t(*)[32]>(pk));
            if (__any_sync(0xffffffffu, grow)) {
                // the unit's previous product has completed: its output holds
                // every product so far, and none is in flight until P(i) is out
                if (i > 0 && !__all_sync(0xffffffffu, wait_bar(&pv_done[u * 2 + ((i - 1) & 1)], ((i - 1) >> 1) & 1))) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < kD; c += 16) {
                    uint32_t ov[16];
                    ptx::tmem_ld16(t_out + (uint32_t)c, ov);
                    ptx::tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                    ptx::tmem_st16(t_out + (uint32_t)c, ov);
                }
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&p_full[u * 2 + sb]);
        }
        if (!ok) {
            misc[2] = 1u;
            if (lane == 0) record_error(P.status, kDevTimeout);
        }
        // ---- epilogue: divide the unit's output by the row's sum and store
        // bf16 (zeros for a row that selected nothing)
        const bool have = __all_sync(0xffffffffu, ok && n > 0 &&
                                               wait_bar(&pv_done[u * 2 + ((n - 1) & 1)], ((n - 1) >> 1) & 1));
        ptx::tc_fence_after();
        const float inv = (have && l > 0.0f) ? 1.0f / l : 0.0f;
        bf16* orow = P.o + (((int64_t)b * P.T + (valid ? t : 0)) * P.H_q + h) * kD;
        const bool store = valid && !(U.dup && u == 1);
#pragma unroll 1
        for (int c = 0; c < kD; c += 16) {
            uint32_t ov[16];
            if (have) {
                ptx::tmem_ld16(t_out + (uint32_t)c, ov);
                ptx::tmem_ld_wait();
            }
            uint32_t pkd[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                // an output that no product has written is never read
                const float a0 = inv != 0.0f ? __uint_as_float(ov[2 * e]) * inv : 0.0f;
                const float a1 = inv != 0.0f ? __uint_as_float(ov[2 * e + 1]) * inv : 0.0f;
                pkd[e] = ptx::pack_bf16(a0, a1);
            }
            if (store) {
                uint4* dst = reinterpret_cast<uint4*>(orow + c);
                dst[0] = make_uint4(pkd[0], pkd[1], pkd[2], pkd[3]);
                dst[1] = make_uint4(pkd[4], pkd[5], pkd[6], pkd[7]);
            }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, kTmemCols);
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

struct MaskLayout {
    int Lw, nqt, nkw;
    size_t mask, occ, end;
};

MaskLayout mask_layout(const Shape& s) {
    MaskLayout m;
    m.Lw = (s.L + kKT - 1) / kKT * 2;           // 2 words per 64-key tile
    m.nqt = (s.T + kQT - 1) / kQT;
    m.nkw = (m.Lw / 2 + 31) / 32;
    m.mask = kStatusBytes;
    m.occ = m.mask + (((size_t)s.B * s.T * m.Lw * 4 + 255) & ~(size_t)255);
    m.end = m.occ + (((size_t)s.B * m.nqt * m.nkw * 4 + 255) & ~(size_t)255);
    return m;
}

}  // namespace

// The masked tensor-core form pays for every key of a visited 64-key tile,
// the gather form for every selected key of every row: prefer the first when
// the rows keep a sizeable share of their causal range.  The estimate assumes
// min(M, p + 1) selected positions per row (what lisa_topm writes).
bool sparse_mask_preferred(const Shape& s) {
    if (s.dtype != LISA_BF16 || s.d != kD || s.T < kQT) return false;
    if (s.L > kMaxTiles * kKT) return false;
    double sel = 0.0, causal = 0.0;
    for (int t = 0; t < s.T; t += 16) {  // every 16th row is plenty for the ratio
        const double p1 = (double)s.n_past + t + 1;
        sel += std::min((double)s.M, p1);
        causal += p1;
    }
    return sel >= causal / 16.0;
}

size_t sparse_mask_ws_bytes(const Shape& s) { return mask_layout(s).end; }

bool sparse_mask_supported(const Shape& s, const void* q, const void* k, const void* v) {
    if (!sparse_mask_preferred(s)) return false;
    if (!(aligned16(q) && aligned16(k) && aligned16(v))) return false;
    return tma_encode_fn() != nullptr;
}

cudaError_t sparse_mask_attention(const Shape& s, const void* q, const void* k, const void* v,
                                  const int32_t* idx, const int32_t* count, void* o, void* ws,
                                  cudaStream_t st) {
    const MaskLayout lay = mask_layout(s);
    char* w8 = static_cast<char*>(ws);
    uint32_t* mask = reinterpret_cast<uint32_t*>(w8 + lay.mask);
    uint32_t* occ = reinterpret_cast<uint32_t*>(w8 + lay.occ);
    cudaError_t e = cudaMemsetAsync(occ, 0, (size_t)s.B * lay.nqt * lay.nkw * 4, st);
    if (e != cudaSuccess) return e;

    MaskParams mp;
    mp.T = s.T; mp.n_past = s.n_past; mp.M = s.M; mp.Lw = lay.Lw; mp.nqt = lay.nqt; mp.nkw = lay.nkw;
    mp.idx = idx; mp.count = count; mp.mask = mask; mp.occ = occ; mp.status = static_cast<unsigned*>(ws);
    k_sel_mask<<<s.B * s.T, 256, (size_t)lay.Lw * 4, st>>>(mp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    CUtensorMap tq, tk, tv;
    memset(&tq, 0, sizeof(tq));
    memset(&tk, 0, sizeof(tk));
    memset(&tv, 0, sizeof(tv));
    const uint64_t qrow = (uint64_t)s.H_q * kD, kvrow = (uint64_t)s.H_kv * kD;
    if (!make_tmap_bf16_3d(&tq, q, qrow, s.T, s.B, qrow, (uint64_t)s.T * qrow, 64, kQT) ||
        !make_tmap_bf16_3d(&tk, k, kvrow, s.L, s.B, kvrow, (uint64_t)s.N_max * kvrow, 64, kKT) ||
        !make_tmap_bf16_3d(&tv, v, kvrow, s.L, s.B, kvrow, (uint64_t)s.N_max * kvrow, 64, kKT))
        return cudaErrorInvalidValue;

    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(k_sparse_mask_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Smem::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    AttnParams ap;
    ap.B = s.B; ap.T = s.T; ap.H_q = s.H_q; ap.H_kv = s.H_kv; ap.group = s.group; ap.nqt = lay.nqt;
    ap.Lw = lay.Lw; ap.nkw = lay.nkw; ap.slots = s.group / 2 + (s.group & 1);
    ap.scale_log2 = s.sm_scale * 1.4426950408889634f;
    ap.mask = mask; ap.occ = occ; ap.o = static_cast<bf16*>(o); ap.status = static_cast<unsigned*>(ws);
    const int64_t grid = (int64_t)s.B * lay.nqt * s.H_kv * ap.slots;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    k_sparse_mask_tc<<<(unsigned)grid, kThreads, Smem::total, st>>>(tq, tk, tv, ap);
    return cudaGetLastError();
}

}  // namespace lisa
