// LISA decode step for B200 (sm_100a): four kernels chained by programmatic
// dependent launch (each starts launching while its predecessor runs), no
// inter-CTA waiting.
//
// Step semantics (LISA, arXiv 2607.19358v1: the generation step of Sec. 3.2 and
// Eq. 1; Sec. 3.1 and Sec. 3.3 Eq. 3-4 for the linear branch): append the new
// token, score every cached key with the Lightning Indexer, keep the top M,
// attend over them, run the linear branch, mix the two with the gate.
//
// K1 scan (grid B x S1, 8 scan warps + 4 linear-branch warps per CTA).
//    Scan warps: CTA j of sequence b scores keys [j*KPC, (j+1)*KPC).  The k_I
//    rows arrive by TMA (128-row boxes, 128-byte swizzle); scan warp w owns
//    ring slot w and scores whole boxes on the tensor cores (mma m16n8k16:
//    keys x indexer heads, K = d_I), then ReLU, head weights and head sum.
//    The order-preserving keys of the scores go to a workspace row, and each
//    key's top 12 bits are counted in a shared-memory histogram of the CTA,
//    added to the sequence's histogram once the CTA's keys are done.
//    Linear-branch warps (concurrently): one slice (sequence, KV head, 32
//    value columns) of S += phi(k)^T v and o_lin = phi(q) S (/ phi(q).z).
//    CTA 0 of each sequence appends the new k, v, k_I to the caches.
// K2 select (grid B, 1024 threads): the exact top-M of the key row (radix
//    select: the 12-bit digit from the histogram, two 10-bit refinements over
//    the keys of the threshold digit, ranks in position order; ties keep the
//    lowest positions), written once as the sequence's index row; clears the
//    histogram for the next call.
// K3 attend (grid B x S2, 256 threads): CTA j takes ranks [j*per, (j+1)*per)
//    of the index row; their K and V rows (all KV heads of a position are one
//    row) are gathered by cp.async into a shared-memory ring and attended with
//    an online softmax on the tensor cores.  Partial (max, sum, output) triples
//    go to the workspace.
// K4 combine (grid B x H_q, one thread per output dim): merges the partials,
//    gates with the linear branch, writes o; advances z (elu+1 mode).
//
// The only waits are on TMA mbarriers, each bounded: a wait that gives up
// records LISA_ERR_TIMEOUT in the status word and dependent work is skipped.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include <algorithm>

#include "lisa_fast.cuh"
#include "lisa_internal.cuh"
#include "attend_core.cuh"
#include "decode_linear.cuh"
#include "select_row.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kD = 128;               // head dimension of this path
constexpr int kDI = 64;               // indexer dimension of this path
constexpr int kScanThreads = 256;
constexpr int kScanRows = 128;        // keys per TMA box (16 per warp)
constexpr int kScanStages = 8;        // boxes in flight per CTA
constexpr int kBoxBytes = kScanRows * kDI * 2;
constexpr int kLaCols = dec::kLaCols;  // linear-state columns per slice
constexpr int kMaxPer = 2048;         // positions per attend CTA in the window step
constexpr uint32_t kWaitTries = 1u << 22;

struct Params {
    int B, n, ns, N_max, H_q, H_kv, group, H_I, H_Ik, M, phi;
    int S1, KPC;        // scan CTAs per sequence, keys per scan CTA
    int S2, per;        // attend CTAs per sequence, selected positions per attend CTA
    int window;         // 1: the sparse branch attends over the last M positions (no indexer)
    int la_slices;      // B * H_kv * (kD / kLaCols)
    int rowbytes;       // bytes of one cached K (or V) row: H_kv * kD * 2
    float scale_log2;   // sm_scale * log2(e)
    const bf16* q;
    const bf16* k_new;
    const bf16* v_new;
    const bf16* q_I;
    const bf16* k_I_new;
    const float* w;
    const bf16* q_L;
    const bf16* k_L;
    const bf16* v_L;
    const bf16* gate;
    bf16* k_cache;
    bf16* v_cache;
    bf16* k_I_cache;
    float* S;
    float* z;
    bf16* o;
    int32_t* idx;
    int32_t* count;
    int32_t* sel;       // [B][M] selected positions: idx, or the workspace copy
    uint32_t* keys;     // workspace [B][ns]: order-preserving keys of the scores
    float* olin;        // workspace [B][H_q][kD]
    float* part;        // workspace [B][S2][H_q][kD + 2]
    unsigned* hist;     // workspace [B][4096]: histogram of the top 12 bits of the score keys
    unsigned* status;
};

__host__ __device__ inline int align_up(int x, int a) { return (x + a - 1) / a * a; }

using dec::kLaThreads;
using dec::kLaBar;
using dec::group_sync;
using dec::feat;
constexpr int kScanBar = 1;  // named barrier of the scan warps (the linear-branch warps use kLaBar)

// ============================================================================ K1: scan
struct ScanSmem {
    static constexpr int ring = 0;                                   // kScanStages boxes
    static constexpr int s_slice = ring + kScanStages * kBoxBytes;   // float[128][32]
    static constexpr int fk = s_slice + kD * kLaCols * 4;            // float[128]
    static constexpr int fq = fk + kD * 4;                           // float[16][128]
    static constexpr int vcol = fq + 16 * kD * 4;                    // float[32]
    static constexpr int zloc = vcol + kLaCols * 4;                  // float[128]
    static constexpr int den = zloc + kD * 4;                        // float[16]
    static constexpr int bars = den + 16 * 4;                        // uint64[kScanStages]
    static constexpr int shist = bars + kScanStages * 8;             // u32[4096] key histogram
    static constexpr int total = shist + 4096 * 4 + 1024;            // + base alignment slack
};

// One box of the paper's indexer form (a key per indexer head, H_I = 8): 16
// positions of 8 key rows each (128-byte rows, 128-byte swizzle).  Lane l
// takes head l / 4 and dims 16 (l % 4) .. + 16; the head's dot product is
// summed over its 4 lanes, ReLU and weight applied, and the heads summed over
// the warp.  The key of position p comes from k_I_new (not yet in the cache).
__device__ __forceinline__ void score_box_per_head(const Params& P, int b, int p, int box0, int k1,
                                                   const uint8_t* tile, uint32_t* srow,
                                                   unsigned* hist, const uint32_t (&qh)[8],
                                                   float w_h) {
    const int lane = threadIdx.x & 31, hh = lane >> 2, part = lane & 3;
    constexpr int kPb = kScanRows / 8;
#pragma unroll 4
    for (int sp = 0; sp < kPb; ++sp) {
        const int pos = box0 + sp;
        const int row = sp * 8 + hh;
        uint4 u0, u1;
        if (pos == p) {
            const uint4* src = reinterpret_cast<const uint4*>(P.k_I_new + ((int64_t)b * 8 + hh) * kDI +
                                                              16 * part);
            u0 = src[0];
            u1 = src[1];
        } else {
            const uint8_t* rp = tile + row * 128;
            const int sw = row & 7;
            u0 = *reinterpret_cast<const uint4*>(rp + (((2 * part) ^ sw) << 4));
            u1 = *reinterpret_cast<const uint4*>(rp + (((2 * part + 1) ^ sw) << 4));
        }
        const uint32_t kw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
        float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw[i]));
            const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qh[i]));
            acc0 = fmaf(kf.x, qf.x, acc0);
            acc1 = fmaf(kf.y, qf.y, acc1);
        }
        float dot = acc0 + acc1;
        dot += __shfl_xor_sync(0xffffffffu, dot, 1);
        dot += __shfl_xor_sync(0xffffffffu, dot, 2);
        float sc = part == 0 ? w_h * fmaxf(dot, 0.0f) : 0.0f;
        sc += __shfl_xor_sync(0xffffffffu, sc, 4);
        sc += __shfl_xor_sync(0xffffffffu, sc, 8);
        sc += __shfl_xor_sync(0xffffffffu, sc, 16);
        if (lane == 0 && pos < k1) {
            const uint32_t kk = order_key(sc);
            srow[pos] = kk;
            atomicAdd(hist + (kk >> 20), 1u);  // the CTA's shared-memory histogram
        }
    }
}

__global__ void __launch_bounds__(kScanThreads + kLaThreads, 1)
    k_decode_scan(const __grid_constant__ CUtensorMap tmap_kI, const Params P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* ring = base + ScanSmem::ring;
    float* s_slice = reinterpret_cast<float*>(base + ScanSmem::s_slice);
    float* fk = reinterpret_cast<float*>(base + ScanSmem::fk);
    float* fq = reinterpret_cast<float*>(base + ScanSmem::fq);
    float* vcol = reinterpret_cast<float*>(base + ScanSmem::vcol);
    float* zloc = reinterpret_cast<float*>(base + ScanSmem::zloc);
    float* den = reinterpret_cast<float*>(base + ScanSmem::den);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + ScanSmem::bars);
    unsigned* shist = reinterpret_cast<unsigned*>(base + ScanSmem::shist);

    ptx::pdl_launch_dependents();
    for (int i = threadIdx.x; i < 4096; i += blockDim.x) shist[i] = 0u;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const int b = blockIdx.x / P.S1, j = blockIdx.x % P.S1;
    const int n = P.n, p = n - 1;
    const int k0 = j * P.KPC;
    const int k1 = min(n, k0 + P.KPC);
    const int nk = P.window ? 0 : max(0, k1 - k0);  // the window step scans nothing
    // a box is 128 k_I rows: 128 positions with one key head, 128 / H_I with a
    // key per indexer head (the paper's form)
    const int pb = kScanRows / P.H_Ik;
    const int nst = (nk + pb - 1) / pb;
    bool ok = true;

    if (tid == 0) {
        for (int i = 0; i < kScanStages; ++i) ptx::mbar_init(&bars[i], 1);
        ptx::fence_mbar_init();
        for (int st = 0; st < min(nst, kScanStages); ++st) {
            ptx::mbar_arrive_expect_tx(&bars[st], kBoxBytes);
            ptx::tma_load_2d(ring + st * kBoxBytes, &tmap_kI, 0,
                             (b * P.N_max + k0 + st * pb) * P.H_Ik, &bars[st]);
        }
    }
    // prefetch this CTA's first linear-state slice
    const int slice = blockIdx.x;
    const int slices_per_b = P.H_kv * (kD / kLaCols);
    const bool la_thread = tid >= kScanThreads;
    if (la_thread && slice < P.la_slices) {
        const int lb = slice / slices_per_b, lg = (slice / (kD / kLaCols)) % P.H_kv;
        const int lc0 = (slice % (kD / kLaCols)) * kLaCols;
        const float* Sg = P.S + ((int64_t)lb * P.H_kv + lg) * kD * kD;
        for (int e = tid - kScanThreads; e < kD * kLaCols / 4; e += kLaThreads) {
            const int i = e / (kLaCols / 4), c = (e % (kLaCols / 4)) * 4;
            ptx::cp_async_16(s_slice + i * kLaCols + c, Sg + (int64_t)i * kD + lc0 + c);
        }
        ptx::cp_async_commit();
    }
    __syncthreads();  // barriers initialised; from here the two warp groups run apart
    if (la_thread) {
        if (slice < P.la_slices) {
            const int lb = slice / slices_per_b, lg = (slice / (kD / kLaCols)) % P.H_kv;
            const int lc0 = (slice % (kD / kLaCols)) * kLaCols;
            dec::linear_slice(P, kScanThreads, lb, lg, lc0, s_slice, fk, fq, vcol, zloc, den);
        }
        for (int sl = slice + gridDim.x; sl < P.la_slices; sl += gridDim.x) {
            const int lb = sl / slices_per_b, lg = (sl / (kD / kLaCols)) % P.H_kv;
            const int lc0 = (sl % (kD / kLaCols)) * kLaCols;
            const float* Sg = P.S + ((int64_t)lb * P.H_kv + lg) * kD * kD;
            for (int e = tid - kScanThreads; e < kD * kLaCols; e += kLaThreads)
                s_slice[e] = Sg[(int64_t)(e / kLaCols) * kD + lc0 + e % kLaCols];
            group_sync(kLaBar, kLaThreads);
            dec::linear_slice(P, kScanThreads, lb, lg, lc0, s_slice, fk, fq, vcol, zloc, den);
        }
        return;
    }
    if (j == 0) {
        // cache append of the new token (K2 reads row p from the inputs, not the cache)
        const int chunks = P.rowbytes / 16;
        const uint4* kn = reinterpret_cast<const uint4*>(P.k_new + (int64_t)b * P.H_kv * kD);
        const uint4* vn = reinterpret_cast<const uint4*>(P.v_new + (int64_t)b * P.H_kv * kD);
        uint4* kd = reinterpret_cast<uint4*>(P.k_cache + ((int64_t)b * P.N_max + p) * P.H_kv * kD);
        uint4* vd = reinterpret_cast<uint4*>(P.v_cache + ((int64_t)b * P.N_max + p) * P.H_kv * kD);
        for (int i = tid; i < chunks; i += kScanThreads) {
            kd[i] = kn[i];
            vd[i] = vn[i];
        }
        if (!P.window && tid < P.H_Ik * kDI / 8) {
            const uint4* kin = reinterpret_cast<const uint4*>(P.k_I_new + (int64_t)b * P.H_Ik * kDI);
            reinterpret_cast<uint4*>(P.k_I_cache + ((int64_t)b * P.N_max + p) * P.H_Ik * kDI)[tid] = kin[tid];
        }
    }

    if (P.window) return;  // no indexer in the sliding-window step

    // Indexer fragments.  mma m16n8k16 with A = 16 keys x 16 dims and B = 16 dims
    // x 8 heads; the thread (gid, tq) holds dims [16 tq, 16 tq + 16) of its rows
    // and k-step s uses dims 16 tq + 4 s + {0,1} / {2,3}: A and B share this dim
    // order, so every dot product is unchanged.
    uint32_t qb[8];
    float w_lo = 0.0f, w_hi = 0.0f;
    if (gid < P.H_I) {
        const uint4* src =
            reinterpret_cast<const uint4*>(P.q_I + ((int64_t)b * P.H_I + gid) * kDI + 16 * tq);
        const uint4 u0 = src[0], u1 = src[1];
        qb[0] = u0.x; qb[1] = u0.y; qb[2] = u0.z; qb[3] = u0.w;
        qb[4] = u1.x; qb[5] = u1.y; qb[6] = u1.z; qb[7] = u1.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) qb[i] = 0u;
    }
    {
        const float* wb = P.w + (int64_t)b * P.H_I;
        if (2 * tq < P.H_I) w_lo = wb[2 * tq];
        if (2 * tq + 1 < P.H_I) w_hi = wb[2 * tq + 1];
    }
    // the paper's form (a key per indexer head): this lane's 16 query dims of
    // head lane / 4, and that head's weight
    uint32_t qh[8];
    float w_h = 0.0f;
    if (P.H_Ik > 1) {
        const int hh = lane >> 2;
        if (hh < P.H_I) {
            const uint4* src =
                reinterpret_cast<const uint4*>(P.q_I + ((int64_t)b * P.H_I + hh) * kDI + 16 * (lane & 3));
            const uint4 u0 = src[0], u1 = src[1];
            qh[0] = u0.x; qh[1] = u0.y; qh[2] = u0.z; qh[3] = u0.w;
            qh[4] = u1.x; qh[5] = u1.y; qh[6] = u1.z; qh[7] = u1.w;
            w_h = P.w[(int64_t)b * P.H_I + hh];
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) qh[i] = 0u;
        }
    }
    // Warp w owns ring slot w: it scores boxes w, w + 8, ... by itself (8 row
    // tiles of 16 keys each) and re-arms its slot; no barrier joins the scan
    // warps.
    uint32_t* srow = P.keys + (int64_t)b * P.ns;
    unsigned* hist = P.hist + (int64_t)b * 4096;
    uint64_t* bar = &bars[warp];
    const uint8_t* tile = ring + warp * kBoxBytes;
    for (int st = warp; st < nst; st += kScanStages) {
        if (!ptx::mbar_wait_bounded(bar, (st / kScanStages) & 1, kWaitTries)) {
            ok = false;
            if (lane == 0) record_error(P.status, kDevTimeout);
            break;
        }
        const int box0 = k0 + st * pb;
        if (P.H_Ik > 1) {
            score_box_per_head(P, b, p, box0, k1, tile, srow, shist, qh, w_h);
        } else
#pragma unroll 2
        for (int rt = 0; rt < kScanRows / 16; ++rt) {
            const int row0 = rt * 16 + gid;
            uint32_t ra[2][8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = row0 + 8 * h;
                uint4 u0, u1;
                if (box0 + row == p) {
                    const uint4* src =
                        reinterpret_cast<const uint4*>(P.k_I_new + (int64_t)b * kDI + 16 * tq);
                    u0 = src[0];
                    u1 = src[1];
                } else {
                    const uint8_t* rp = tile + row * 128;
                    const int sw = row & 7;
                    u0 = *reinterpret_cast<const uint4*>(rp + (((2 * tq) ^ sw) << 4));
                    u1 = *reinterpret_cast<const uint4*>(rp + (((2 * tq + 1) ^ sw) << 4));
                }
                ra[h][0] = u0.x; ra[h][1] = u0.y; ra[h][2] = u0.z; ra[h][3] = u0.w;
                ra[h][4] = u1.x; ra[h][5] = u1.y; ra[h][6] = u1.z; ra[h][7] = u1.w;
            }
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s4 = 0; s4 < 4; ++s4) {
                const uint32_t a[4] = {ra[0][2 * s4], ra[1][2 * s4], ra[0][2 * s4 + 1], ra[1][2 * s4 + 1]};
                ptx::mma_bf16(acc, a, qb[2 * s4], qb[2 * s4 + 1]);
            }
            float s0 = w_lo * fmaxf(acc[0], 0.0f) + w_hi * fmaxf(acc[1], 0.0f);
            float s1 = w_lo * fmaxf(acc[2], 0.0f) + w_hi * fmaxf(acc[3], 0.0f);
            s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
            s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
            // lane tq == 0 keeps key row0, tq == 1 key row0 + 8
            const int pos = box0 + row0 + 8 * tq;
            if (tq < 2 && pos < k1) {
                const uint32_t kk = order_key(tq == 0 ? s0 : s1);
                srow[pos] = kk;
                atomicAdd(shist + (kk >> 20), 1u);
            }
        }
        if (st + kScanStages < nst) {
            // the slot's reads are done: hand it back to the copy engine
            __syncwarp();
            if (lane == 0) {
                ptx::fence_proxy_async_shared();
                ptx::mbar_arrive_expect_tx(bar, kBoxBytes);
                ptx::tma_load_2d(ring + warp * kBoxBytes, &tmap_kI, 0,
                                 (b * P.N_max + k0 + (st + kScanStages) * pb) * P.H_Ik, bar);
            }
        }
    }
    // the CTA's key histogram joins the sequence's: one reduction per non-empty
    // bin (the keys of a row crowd into few bins, so per-key global atomics
    // would queue on the same addresses)
    group_sync(kScanBar, kScanThreads);
    for (int i = tid; i < 4096; i += kScanThreads) {
        const unsigned c = shist[i];
        if (c) atomicAdd(hist + i, c);
    }
    if (!ok && lane == 0) {
        // give this warp's copy still in flight a bounded chance to land before exit
        for (uint32_t par = 0; par < 2; ++par) ptx::mbar_wait_bounded(bar, par, 1u << 16);
    }
}

// ============================================================================ K2: select
// One CTA of kSelNT threads per sequence: the exact top-M of the score row
// (row_topm), written once to the sequence's index row for the attend CTAs.
constexpr int kSelNT = 1024;
constexpr int kSelKeyCap = 40960;  // score keys of a row held in shared memory

struct SelSmem {
    static constexpr int hist = 0;                         // u32[4096]
    static constexpr int cand = hist + 4096 * 4;           // uint2[kCandTotal]
    static constexpr int bc = cand + kCandTotal * 8;       // int[64]
    static constexpr int bar = bc + 64 * 4;                // mbarrier
    static constexpr int row = bar + 128;                  // u32[kSelKeyCap]
    static constexpr int total = row + kSelKeyCap * 4;
    static_assert(total <= 227 * 1024, "shared memory per CTA");
};

// Clears the key histogram of sequence b for the next call (once its reader,
// the select kernel, no longer needs it).
__device__ __forceinline__ void clear_hist(const Params& P, int b) {
    uint4* hz = reinterpret_cast<uint4*>(P.hist + (int64_t)b * 4096);
    for (int i = threadIdx.x; i < 4096 / 4; i += blockDim.x) hz[i] = make_uint4(0u, 0u, 0u, 0u);
}

__global__ void __launch_bounds__(kSelNT, 1) k_decode_select(const Params P) {
    extern __shared__ __align__(128) uint8_t sel_raw[];
    uint64_t* rowbar = reinterpret_cast<uint64_t*>(sel_raw + SelSmem::bar);
    uint32_t* row_smem = reinterpret_cast<uint32_t*>(sel_raw + SelSmem::row);
    const int tid = threadIdx.x, b = blockIdx.x;
    const int n = P.n;
    ptx::pdl_launch_dependents();
    if (tid == 0) {
        ptx::mbar_init(rowbar, 1);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    ptx::pdl_wait_prior();  // score keys and histogram of this call are ready
    int32_t* out = P.sel + (int64_t)b * P.M;
    const int cnt = min(P.M, n);
    if (tid == 0 && P.count) P.count[b] = cnt;
    if (n <= P.M) {
        for (int i = tid; i < P.M; i += kSelNT) out[i] = i < n ? i : -1;
        clear_hist(P, b);
        return;
    }
    // Radix select on the order-preserving score keys, most significant digit
    // first: 12 bits (the histogram the scan kernel built), then 10 and 10 bits
    // over the keys that share the digits found so far.  Ties at the M-th key
    // keep the lowest positions.
    const uint32_t* srow = P.keys + (int64_t)b * P.ns;
    SelectSmem sel;
    sel.hist = reinterpret_cast<unsigned*>(sel_raw + SelSmem::hist);
    sel.bc = reinterpret_cast<int*>(sel_raw + SelSmem::bc);
    sel.cand = reinterpret_cast<uint2*>(sel_raw + SelSmem::cand);
    if (n <= kSelRound) {
        // every thread holds its 16 keys in registers, read from L2
        row_topm<kSelNT, true>(srow, false, n, P.M, P.hist + (int64_t)b * 4096, sel, 0, P.M, out,
                               nullptr, P.status);
        clear_hist(P, b);  // every read of it preceded row_topm's barriers
        return;
    }
    const bool resident = n <= kSelKeyCap;
    if (resident && tid == 0) {
        const int bytes = ((n + 3) / 4) * 16;
        ptx::mbar_arrive_expect_tx(rowbar, bytes);
        for (int off = 0; off < bytes; off += 16384)
            ptx::bulk_load(reinterpret_cast<uint8_t*>(row_smem) + off, srow + off / 4,
                           min(16384, bytes - off), rowbar);
    }
    row_topm<kSelNT>(resident ? row_smem : srow, resident, n, P.M, P.hist + (int64_t)b * 4096, sel,
                     0, P.M, out, resident ? rowbar : nullptr, P.status);
    clear_hist(P, b);
}


// ============================================================================ K3: attend
template <int HKV>
struct Att : AttGeo<HKV> {
    using G = AttGeo<HKV>;
    static constexpr int spos = 0;                                     // int[stages][keys]
    static constexpr int wpos = (kAttStages * G::keys * 4 + 127) / 128 * 128;  // int[kMaxPer] (window step)
    static constexpr int ring = wpos + kMaxPer * 4;
    static constexpr int total = ring + G::ring_bytes;
    static_assert(total <= 227 * 1024, "shared memory per CTA");
};

template <int HKV>
__global__ void __launch_bounds__(kAttThreads, 1) k_decode_attend(const Params P) {
    using A = Att<HKV>;
    extern __shared__ __align__(128) uint8_t att_raw[];
    int* spos = reinterpret_cast<int*>(att_raw + A::spos);
    const int tid = threadIdx.x;
    const int b = blockIdx.x / P.S2, j = blockIdx.x % P.S2;
    const int n = P.n, p = n - 1;
    ptx::pdl_launch_dependents();
    const AttQ q = attn_load_q<HKV>(P.q + (int64_t)b * P.H_q * kD, P.group);  // an input: before the wait
    ptx::pdl_wait_prior();  // the index row of this sequence is complete
    const int cnt = min(P.M, n);
    const int lo = j * P.per, hi = min(cnt, lo + P.per);
    const int mine = max(0, hi - lo);
    const int* pos = P.sel + (int64_t)b * P.M + lo;
    if (P.window) {
        // the last cnt positions; this CTA's share is [n - cnt + lo, n - cnt + hi)
        int* wpos = reinterpret_cast<int*>(att_raw + A::wpos);
        const int first = n - cnt + lo;
        for (int i = tid; i < mine; i += kAttThreads) {
            wpos[i] = first + i;
            if (P.idx) P.idx[(int64_t)b * P.M + lo + i] = first + i;
        }
        if (j == 0) {
            if (P.idx)
                for (int i = cnt + tid; i < P.M; i += kAttThreads) P.idx[(int64_t)b * P.M + i] = -1;
            if (P.count && tid == 0) P.count[b] = cnt;
        }
        pos = wpos;  // attn_core's first barrier publishes the list
    }

    // ---- gather + attention over this CTA's share of the selected positions
    constexpr int kb_row = HKV * kD;
    AttOut r;
    const AttSrc src{P.k_cache, P.v_cache, (int64_t)b * P.N_max, p, p, P.k_new + (int64_t)b * kb_row,
                     P.v_new + (int64_t)b * kb_row};
    attn_core<HKV>(q, att_raw + A::ring, spos, pos, mine, src,
                   P.scale_log2, P.status, r);
    // partial (m, l, O) of this CTA for every query head, from the first warp
    // of each KV head
    const int lane = tid & 31, warp = tid >> 5;
    if (warp % AttGeo<HKV>::wph != 0) return;
    const int g = warp / AttGeo<HKV>::wph, gid = lane >> 2, tq = lane & 3;
    float* prow = P.part + (((int64_t)b * P.S2 + j) * P.H_q + g * P.group) * (kD + 2);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int slot = 2 * tq + h;
        if (slot >= P.group) continue;
        float* rec = prow + (int64_t)slot * (kD + 2);
        if (gid == 0) {
            rec[0] = r.m[h];
            rec[1] = r.l[h];
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            rec[2 + t * 16 + gid] = r.o[t][h];
            rec[2 + t * 16 + gid + 8] = r.o[t][h + 2];
        }
    }
}

// ============================================================================ K4: combine
// One CTA per (sequence, query head), one thread per output dimension: merge
// the attend CTAs' partial (max, sum, output) triples, mix with the linear
// branch through the gate, write o.  Also advances the elu+1 normaliser z.
__global__ void __launch_bounds__(kD) k_decode_combine(const Params P) {
    constexpr int kChunk = 32;  // partials loaded together
    const int b = blockIdx.x / P.H_q, h = blockIdx.x % P.H_q, c = threadIdx.x;
    ptx::pdl_wait_prior();  // the attend kernel's partials are complete
    const float x = __bfloat162float(P.gate[(int64_t)b * P.H_q + h]);
    const float o_lin = __ldcg(P.olin + ((int64_t)b * P.H_q + h) * kD + c);
    const int64_t jstride = (int64_t)P.H_q * (kD + 2);
    const float* rec0 = P.part + ((int64_t)b * P.S2 * P.H_q + h) * (kD + 2);
    float M = -INFINITY, Lsum = 0.0f, O = 0.0f;
#pragma unroll 1
    for (int j0 = 0; j0 < P.S2; j0 += kChunk) {
        float mm[kChunk], ll[kChunk], oo[kChunk];
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
            mm[u] = -INFINITY;
            ll[u] = 0.0f;
            oo[u] = 0.0f;
            if (j0 + u < P.S2) {
                const float* rec = rec0 + (j0 + u) * jstride;
                mm[u] = __ldcg(rec);
                ll[u] = __ldcg(rec + 1);
                oo[u] = __ldcg(rec + 2 + c);
            }
        }
        float cm = M;
#pragma unroll
        for (int u = 0; u < kChunk; ++u) cm = fmaxf(cm, mm[u]);
        if (cm == -INFINITY) continue;
        const float a = exp2f(M - cm);  // M = -inf gives 0
        Lsum *= a;
        O *= a;
#pragma unroll
        for (int u = 0; u < kChunk; ++u) {
            const float wgt = exp2f(mm[u] - cm);  // an empty partial (-inf) weighs 0
            Lsum = fmaf(ll[u], wgt, Lsum);
            O = fmaf(oo[u], wgt, O);
        }
        M = cm;
    }
    const float o_sp = Lsum > 0.0f ? O / Lsum : 0.0f;
    const float gt = 1.0f / (1.0f + __expf(-x));
    P.o[((int64_t)b * P.H_q + h) * kD + c] = __float2bfloat16_rn(gt * o_lin + (1.0f - gt) * o_sp);
    if (P.phi == LISA_PHI_ELU1_NORM && h < P.H_kv) {
        // z <- z + phi(k_L): every reader of the old z (the scan kernel) has finished
        const int64_t zi = ((int64_t)b * P.H_kv + h) * kD + c;
        P.z[zi] += feat(P.phi, __bfloat162float(P.k_L[zi]));
    }
}

// ============================================================================ host side
int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            sms = 148;
    }
    return sms;
}

struct Plan {
    int S1, KPC, S2, per, ns;
    size_t scores, olin, part, hist, sel, end;
};

Plan make_plan(const Shape& s) {
    Plan pl;
    const int sms = num_sms();
    const int n = s.L;
    pl.S1 = std::max(1, std::min(sms / std::max(1, s.B), (n + 15) / 16));
    pl.KPC = align_up((n + pl.S1 - 1) / pl.S1, 16);  // a multiple of the positions per box (16 or 128)
    pl.S1 = (n + pl.KPC - 1) / pl.KPC;
    const int cnt = std::min(s.M, n);
    pl.S2 = std::max(1, std::min(sms / std::max(1, s.B), (cnt + 31) / 32));
    pl.per = (cnt + pl.S2 - 1) / pl.S2;
    pl.S2 = (cnt + pl.per - 1) / pl.per;
    pl.ns = align_up(n, 32);
    size_t off = decode_scratch_offset(s.B);
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    pl.scores = take(sizeof(uint32_t) * (size_t)s.B * pl.ns);
    pl.olin = take(sizeof(float) * (size_t)s.B * s.H_q * kD);
    pl.part = take(sizeof(float) * (size_t)s.B * pl.S2 * s.H_q * (kD + 2));
    pl.hist = decode_hist_offset();
    pl.sel = take(sizeof(int32_t) * (size_t)s.B * s.M);
    pl.end = off;
    return pl;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

size_t fast_decode_ws_bytes(const Shape& s) {
    if (s.B <= 0 || s.L <= 0) return kStatusBytes;
    return std::max(make_plan(s).end, coop_decode_ws_bytes(s));
}

bool fast_decode_supported(const Shape& s, const lisa_decode_args& a, bool window) {
    if (s.dtype != LISA_BF16 || s.T != 1 || s.d != kD) return false;
    if (!window && (s.d_I != kDI || s.H_I > 8)) return false;
    if (!window && !(s.H_Ik == 1 || (s.H_Ik == 8 && s.H_I == 8))) return false;
    if (s.group > 8 || !(s.H_kv == 1 || s.H_kv == 2 || s.H_kv == 4)) return false;
    if (s.L < 1 || s.M < 1 || s.B < 1) return false;
    if (window && make_plan(s).per > kMaxPer) return false;
    const void* ptrs[] = {a.q, a.k_new, a.v_new, a.q_L, a.k_L, a.v_L, a.k_cache, a.v_cache, a.S, a.o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return false;
    if (!window && (!aligned16(a.q_I) || !aligned16(a.k_I_new) || !aligned16(a.k_I_cache)))
        return false;
    if (s.phi == LISA_PHI_ELU1_NORM && !aligned16(a.z)) return false;
    if (!window && !tma_encode_fn()) return false;
    return true;
}

cudaError_t fast_decode_step(const Shape& s, const lisa_decode_args& a, void* ws, cudaStream_t st,
                             bool window) {
    if (coop_decode_supported(s, a, window)) {
        const cudaError_t e = coop_decode_step(s, a, ws, st, window);
        // a cooperative grid that does not fit the device right now takes the
        // four-kernel form below
        if (e != cudaErrorCooperativeLaunchTooLarge) return e;
        (void)cudaGetLastError();
    }
    const Plan pl = make_plan(s);
    Params P;
    P.B = s.B; P.n = s.L; P.ns = pl.ns; P.N_max = s.N_max; P.H_q = s.H_q; P.H_kv = s.H_kv;
    P.group = s.group; P.H_I = s.H_I; P.H_Ik = s.H_Ik; P.M = s.M; P.phi = s.phi;
    P.S1 = pl.S1; P.KPC = pl.KPC; P.S2 = pl.S2; P.per = pl.per; P.window = window ? 1 : 0;
    P.la_slices = s.B * s.H_kv * (kD / kLaCols);
    P.rowbytes = s.H_kv * kD * 2;
    P.scale_log2 = s.sm_scale * 1.4426950408889634f;
    P.q = (const bf16*)a.q; P.k_new = (const bf16*)a.k_new; P.v_new = (const bf16*)a.v_new;
    P.q_I = (const bf16*)a.q_I; P.k_I_new = (const bf16*)a.k_I_new; P.w = a.w;
    P.q_L = (const bf16*)a.q_L; P.k_L = (const bf16*)a.k_L; P.v_L = (const bf16*)a.v_L;
    P.gate = (const bf16*)a.gate_logit_lin;
    P.k_cache = (bf16*)a.k_cache; P.v_cache = (bf16*)a.v_cache; P.k_I_cache = (bf16*)a.k_I_cache;
    P.S = a.S; P.z = a.z; P.o = (bf16*)a.o; P.idx = a.idx; P.count = a.count;
    char* w8 = (char*)ws;
    P.status = (unsigned*)ws;
    P.keys = (uint32_t*)(w8 + pl.scores);
    P.olin = (float*)(w8 + pl.olin);
    P.part = (float*)(w8 + pl.part);
    P.hist = (unsigned*)(w8 + pl.hist);
    P.sel = a.idx ? a.idx : (int32_t*)(w8 + pl.sel);

    CUtensorMap tmap;
    memset(&tmap, 0, sizeof(tmap));  // unused by the window step (it scans no keys)
    if (!window && !make_tmap_bf16_rows(&tmap, a.k_I_cache, kDI, (uint64_t)s.B * s.N_max * s.H_Ik,
                                        kScanRows))
        return cudaErrorInvalidValue;

    static bool attrs_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_decode_scan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             ScanSmem::total);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_decode_select, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     SelSmem::total);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_decode_attend<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Att<1>::total);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_decode_attend<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Att<2>::total);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(k_decode_attend<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Att<4>::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attrs_set[dev] = true;
    }
    k_decode_scan<<<s.B * pl.S1, kScanThreads + kLaThreads, ScanSmem::total, st>>>(tmap, P);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(s.B * pl.S2);
    cfg.blockDim = dim3(kAttThreads);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!window) {
        cfg.gridDim = dim3(s.B);
        cfg.blockDim = dim3(kSelNT);
        cfg.dynamicSmemBytes = SelSmem::total;
        e = cudaLaunchKernelEx(&cfg, k_decode_select, P);
        if (e != cudaSuccess) return e;
    }
    cfg.gridDim = dim3(s.B * pl.S2);
    cfg.blockDim = dim3(kAttThreads);
    switch (s.H_kv) {
        case 1: cfg.dynamicSmemBytes = Att<1>::total; e = cudaLaunchKernelEx(&cfg, k_decode_attend<1>, P); break;
        case 2: cfg.dynamicSmemBytes = Att<2>::total; e = cudaLaunchKernelEx(&cfg, k_decode_attend<2>, P); break;
        default: cfg.dynamicSmemBytes = Att<4>::total; e = cudaLaunchKernelEx(&cfg, k_decode_attend<4>, P); break;
    }
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(s.B * s.H_q);
    cfg.blockDim = dim3(kD);
    cfg.dynamicSmemBytes = 0;
    return cudaLaunchKernelEx(&cfg, k_decode_combine, P);
}

}  // namespace lisa
