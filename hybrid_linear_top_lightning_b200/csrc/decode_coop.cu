// LISA decode step for B200 (sm_100a) as ONE cooperative kernel.
//
// Step semantics (LISA, arXiv 2607.19358v1: the generation step of Sec. 3.2
// and Eq. 1; Sec. 3.1 and Sec. 3.3 Eq. 3-4 for the linear branch): append the
// new token, score every cached key with the Lightning Indexer, keep the top
// M, attend over them, run the linear branch, mix the two with the gate.
//
// Each sequence b owns `ncta` CTAs (one per SM, all resident: cooperative
// launch); CTA j owns the positions [j*KPC, (j+1)*KPC) from start to end.
//  A. Scan warps 0-7: the CTA's k_I rows arrive by TMA (128-row boxes, 16-row
//     boxes for the range's tail; 128-byte swizzle) into 8 warp-owned slots;
//     each warp scores its slot on the tensor cores (keys x indexer heads),
//     applies ReLU, weights and the head sum, and keeps the order-preserving
//     32-bit keys of the scores in shared memory with a histogram of their top
//     12 bits.  Linear-branch warps 8-11 meanwhile advance the CTA's slices of
//     the state S and read o_lin out.  CTA 0 appends the new token.
//  B. The exact top-M threshold, agreed by the sequence's CTAs through global
//     memory.  Exchange 1: the CTA histograms are summed and every CTA finds
//     the 12-bit digit D1 holding the M-th largest key.  Keys above D1 are
//     selected whatever the exact threshold is: warps 0-7 list this CTA's in
//     one pass that also publishes its keys of digit D1 as (key, position)
//     candidates and adds their bits [19:10] to the sequence's second-digit
//     histogram (exchange 2), and the gather starts.  Meanwhile warps 9-11
//     refine: the second digit from that histogram, the third from the
//     candidates, giving the exact M-th key tau and how many keys equal to
//     tau are kept (the lowest positions); the CTA's selected keys of digit D1
//     are then appended to its list.
//  C. The K rows of the listed positions (all KV heads of a position are one
//     row) arrive by 1-D bulk copies of warp 8 in a ring of 16-key stages; each
//     attention warp (0-7) fetches its own KV head's part of the V rows by
//     16-byte cp.async copies and consumes the stages on the tensor cores
//     (keys on the MMA M side, the query heads of a GQA group on N) with an
//     online softmax.  The partial (max, sum, output) of every query head goes
//     to global memory.
//  D. After exchange 3: every CTA writes its share of the index row (when
//     asked for), merges the partials of a few query heads, gates them with
//     the linear branch and writes o; z advances in the elu+1 mode.
//
// The exchanges are counters in the workspace that are zero between calls: a
// CTA arrives with a release add and polls with acquire loads until all ncta
// have arrived; the last CTA to leave exchange 3 zeroes them.  Every wait
// (counter polls, TMA and bulk-copy mbarriers) is bounded; one that gives up
// records LISA_ERR_TIMEOUT and the kernel runs on to its end with every access
// still inside its buffers.  After LISA_ERR_TIMEOUT the workspace must be
// zero-filled again before the next call.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include <algorithm>

#include "attend_core.cuh"
#include "decode_linear.cuh"
#include "lisa_fast.cuh"
#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;
using dec::feat;
using dec::group_sync;

constexpr int kD = 128;                  // head dimension of this path
constexpr int kDI = 64;                  // indexer dimension of this path
constexpr int kMainThreads = 256;        // warps 0-7: scan, then attention
constexpr int kThreads = kMainThreads + dec::kLaThreads;  // + warps 8-11: linear branch, gather
constexpr int kLaCols = dec::kLaCols;
constexpr int kSlots = 8;                // scan slots, one per scan warp
constexpr int kSlotRows = 128;           // k_I rows per slot
constexpr int kSlotBytes = kSlotRows * kDI * 2;
constexpr int kBoxRows = 16;             // rows per TMA box
constexpr int kBoxBytes = kBoxRows * kDI * 2;
constexpr int kGK = 16;                  // keys per gather stage
constexpr int kMaxStages = 16;
// The ring holds the scan slots in phase A, the gather stages in phase C and
// the exchange of softmax states at the end of C.
constexpr int kRingBytes = 163 * 1024;
// The ring's top: the linear-branch buffers in phase A, then the candidates of
// the threshold digit (both used by warps 8-11 only); the gather stages (4 of 16
// keys at 4 KV heads) stay below it, so the attention warps can fill them while
// the linear branch still runs.
constexpr int kCandBytes = 32 * 1024;
constexpr int kCandOff = kRingBytes - kCandBytes;
constexpr int kCandSmem = kCandBytes / 8;
constexpr int kLaOff = kCandOff;
constexpr int kLaBytes = kD * kLaCols * 4 + kD * 4 + 8 * kD * 4 + kLaCols * 4 + kD * 4 + 16 * 4;
constexpr int kHistOff = kRingBytes;                 // u32[4096]
constexpr int kBarOff = kHistOff + 4096 * 4;         // mbarriers: full[16], empty[16], scan[8]
constexpr int kMiscOff = kBarOff + 512;              // int[128]
constexpr int kKeysOff = kMiscOff + 512;             // u32[KPC], then int[sel_cap]
constexpr int kMaxKPC = 8192;
constexpr int kConsBar = 1;              // named barrier of the attention warps (0-7)
constexpr int kMiscCBase = 96;    // misc: this CTA's range of the candidate list
constexpr int kRefBar = 4;               // named barrier of the refinement warps (9-11)
constexpr int kRefFirst = kMainThreads + 32;
constexpr int kRefThreads = kThreads - kRefFirst;
constexpr uint32_t kWaitTries = 1u << 22;
constexpr uint32_t kSpinTries = 1u << 20;
static_assert(kLaOff + kLaBytes <= kRingBytes && kSlots * kSlotBytes <= kLaOff,
              "linear-branch buffers above the scan slots and the gather stages");
static_assert(8 * 36 * 32 * 4 <= kCandOff, "softmax-state exchange below the candidates");

struct CoopParams {
    int B, n, N_max, H_q, H_kv, group, H_I, H_Ik, M, phi;
    int window;         // 1: the Stage-1 step, attending over the last M positions (no indexer)
    int ncta, KPC;      // CTAs per sequence, positions per CTA
    int nstg;           // gather stages in the ring
    int rowbytes;       // bytes of one cached K (or V) row: H_kv * kD * 2
    int krow;           // its padded shared-memory row
    int stage_bytes;    // 2 * kGK * krow
    int sel_cap;        // min(KPC, M): selected positions a CTA can hold
    int ns;             // candidate capacity per sequence
    int spos_off;       // shared-memory offset of the selected positions
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
    unsigned* status;
    unsigned* ghist;    // [B][4096] sums of the CTA histograms (zero between calls)
    unsigned* ghist2;   // [B][1024] histogram of bits [19:10] of the keys of digit D1 (zero between calls)
    unsigned* sync;     // [B][32]: arrivals of the 3 exchanges, departures, candidate count
    float* olin;        // [B][H_q][kD]
    float* part;        // [B][ncta][H_q][kD + 2]
    uint2* cand;        // [B][ns] (key, position)
    int* gsel;          // [B][ncta] selected positions per CTA
};

__host__ __device__ inline int align_up(int x, int a) { return (x + a - 1) / a * a; }

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Barrier of a group of NT threads starting at a warp boundary: bar.sync 0
// for the whole block, a named barrier otherwise.
template <int NT>
__device__ __forceinline__ void gsync(int bar) {
    if (NT == kThreads)
        __syncthreads();
    else
        asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(NT) : "memory");
}

// Arrival on counter c (release: this thread's earlier writes, and those
// ordered before it by a barrier, are visible to whoever acquires the count).
__device__ __forceinline__ void seq_arrive(unsigned* c) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(c) : "memory");
}
// Polls (at most `tries` times) until all ncta CTAs have arrived on counter c.
__device__ __forceinline__ void seq_wait(const unsigned* c, int ncta, unsigned* status,
                                         uint32_t tries = kSpinTries) {
    uint32_t i = 0;
    while (ld_acquire_gpu(c) < (unsigned)ncta) {
        if (++i > tries) {
            record_error(status, kDevTimeout);
            break;
        }
    }
}

// The CTAs of one sequence meet here: each arrives on counter c, then polls
// (bounded) until all ncta have; memory written before the meeting by the
// group's threads of any of them is visible to all after it.  Called by a
// group of NT threads (lt = thread index within the group).  `skip_arrival`
// and `tries` serve the fault-injection hook of the workspace header only.
template <int NT>
__device__ void seq_barrier(unsigned* c, int ncta, unsigned* status, int bar, int lt,
                            bool skip_arrival = false, uint32_t tries = kSpinTries) {
    gsync<NT>(bar);
    if (lt == 0) {
        if (!skip_arrival) seq_arrive(c);
        seq_wait(c, ncta, status, tries);
    }
    gsync<NT>(bar);
}

// Exclusive scan of v over a group of NT threads; `total` gets the sum.
template <int NT>
__device__ __forceinline__ int grp_excl_scan(int v, int lt, int bar, int* scratch, int& total) {
    constexpr int kW = NT / 32;
    const int lane = lt & 31, w = lt >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) scratch[w] = incl;
    gsync<NT>(bar);
    const int ws = lane < kW ? scratch[lane] : 0;
    int wincl = ws;
#pragma unroll
    for (int o = 1; o < kW; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wincl, o);
        if (lane >= o) wincl += y;
    }
    total = __shfl_sync(0xffffffffu, wincl, kW - 1);
    const int woff = __shfl_sync(0xffffffffu, wincl - ws, w);
    gsync<NT>(bar);
    return woff + incl - v;
}

// The bin of a histogram h[0..nbins) (larger bin = larger keys) holding the
// need-th largest key, 1 <= need <= sum(h): bc[0] = the bin, bc[1] = the rank
// of that key within the bin counted from its top, bc[2] = the bin's count.
// Thread lt of the group sums bins [lt*bpt, (lt+1)*bpt); a scan of the sums
// tells the thread whose range holds the key.  bc[32..] is scan scratch.
// Ends with a barrier of the group.
template <int NT>
__device__ void find_bin(const unsigned* h, int nbins, int need, int* bc, int lt, int bar) {
    const int bpt = (nbins + NT - 1) / NT;
    const int lo = min(nbins, lt * bpt), hi = min(nbins, lo + bpt);
    int tsum = 0;
    for (int q = lo; q < hi; ++q) tsum += (int)h[q];
    if (lt == 0) {  // safe values, should no bin qualify (inconsistent counts)
        bc[0] = 0;
        bc[1] = 1;
        bc[2] = 0;
    }
    int total;
    const int below = grp_excl_scan<NT>(tsum, lt, bar, bc + 32, total);
    const int above = total - below - tsum;
    if (above < need && need <= above + tsum) {
        int acc = above;
        for (int q = hi - 1; q >= lo; --q) {
            if (acc + (int)h[q] >= need) {
                bc[0] = q;
                bc[1] = need - acc;
                bc[2] = (int)h[q];
                break;
            }
            acc += (int)h[q];
        }
    }
    gsync<NT>(bar);
}

// ---------------------------------------------------------------- phase A: scoring
// One slot of keys with one key head (H_Ik = 1): positions pos0 .. pos0+npos.
// mma m16n8k16 with A = 16 keys x 16 dims (rows of the slot, 128-byte
// swizzle) and B = 16 dims x 8 indexer heads: thread (gid, tq) holds dims
// [16 tq, 16 tq + 16) and k-step s uses dims 16 tq + 4 s + {0,1} / {2,3} in
// both operands, which leaves every dot product unchanged.
__device__ __forceinline__ void score_slot(const CoopParams& P, int b, int p, int pos0, int npos,
                                           int k0, const uint8_t* slot, uint32_t* skeys,
                                           unsigned* shist, const uint32_t (&qb)[8], float w_lo,
                                           float w_hi) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tq = lane & 3;
    const int tiles = (npos + 15) / 16;
#pragma unroll 2
    for (int rt = 0; rt < tiles; ++rt) {
        const int row0 = rt * 16 + gid;
        uint32_t ra[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = row0 + 8 * h;
            uint4 u0, u1;
            if (pos0 + row == p) {  // the new token's key is not in the cache yet
                const uint4* src = reinterpret_cast<const uint4*>(P.k_I_new + (int64_t)b * kDI + 16 * tq);
                u0 = src[0];
                u1 = src[1];
            } else {
                const uint8_t* rp = slot + row * 128;
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
        const int r = row0 + 8 * tq;
        if (tq < 2 && r < npos) {
            const uint32_t kk = order_key(tq == 0 ? s0 : s1);
            skeys[pos0 + r - k0] = kk;
            atomicAdd(shist + (kk >> 20), 1u);
        }
    }
}

// One slot of the paper's indexer form (a key per indexer head, H_Ik = H_I =
// 8): 16 positions of 8 key rows each.  Lane l takes head l / 4 and dims
// 16 (l % 4) .. + 16; the head's dot product is summed over its 4 lanes, ReLU
// and weight applied, and the heads summed over the warp.
__device__ __forceinline__ void score_slot_per_head(const CoopParams& P, int b, int p, int pos0,
                                                    int npos, int k0, const uint8_t* slot,
                                                    uint32_t* skeys, unsigned* shist,
                                                    const uint32_t (&qh)[8], float w_h) {
    const int lane = threadIdx.x & 31, hh = lane >> 2, part = lane & 3;
#pragma unroll 4
    for (int sp = 0; sp < npos; ++sp) {
        const int row = sp * 8 + hh;
        uint4 u0, u1;
        if (pos0 + sp == p) {
            const uint4* src =
                reinterpret_cast<const uint4*>(P.k_I_new + ((int64_t)b * 8 + hh) * kDI + 16 * part);
            u0 = src[0];
            u1 = src[1];
        } else {
            const uint8_t* rp = slot + row * 128;
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
        if (lane == 0) {
            const uint32_t kk = order_key(sc);
            skeys[pos0 + sp - k0] = kk;
            atomicAdd(shist + (kk >> 20), 1u);
        }
    }
}

// ---------------------------------------------------------------- the kernel
__global__ void __launch_bounds__(kThreads, 1)
    k_decode_coop(const __grid_constant__ CUtensorMap tmap_slot, const __grid_constant__ CUtensorMap tmap_tail,
                  const CoopParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* ring = base;
    unsigned* shist = reinterpret_cast<unsigned*>(base + kHistOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + kBarOff);
    uint64_t* empty = full + kMaxStages;
    uint64_t* scanb = full + 2 * kMaxStages;
    int* misc = reinterpret_cast<int*>(base + kMiscOff);
    uint32_t* skeys = reinterpret_cast<uint32_t*>(base + kKeysOff);
    int* spos = reinterpret_cast<int*>(base + P.spos_off);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const int b = blockIdx.x / P.ncta, j = blockIdx.x % P.ncta;
    const int n = P.n, p = n - 1;
    // the positions the CTAs of a sequence share out: all n, or the window's last min(M, n)
    const int first = P.window ? n - min(P.M, n) : 0;
    const int k0 = first + j * P.KPC;
    const int k1 = min(n, k0 + P.KPC);
    const int nk = max(0, k1 - k0);
    const bool sel_all = P.window || n <= P.M;  // every position is kept: no scores needed
    unsigned* sync = P.sync + (int64_t)b * 32;
    // Fault-injection hook (words 2-3 of the workspace header, zero in normal
    // use): word 2 = 1 + the index of a CTA of every sequence that leaves out
    // its arrival at exchange 1, word 3 = the poll limit of that exchange (0:
    // the default).  Tests use it to watch a bounded wait give up.
    uint2 hook = make_uint2(0u, 0u);

    for (int i = tid; i < 4096; i += kThreads) shist[i] = 0u;
    if (tid == 0) {
        for (int i = 0; i < kMaxStages; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], P.H_kv);
        }
        for (int i = 0; i < kSlots; ++i) ptx::mbar_init(&scanb[i], 1);
        ptx::mbar_init(scanb + kSlots, 1);      // selection ready
        ptx::mbar_init(scanb + kSlots + 1, 1);  // certainly selected positions listed
        ptx::fence_mbar_init();
    }
    __syncthreads();
    // Launched as a programmatic dependent of the previous kernel on the stream,
    // this CTA has set up its shared memory while that kernel finished; nothing
    // global is touched before the previous kernel has completed.  The next
    // kernel may start its own set-up once every CTA of this one is resident.
    ptx::pdl_wait_prior();
    ptx::pdl_launch_dependents();
    if (tid == 0) hook = __ldcg(reinterpret_cast<const uint2*>(P.status + 2));

    // ======================================================== A: scan | linear branch
    if (warp < kSlots) {
        const int pb = kSlotRows / P.H_Ik;  // positions per slot fill
        const int nfill = sel_all ? 0 : (nk + pb - 1) / pb;
        uint64_t* bar = &scanb[warp];
        uint8_t* slot = ring + warp * kSlotBytes;
        auto issue = [&](int f) {  // lane 0: fill f of this warp's slot
            const int pos0 = k0 + f * pb;
            const int rows = min(pb, k1 - pos0) * P.H_Ik;
            const int row0 = (b * P.N_max + pos0) * P.H_Ik;
            if (rows == kSlotRows) {  // a full slot: one box
                ptx::mbar_arrive_expect_tx(bar, kSlotBytes);
                ptx::tma_load_2d(slot, &tmap_slot, 0, row0, bar);
            } else {  // the range's tail: 16-row boxes
                const int boxes = (rows + kBoxRows - 1) / kBoxRows;
                ptx::mbar_arrive_expect_tx(bar, boxes * kBoxBytes);
                for (int i = 0; i < boxes; ++i)
                    ptx::tma_load_2d(slot + i * kBoxBytes, &tmap_tail, 0, row0 + i * kBoxRows, bar);
            }
        };
        if (lane == 0 && warp < nfill) issue(warp);
        if (j == 0) {
            // cache append of the new token (the scan and the gather read row p from
            // the inputs, not from the caches)
            const int chunks = P.rowbytes / 16;
            const uint4* kn = reinterpret_cast<const uint4*>(P.k_new + (int64_t)b * P.H_kv * kD);
            const uint4* vn = reinterpret_cast<const uint4*>(P.v_new + (int64_t)b * P.H_kv * kD);
            uint4* kd = reinterpret_cast<uint4*>(P.k_cache + ((int64_t)b * P.N_max + p) * P.H_kv * kD);
            uint4* vd = reinterpret_cast<uint4*>(P.v_cache + ((int64_t)b * P.N_max + p) * P.H_kv * kD);
            for (int i = tid; i < chunks; i += kMainThreads) {
                kd[i] = kn[i];
                vd[i] = vn[i];
            }
            if (!P.window && tid < P.H_Ik * kDI / 8) {
                const uint4* kin = reinterpret_cast<const uint4*>(P.k_I_new + (int64_t)b * P.H_Ik * kDI);
                reinterpret_cast<uint4*>(P.k_I_cache + ((int64_t)b * P.N_max + p) * P.H_Ik * kDI)[tid] =
                    kin[tid];
            }
        }
        // query fragments of the indexer (one key head), or of this lane's head
        // in the paper's form
        uint32_t qb[8], qh[8];
        float w_lo = 0.0f, w_hi = 0.0f, w_h = 0.0f;
        const float* wb = P.w + (int64_t)b * P.H_I;
        if (sel_all) {
            // nothing to score (the window step's indexer inputs may be null)
        } else if (P.H_Ik == 1) {
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
            if (2 * tq < P.H_I) w_lo = wb[2 * tq];
            if (2 * tq + 1 < P.H_I) w_hi = wb[2 * tq + 1];
        } else {
            const int hh = lane >> 2;
            if (hh < P.H_I) {
                const uint4* src = reinterpret_cast<const uint4*>(
                    P.q_I + ((int64_t)b * P.H_I + hh) * kDI + 16 * (lane & 3));
                const uint4 u0 = src[0], u1 = src[1];
                qh[0] = u0.x; qh[1] = u0.y; qh[2] = u0.z; qh[3] = u0.w;
                qh[4] = u1.x; qh[5] = u1.y; qh[6] = u1.z; qh[7] = u1.w;
                w_h = wb[hh];
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) qh[i] = 0u;
            }
        }
        bool ok = true;
        int it = 0;
        for (int f = warp; f < nfill; f += kSlots, ++it) {
            if (!ptx::mbar_wait_bounded(bar, it & 1, kWaitTries)) {
                ok = false;
                if (lane == 0) record_error(P.status, kDevTimeout);
                break;
            }
            const int pos0 = k0 + f * pb;
            const int npos = min(pb, k1 - pos0);
            if (P.H_Ik == 1)
                score_slot(P, b, p, pos0, npos, k0, slot, skeys, shist, qb, w_lo, w_hi);
            else
                score_slot_per_head(P, b, p, pos0, npos, k0, slot, skeys, shist, qh, w_h);
            if (f + kSlots < nfill) {
                // the slot's reads are done: hand it back to the copy engine
                __syncwarp();
                if (lane == 0) {
                    ptx::fence_proxy_async_shared();
                    issue(f + kSlots);
                }
            }
        }
        if (!ok && lane == 0) {
            // give the copy still in flight a bounded chance to land before the slot is reused
            for (uint32_t par = 0; par < 2; ++par) ptx::mbar_wait_bounded(bar, par, 1u << 16);
        }
    } else {
        // the linear branch: slices (KV head g, 32 value columns) of this sequence
        float* s_slice = reinterpret_cast<float*>(ring + kLaOff);
        float* fk = s_slice + kD * kLaCols;
        float* fq = fk + kD;
        float* vcol = fq + 8 * kD;
        float* zloc = vcol + kLaCols;
        float* den = zloc + kD;
        const int lt = tid - kMainThreads;
        const int per_head = kD / kLaCols;
        for (int sl = j; sl < P.H_kv * per_head; sl += P.ncta) {
            const int g = sl / per_head, c0 = (sl % per_head) * kLaCols;
            const float* Sg = P.S + ((int64_t)b * P.H_kv + g) * kD * kD;
            for (int e = lt; e < kD * kLaCols / 4; e += dec::kLaThreads) {
                const int i = e / (kLaCols / 4), c = (e % (kLaCols / 4)) * 4;
                ptx::cp_async_16(s_slice + i * kLaCols + c, Sg + (int64_t)i * kD + c0 + c);
            }
            ptx::cp_async_commit();
            dec::linear_slice(P, kMainThreads, b, g, c0, s_slice, fk, fq, vcol, zloc, den);
        }
    }

    // ======================================================== B: the threshold digit
    // Selection state shared with the attention warps and phase D:
    // ssel[0] tau (the exact M-th key), [1] ties this CTA may still take (in
    // position order), [2] all keys equal to tau kept, [3] selected positions
    // of this CTA, [4] of them certainly selected (key digit above the
    // threshold digit: the gather starts with these).
    int* ssel = misc + 100;
    uint64_t* sel_ready = full + 2 * kMaxStages + kSlots;  // the refinement has finished
    uint32_t D1 = 0u;
    int need1 = 0;
    if (warp < 8 && !sel_all) {
        // (the scan warps alone: the linear-branch warps finish meanwhile)
        gsync<kMainThreads>(kConsBar);  // the CTA histogram is complete
        unsigned* gh = P.ghist + (int64_t)b * 4096;
        for (int i = tid; i < 4096; i += kMainThreads) {
            const unsigned c = shist[i];
            if (c) atomicAdd(gh + i, c);
        }
        seq_barrier<kMainThreads>(sync + 0, P.ncta, P.status, kConsBar, tid,
                                  hook.x == (unsigned)j + 1u, hook.y ? hook.y : kSpinTries);
        // the summed histogram from L2: thread t holds bins [16t, 16t + 16)
        static_assert(4096 == 16 * kMainThreads, "16 bins per thread");
        unsigned hv[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(gh) + tid * 4 + k);
            hv[4 * k] = v.x;
            hv[4 * k + 1] = v.y;
            hv[4 * k + 2] = v.z;
            hv[4 * k + 3] = v.w;
        }
        int tsum = 0;
#pragma unroll
        for (int q = 0; q < 16; ++q) tsum += (int)hv[q];
        if (tid == 0) {
            misc[0] = 0;
            misc[1] = 1;
        }
        int total;
        const int below = grp_excl_scan<kMainThreads>(tsum, tid, kConsBar, misc + 32, total);
        const int above = total - below - tsum;
        if (above < P.M && P.M <= above + tsum) {
            int acc = above;
#pragma unroll
            for (int q = 15; q >= 0; --q) {
                if (acc < P.M && acc + (int)hv[q] >= P.M) {
                    misc[0] = tid * 16 + q;
                    misc[1] = P.M - acc;
                }
                acc += (int)hv[q];
            }
        }
        gsync<kMainThreads>(kConsBar);
        D1 = (uint32_t)misc[0];
        need1 = misc[1];
    }
    // From here the warps part: 0-7 list the certainly selected positions, then
    // attend; 8 gathers; 9-11 refine the threshold (when n > M).
    uint64_t* def_ready = sel_ready + 1;  // the certainly selected positions are listed
    int def_full = 0;
    if (warp < 8) {
        if (!sel_all) {
            // keys whose digit is above D1 are selected whatever tau is: listed for
            // the gather; keys of digit D1 are published as candidates for exchange 2
            // (thread t owns keys [t*ch, (t+1)*ch), so both stay in position order;
            // the two counts share one scan, 16 bits each)
            const int ch = (nk + kMainThreads - 1) / kMainThreads;
            const int c_lo = min(nk, tid * ch), c_hi = min(nk, c_lo + ch);
            int mine = 0;
            for (int i = c_lo; i < c_hi; ++i) {
                const uint32_t d = skeys[i] >> 20;
                mine += d > D1 ? 1 : (d == D1 ? 1 << 16 : 0);
            }
            int tot;
            const int at0 = grp_excl_scan<kMainThreads>(mine, tid, kConsBar, misc + 32, tot);
            const int tot_def = tot & 0xFFFF, tot_c = tot >> 16;
            unsigned cbase = 0;
            if (tid == 0 && tot_c) cbase = atomicAdd(sync + 4, (unsigned)tot_c);  // used after def_ready
            int at = at0 & 0xFFFF;
            for (int i = c_lo; i < c_hi; ++i)
                if ((skeys[i] >> 20) > D1) {
                    if (at < P.sel_cap) spos[at] = k0 + i;
                    ++at;
                }
            const int cnt_def = min(tot_def, P.sel_cap);
            def_full = cnt_def / kGK * kGK;
            if (tid == 0) ssel[4] = cnt_def;
            gsync<kMainThreads>(kConsBar);
            if (tid == 0) {
                ptx::mbar_arrive(def_ready);  // the gather starts
                misc[kMiscCBase] = (int)cbase;
            }
            gsync<kMainThreads>(kConsBar);
            uint2* cand = P.cand + (int64_t)b * P.ns;
            unsigned* gh2 = P.ghist2 + (int64_t)b * 1024;
            int ca = misc[kMiscCBase] + (at0 >> 16);
            for (int i = c_lo; i < c_hi; ++i) {
                const uint32_t key = skeys[i];
                if ((key >> 20) == D1) {
                    if (ca < P.ns) cand[ca] = make_uint2(key, (uint32_t)(k0 + i));
                    ++ca;
                    atomicAdd(gh2 + ((key >> 10) & 1023u), 1u);  // the sequence's second digit
                }
            }
            gsync<kMainThreads>(kConsBar);
            if (tid == 0) seq_arrive(sync + 1);  // exchange 2: this CTA's candidates are out
        } else {
            for (int i = tid; i < nk; i += kMainThreads) spos[i] = k0 + i;
            def_full = nk;
            if (tid == 0) {
                ssel[0] = 0;
                ssel[1] = 0;
                ssel[2] = 1;
                ssel[3] = nk;
                ssel[4] = nk;
                if (P.idx) P.gsel[(int64_t)b * P.ncta + j] = nk;
            }
        }
        if (sel_all) {
            gsync<kMainThreads>(kConsBar);
            if (tid == 0) ptx::mbar_arrive(def_ready);
        }
    }

    // ======================================================== C: gather + attention
    if (warp < 8) {
        const int H_kv = P.H_kv, NG = 8 / H_kv;
        const int g = warp % H_kv, qg = warp / H_kv;
        // query fragments (B operand of the score MMA): head gid of the group,
        // dims ks*16 + 2tq (+1) and + 8 (+9); heads past the group are zero
        uint32_t qf[8][2];
        {
            const bool live = gid < P.group;
            const uint32_t* qh = reinterpret_cast<const uint32_t*>(
                P.q + ((int64_t)b * P.H_q + g * P.group + (live ? gid : 0)) * kD);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                qf[ks][0] = live ? __ldg(qh + ks * 8 + tq) : 0u;
                qf[ks][1] = live ? __ldg(qh + ks * 8 + 4 + tq) : 0u;
            }
        }
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
        float o[8][4];
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[t][e] = 0.0f;
        const uint32_t head_off = (uint32_t)(g * kD * 2);
        const int krow = P.krow;
        // stages below `known` positions exist; past it, the count is final once
        // the refinement has reported
        int known = def_full;
        bool fin = sel_all;
        // This warp fetches the V bytes it alone reads (its KV head's 256 bytes
        // of each V row of its stages) with 16-byte cp.async copies, one own stage
        // ahead; the K rows come by the gather warp's bulk copies.  A slot is
        // reused every nstg stages, a multiple of NG, so the V bytes a warp
        // overwrites are ones it has read itself.
        const int64_t rowel = (int64_t)P.H_kv * kD;
        const bf16* vsrc0 = P.v_cache + (int64_t)b * P.N_max * rowel + g * kD;
        const bf16* vnew = P.v_new + (int64_t)b * rowel + g * kD;
        const int ahead = P.nstg / NG - 1;  // own stages of V in flight beyond the current one
        int v_next = qg;                    // the next own stage whose V is not requested yet
        auto request_v = [&](int s) {
            const int nin = min(kGK, known - s * kGK);
            uint8_t* vdst = ring + (s % P.nstg) * P.stage_bytes + kGK * krow + g * kD * 2;
#pragma unroll
            for (int u = 0; u < kGK * 16 / 32; ++u) {
                const int c = lane + 32 * u, key = c >> 4, off = c & 15;
                const int pos = spos[s * kGK + min(key, nin - 1)];
                const bf16* src = pos == p ? vnew : vsrc0 + pos * rowel;
                ptx::cp_async_16(vdst + key * krow + off * 16, reinterpret_cast<const uint4*>(src) + off);
            }
            ptx::cp_async_commit();
        };
#pragma unroll 1
        for (int st = qg;; st += NG) {
            if (st * kGK >= known) {
                if (!fin) {
                    if (!ptx::mbar_wait_bounded(sel_ready, 0, kWaitTries)) {
                        if (lane == 0) record_error(P.status, kDevTimeout);
                        break;
                    }
                    known = reinterpret_cast<volatile int*>(ssel)[3];
                    fin = true;
                }
                if (st * kGK >= known) break;
            }
            while (v_next <= st + NG * ahead && v_next * kGK < known) {
                request_v(v_next);
                v_next += NG;
            }
            if (v_next > st + NG)
                ptx::cp_async_wait_group<1>();  // this stage's V landed (the next one may not have)
            else
                ptx::cp_async_wait_group<0>();
            __syncwarp();
            const int slot = st % P.nstg;
            if (!ptx::mbar_wait_bounded(&full[slot], (st / P.nstg) & 1, kWaitTries)) {
                if (lane == 0) record_error(P.status, kDevTimeout);
                break;
            }
            const uint32_t kb = ptx::smem_u32(ring + slot * P.stage_bytes);
            const int left = known - st * kGK;  // keys of this stage in the list
            attn_stage16(qf, kb, kb + kGK * krow, krow, head_off,
                         left >= kGK ? 0xFFFFu : (1u << left) - 1u, P.scale_log2, m, l, o);
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[slot]);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l[h] += __shfl_xor_sync(0xffffffffu, l[h], 4);
            l[h] += __shfl_xor_sync(0xffffffffu, l[h], 8);
            l[h] += __shfl_xor_sync(0xffffffffu, l[h], 16);
        }
        // the warps of a KV head hand their states to warp g (the ring is free
        // once every attention warp is past its last stage)
        ptx::cp_async_wait_all();  // (V copies requested for stages past a timeout)
        group_sync(kConsBar, kMainThreads);
        float* xf = reinterpret_cast<float*>(ring) + warp * 36 * 32 + lane;  // [36][32] per warp
        if (qg != 0) {
            xf[0] = m[0]; xf[32] = m[1]; xf[64] = l[0]; xf[96] = l[1];
#pragma unroll
            for (int t = 0; t < 8; ++t)
#pragma unroll
                for (int e = 0; e < 4; ++e) xf[(4 + t * 4 + e) * 32] = o[t][e];
        }
        group_sync(kConsBar, kMainThreads);
        if (qg == 0) {
#pragma unroll 1
            for (int k = 1; k < NG; ++k) {
                const float* yf = reinterpret_cast<const float*>(ring) + (warp + k * H_kv) * 36 * 32 + lane;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float mk = yf[h * 32], lk = yf[(2 + h) * 32];
                    const float Mx = fmaxf(m[h], mk);
                    const float a = (m[h] == -INFINITY) ? 0.0f : exp2f(m[h] - Mx);
                    const float c = (mk == -INFINITY) ? 0.0f : exp2f(mk - Mx);
                    m[h] = Mx;
                    l[h] = l[h] * a + lk * c;
#pragma unroll
                    for (int t = 0; t < 8; ++t)
#pragma unroll
                        for (int e = h; e < 4; e += 2) o[t][e] = o[t][e] * a + yf[(4 + t * 4 + e) * 32] * c;
                }
            }
            // partial (m, l, O) of this CTA for the group's query heads
            float* prow = P.part + (((int64_t)b * P.ncta + j) * P.H_q + g * P.group) * (kD + 2);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int hs = 2 * tq + h;
                if (hs >= P.group) continue;
                float* rec = prow + (int64_t)hs * (kD + 2);
                if (gid == 0) {
                    rec[0] = m[h];
                    rec[1] = l[h];
                }
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    rec[2 + t * 16 + gid] = o[t][h];
                    rec[2 + t * 16 + gid + 8] = o[t][h + 2];
                }
            }
        }
    } else if (warp == 8) {
        // producer: the K rows of stage st by 1-D bulk copies, key i by lane i (the
        // attention warps fetch the V rows); a short last stage repeats its first
        // position (those keys are masked)
        const int64_t rowel = (int64_t)P.H_kv * kD;
        const bf16* kn = P.k_new + (int64_t)b * rowel;
        int issued = 0;
        bool ok = ptx::mbar_wait_bounded(def_ready, 0, kWaitTries);
        if (!ok && lane == 0) record_error(P.status, kDevTimeout);
        const int cnt_def = reinterpret_cast<volatile int*>(ssel)[4];
        int known = ok ? (sel_all ? cnt_def : cnt_def / kGK * kGK) : 0;
        bool fin = sel_all || !ok;
        for (int st = 0;; ++st) {
            if (st * kGK >= known) {
                if (!fin) {
                    if (!ptx::mbar_wait_bounded(sel_ready, 0, kWaitTries)) {
                        ok = false;
                        if (lane == 0) record_error(P.status, kDevTimeout);
                        break;
                    }
                    known = reinterpret_cast<volatile int*>(ssel)[3];
                    fin = true;
                }
                if (st * kGK >= known) break;
            }
            const int slot = st % P.nstg;
            if (st >= P.nstg) {
                if (!ptx::mbar_wait_bounded(&empty[slot], ((st / P.nstg) - 1) & 1, kWaitTries)) {
                    ok = false;
                    if (lane == 0) record_error(P.status, kDevTimeout);
                    break;
                }
                ptx::fence_proxy_async_shared();
            }
            uint8_t* dst = ring + slot * P.stage_bytes;
            if (lane == 0) ptx::mbar_arrive_expect_tx(&full[slot], kGK * (uint32_t)P.rowbytes);
            __syncwarp();
            const int nin = min(kGK, known - st * kGK);
            if (lane < kGK) {
                const int pos = spos[st * kGK + min(lane, nin - 1)];
                const bf16* src = pos == p ? kn : P.k_cache + ((int64_t)b * P.N_max + pos) * rowel;
                ptx::bulk_load(dst + lane * P.krow, src, (uint32_t)P.rowbytes, &full[slot]);
            }
            issued = st + 1;
        }
        if (!ok) {
            // copies still in flight land before the ring is reused or the CTA exits
            for (int st = max(0, issued - P.nstg); st < issued; ++st)
                ptx::mbar_wait_bounded(&full[st % P.nstg], (st / P.nstg) & 1, 1u << 16);
        }
    } else if (!sel_all) {
        // refinement (warps 9-11), while the certainly selected rows are gathered:
        // the exact tau among the keys of digit D1 of the whole sequence
        constexpr int NT = kRefThreads;
        const int rt = tid - kRefFirst;
        if (!ptx::mbar_wait_bounded(def_ready, 0, kWaitTries) && rt == 0)
            record_error(P.status, kDevTimeout);
        D1 = (uint32_t)misc[0];
        need1 = misc[1];
        int* rmisc = misc + 48;  // find_bin results [0..2], tie counter [3], scan scratch [32..]
        uint2* cand = P.cand + (int64_t)b * P.ns;
        // thread rt owns keys [rt*ch, (rt+1)*ch)
        const int ch = (nk + NT - 1) / NT;
        const int c_lo = min(nk, rt * ch), c_hi = min(nk, c_lo + ch);
        // exchange 2: every CTA's candidates are out (published by warps 0-7)
        if (rt == 0) seq_wait(sync + 1, P.ncta, P.status);
        gsync<NT>(kRefBar);
        {
            // no CTA reads the summed histogram any more: clear a share of it
            unsigned* gh = P.ghist + (int64_t)b * 4096;
            const int per = (4096 + P.ncta - 1) / P.ncta;
            const int lo = j * per, hi = min(4096, lo + per);
            for (int i = lo + rt; i < hi; i += NT) gh[i] = 0u;
        }
        // the first 8 * NT list entries are loaded with the count (entries past it
        // are discarded), the rest, if any, once the count is known
        constexpr int kCL = 16;  // list entries loaded per thread with the count
        uint2 v[kCL];
#pragma unroll
        for (int k = 0; k < kCL; ++k) v[k] = __ldcg(cand + min(rt + k * NT, P.ns - 1));
        // with them, the sequence's histogram of key bits [19:10] over digit D1
        const uint4* gh2 = reinterpret_cast<const uint4*>(P.ghist2 + (int64_t)b * 1024);
        constexpr int kH2 = (256 + NT - 1) / NT;
        uint4 h2[kH2];
#pragma unroll
        for (int k = 0; k < kH2; ++k)
            if (rt + k * NT < 256) h2[k] = __ldcg(gh2 + rt + k * NT);
        const int C = min((int)__ldcg(sync + 4), P.ns);
        const bool in_smem = C <= kCandSmem;
        uint2* sc = reinterpret_cast<uint2*>(ring + kCandOff);
        if (in_smem) {
#pragma unroll
            for (int k = 0; k < kCL; ++k) {
                const int i = rt + k * NT;
                if (i < C) sc[i] = v[k];
            }
            for (int i0 = kCL * NT; i0 < C; i0 += kCL * NT) {  // kCL loads in flight per thread
#pragma unroll
                for (int k = 0; k < kCL; ++k) {
                    const int i = i0 + rt + k * NT;
                    if (i < C) v[k] = __ldcg(cand + i);
                }
#pragma unroll
                for (int k = 0; k < kCL; ++k) {
                    const int i = i0 + rt + k * NT;
                    if (i < C) sc[i] = v[k];
                }
            }
        }
        auto cand_at = [&](int i) { return in_smem ? sc[i] : __ldcg(cand + i); };
        // second digit: key bits [19:10], from the histogram the CTAs built
#pragma unroll
        for (int k = 0; k < kH2; ++k)
            if (rt + k * NT < 256) reinterpret_cast<uint4*>(shist)[rt + k * NT] = h2[k];
        gsync<NT>(kRefBar);
        find_bin<NT>(shist, 1024, need1, rmisc, rt, kRefBar);
        const uint32_t D2 = (uint32_t)rmisc[0];
        const int need2 = rmisc[1];
        const int cnt2 = rmisc[2];  // keys of the sequence in the 20-bit bin (D1, D2)
        gsync<NT>(kRefBar);
        uint32_t tau;
        int need_eq, tie_prefix = 0;
        bool all_ties;
        if (cnt2 <= 32) {
            // few keys share the 20-bit bin (the usual case): collect them and
            // let one warp rank them directly (descending key; every key equal
            // to tau is among them, so the ties before this CTA's range are too)
            uint2* few = reinterpret_cast<uint2*>(shist);
            if (rt == 0) rmisc[4] = 0;
            gsync<NT>(kRefBar);
            for (int i = rt; i < C; i += NT) {
                const uint2 e = cand_at(i);
                if (((e.x >> 10) & 1023u) == D2) {
                    const int at = atomicAdd(rmisc + 4, 1);
                    if (at < 32) few[at] = e;
                }
            }
            gsync<NT>(kRefBar);
            if (rt < 32) {
                const int m = min(rmisc[4], 32);
                const uint2 me = rt < m ? few[rt] : make_uint2(0u, 0u);
                int gt = 0, eq = 0;
                for (int o = 0; o < m; ++o) {
                    const uint32_t kx = __shfl_sync(0xffffffffu, me.x, o);
                    gt += kx > me.x ? 1 : 0;
                    eq += kx == me.x ? 1 : 0;
                }
                const bool hit = rt < m && gt < need2 && need2 <= gt + eq;
                const unsigned who = __ballot_sync(0xffffffffu, hit);
                const int src = who ? __ffs(who) - 1 : 0;
                const uint32_t tk = __shfl_sync(0xffffffffu, me.x, src);
                const int tgt = __shfl_sync(0xffffffffu, gt, src);
                const int teq = __shfl_sync(0xffffffffu, eq, src);
                const unsigned before =
                    __ballot_sync(0xffffffffu, rt < m && me.x == tk && (int)me.y < k0);
                if (rt == 0) {
                    rmisc[0] = who ? (int)(tk & 1023u) : 0;  // (safe values if the counts disagree)
                    rmisc[1] = who ? need2 - tgt : 1;
                    rmisc[2] = who ? teq : 0;
                    rmisc[3] = __popc(before);
                }
            }
            gsync<NT>(kRefBar);
            tau = (D1 << 20) | (D2 << 10) | (uint32_t)rmisc[0];
            need_eq = rmisc[1];
            all_ties = need_eq >= rmisc[2];
            if (!all_ties) tie_prefix = rmisc[3];
            gsync<NT>(kRefBar);
        } else {
            // third digit: key bits [9:0] of the candidates that share D2
            for (int i = rt; i < 1024; i += NT) shist[i] = 0u;
            gsync<NT>(kRefBar);
            for (int i = rt; i < C; i += NT) {
                const uint32_t key = cand_at(i).x;
                if (((key >> 10) & 1023u) == D2) atomicAdd(shist + (key & 1023u), 1u);
            }
            gsync<NT>(kRefBar);
            find_bin<NT>(shist, 1024, need2, rmisc, rt, kRefBar);
            tau = (D1 << 20) | (D2 << 10) | (uint32_t)rmisc[0];
            need_eq = rmisc[1];
            all_ties = need_eq >= rmisc[2];
            gsync<NT>(kRefBar);
            if (!all_ties) {
                // keys equal to tau at positions before this CTA's range
                if (rt == 0) rmisc[3] = 0;
                gsync<NT>(kRefBar);
                int c = 0;
                for (int i = rt; i < C; i += NT) {
                    const uint2 e = cand_at(i);
                    c += (e.x == tau && (int)e.y < k0) ? 1 : 0;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
                if (lane == 0 && c) atomicAdd(rmisc + 3, c);
                gsync<NT>(kRefBar);
                tie_prefix = rmisc[3];
            }
        }
        // this CTA's selected keys of digit D1, appended after the certain ones
        // (ties ranked by position)
        int n_gt = 0, n_eq = 0;
        for (int i = c_lo; i < c_hi; ++i) {
            const uint32_t key = skeys[i];
            n_gt += ((key >> 20) == D1 && key > tau) ? 1 : 0;
            n_eq += key == tau ? 1 : 0;
        }
        int take_eq = n_eq, tot;
        if (!all_ties) {
            const int eq_before = grp_excl_scan<NT>(n_eq, rt, kRefBar, rmisc + 32, tot);
            take_eq = max(0, min(n_eq, need_eq - tie_prefix - eq_before));
        }
        const int cnt_def = ssel[4];
        int at = cnt_def + grp_excl_scan<NT>(n_gt + take_eq, rt, kRefBar, rmisc + 32, tot);
        int eq_seen = 0;
        for (int i = c_lo; i < c_hi; ++i) {
            const uint32_t key = skeys[i];
            const bool s = ((key >> 20) == D1 && key > tau) || (key == tau && eq_seen++ < take_eq);
            if (s) {
                if (at < P.sel_cap) spos[at] = k0 + i;
                ++at;
            }
        }
        gsync<NT>(kRefBar);  // the appended positions are written
        if (rt == 0) {
            const int cnt = min(cnt_def + tot, P.sel_cap);
            ssel[0] = (int)tau;
            ssel[1] = need_eq - tie_prefix;
            ssel[2] = all_ties ? 1 : 0;
            ssel[3] = cnt;
            if (P.idx) P.gsel[(int64_t)b * P.ncta + j] = cnt;
            ptx::mbar_arrive(sel_ready);
        }
    }
    seq_barrier<kThreads>(sync + 2, P.ncta, P.status, 0, tid);

    // ======================================================== D: index row, combine, gate
    if (P.idx) {
        if (warp == 0) {
            int s = 0;
            for (int i = lane; i < j; i += 32) s += __ldcg(P.gsel + (int64_t)b * P.ncta + i);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            if (lane == 0) misc[4] = s;
        }
        __syncthreads();
        // this CTA's selected positions in order: key > tau, or key == tau among
        // the first ssel[1] ties (thread t owns keys [t*ch, (t+1)*ch))
        const uint32_t tau = (uint32_t)ssel[0];
        const int ties = ssel[1];
        const bool all_ties = ssel[2] != 0;
        const int cnt = ssel[3];
        const int ch = (nk + kThreads - 1) / kThreads;
        const int c_lo = min(nk, tid * ch), c_hi = min(nk, c_lo + ch);
        int n_gt = 0, n_eq = 0;
        if (sel_all) {
            n_gt = c_hi - c_lo;
        } else {
            for (int i = c_lo; i < c_hi; ++i) {
                const uint32_t key = skeys[i];
                n_gt += key > tau ? 1 : 0;
                n_eq += key == tau ? 1 : 0;
            }
        }
        int take_eq = n_eq, tot;
        if (!sel_all && !all_ties) {
            const int eq_before = grp_excl_scan<kThreads>(n_eq, tid, 0, misc + 32, tot);
            take_eq = max(0, min(n_eq, ties - eq_before));
        }
        int at = misc[4] + grp_excl_scan<kThreads>(n_gt + take_eq, tid, 0, misc + 32, tot);
        int32_t* row = P.idx + (int64_t)b * P.M;
        int eq_seen = 0;
        for (int i = c_lo; i < c_hi; ++i) {
            bool s = true;
            if (!sel_all) {
                const uint32_t key = skeys[i];
                s = key > tau || (key == tau && eq_seen++ < take_eq);
            }
            if (s) {
                if (at < P.M) row[at] = k0 + i;
                ++at;
            }
        }
        if (j == P.ncta - 1)
            for (int i = misc[4] + cnt + tid; i < P.M; i += kThreads) row[i] = -1;
    }
    if (j == 0 && tid == 0 && P.count) P.count[b] = min(P.M, n);
    if (!sel_all) {
        // every CTA read the second-digit histogram before exchange 3: clear a share
        unsigned* gh2 = P.ghist2 + (int64_t)b * 1024;
        const int per = (1024 + P.ncta - 1) / P.ncta;
        const int lo = j * per, hi = min(1024, lo + per);
        for (int i = lo + tid; i < hi; i += kThreads) gh2[i] = 0u;
    }
    {
        constexpr int kChunk = 24;  // partials loaded together (every CTA's at B = 8)
        const int c = tid & (kD - 1), sub = tid / kD;
        const int64_t jstride = (int64_t)P.H_q * (kD + 2);
        for (int h = j + sub * P.ncta; h < P.H_q; h += (kThreads / kD) * P.ncta) {
            const float* rec0 = P.part + ((int64_t)b * P.ncta * P.H_q + h) * (kD + 2);
            // the gate logit and the linear branch's output load with the partials
            const float x = __bfloat162float(P.gate[(int64_t)b * P.H_q + h]);
            const float o_lin = __ldcg(P.olin + ((int64_t)b * P.H_q + h) * kD + c);
            float Mx = -INFINITY, Lsum = 0.0f, O = 0.0f;
#pragma unroll 1
            for (int i0 = 0; i0 < P.ncta; i0 += kChunk) {
                float mm[kChunk], ll[kChunk], oo[kChunk];
#pragma unroll
                for (int u = 0; u < kChunk; ++u) {
                    mm[u] = -INFINITY;
                    ll[u] = 0.0f;
                    oo[u] = 0.0f;
                    if (i0 + u < P.ncta) {
                        const float* rec = rec0 + (i0 + u) * jstride;
                        mm[u] = __ldcg(rec);
                        ll[u] = __ldcg(rec + 1);
                        oo[u] = __ldcg(rec + 2 + c);
                    }
                }
                float cm = Mx;
#pragma unroll
                for (int u = 0; u < kChunk; ++u) cm = fmaxf(cm, mm[u]);
                if (cm == -INFINITY) continue;
                const float a = exp2f(Mx - cm);  // Mx = -inf gives 0
                Lsum *= a;
                O *= a;
#pragma unroll
                for (int u = 0; u < kChunk; ++u) {
                    const float wgt = exp2f(mm[u] - cm);  // an empty partial (-inf) weighs 0
                    Lsum = fmaf(ll[u], wgt, Lsum);
                    O = fmaf(oo[u], wgt, O);
                }
                Mx = cm;
            }
            const float o_sp = Lsum > 0.0f ? O / Lsum : 0.0f;
            const float gt = 1.0f / (1.0f + __expf(-x));
            P.o[((int64_t)b * P.H_q + h) * kD + c] = __float2bfloat16_rn(gt * o_lin + (1.0f - gt) * o_sp);
        }
        if (P.phi == LISA_PHI_ELU1_NORM && tid < kD) {
            // z <- z + phi(k_L): every reader of the old z (the linear-branch warps
            // of this sequence) is past the third exchange
            for (int g = j; g < P.H_kv; g += P.ncta) {
                const int64_t zi = ((int64_t)b * P.H_kv + g) * kD + tid;
                P.z[zi] += feat(P.phi, __bfloat162float(P.k_L[zi]));
            }
        }
    }
    if (tid == 0) {
        // the last CTA to leave zeroes the exchange counters for the next call
        if (atomicAdd(sync + 3, 1u) == (unsigned)P.ncta - 1) {
            volatile unsigned* vs = sync;
            vs[0] = 0u;
            vs[1] = 0u;
            vs[2] = 0u;
            vs[4] = 0u;
            vs[3] = 0u;
        }
    }
}

// ---------------------------------------------------------------- host side
// SM count of the current device (cached per device).
int coop_num_sms() {
    constexpr int kMaxDev = 64;
    static int sms_of[kMaxDev] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    int sms = (dev >= 0 && dev < kMaxDev) ? sms_of[dev] : 0;
    if (sms <= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            sms <= 0)
            sms = 148;
        if (dev >= 0 && dev < kMaxDev) sms_of[dev] = sms;
    }
    return sms;
}

struct CoopPlan {
    int ncta, KPC, nstg, krow, stage_bytes, sel_cap, ns, spos_off, smem;
    size_t olin, part, cand, gsel, end;
    bool fits;
};

CoopPlan coop_plan(const Shape& s, bool window) {
    CoopPlan pl;
    const int sms = coop_num_sms();
    const int n = window ? std::min(s.M, s.L) : s.L;  // positions shared out over the CTAs
    const int per_b = sms / std::max(1, s.B);
    pl.ncta = std::max(1, std::min(per_b, (n + 15) / 16));
    pl.KPC = align_up((n + pl.ncta - 1) / pl.ncta, 16);
    pl.ncta = (n + pl.KPC - 1) / pl.KPC;
    pl.krow = s.H_kv * kD * 2 + 16;
    pl.stage_bytes = 2 * kGK * pl.krow;
    pl.nstg = std::min(kMaxStages, kCandOff / pl.stage_bytes);
    pl.nstg -= pl.nstg % (8 / std::max(1, s.H_kv));  // a multiple of the warps per KV head
    pl.sel_cap = std::min(pl.KPC, s.M);
    pl.ns = align_up(s.L, 32);
    pl.spos_off = kKeysOff + align_up(4 * pl.KPC, 128);
    pl.smem = pl.spos_off + align_up(4 * pl.sel_cap, 128) + 1024;  // + base alignment slack
    size_t off = decode_scratch_offset(s.B);
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    pl.olin = take(sizeof(float) * (size_t)s.B * s.H_q * kD);
    pl.part = take(sizeof(float) * (size_t)s.B * pl.ncta * s.H_q * (kD + 2));
    pl.cand = take(sizeof(uint2) * (size_t)s.B * pl.ns);
    pl.gsel = take(sizeof(int) * (size_t)s.B * pl.ncta);
    pl.end = off;
    pl.fits = per_b >= 1 && s.B * pl.ncta <= sms && pl.KPC <= kMaxKPC && pl.smem <= 227 * 1024 &&
              pl.nstg >= 2;
    return pl;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

size_t coop_decode_ws_bytes(const Shape& s) {
    if (s.B <= 0 || s.L <= 0) return kStatusBytes;
    return std::max(coop_plan(s, false).end, coop_plan(s, true).end);
}

bool coop_decode_supported(const Shape& s, const lisa_decode_args& a, bool window) {
    if (s.dtype != LISA_BF16 || s.T != 1 || s.d != kD) return false;
    if (!window && (s.d_I != kDI || s.H_I > 8 || !(s.H_Ik == 1 || (s.H_Ik == 8 && s.H_I == 8))))
        return false;
    if (s.group > 8 || !(s.H_kv == 1 || s.H_kv == 2 || s.H_kv == 4)) return false;
    if (s.L < 1 || s.M < 1 || s.B < 1) return false;
    if (!coop_plan(s, window).fits) return false;
    const void* ptrs[] = {a.q, a.k_new, a.v_new, a.q_L, a.k_L, a.v_L, a.k_cache, a.v_cache, a.S, a.o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return false;
    if (!window && (!aligned16(a.q_I) || !aligned16(a.k_I_new) || !aligned16(a.k_I_cache)))
        return false;
    if (s.phi == LISA_PHI_ELU1_NORM && !aligned16(a.z)) return false;
    return window || tma_encode_fn() != nullptr;
}

cudaError_t coop_decode_step(const Shape& s, const lisa_decode_args& a, void* ws, cudaStream_t st,
                             bool window) {
    const CoopPlan pl = coop_plan(s, window);
    CoopParams P;
    P.B = s.B; P.n = s.L; P.N_max = s.N_max; P.H_q = s.H_q; P.H_kv = s.H_kv; P.group = s.group;
    P.H_I = s.H_I; P.H_Ik = s.H_Ik; P.M = s.M; P.phi = s.phi;
    P.window = window ? 1 : 0;
    P.ncta = pl.ncta; P.KPC = pl.KPC; P.nstg = pl.nstg;
    P.rowbytes = s.H_kv * kD * 2; P.krow = pl.krow; P.stage_bytes = pl.stage_bytes;
    P.sel_cap = pl.sel_cap; P.ns = pl.ns; P.spos_off = pl.spos_off;
    P.scale_log2 = s.sm_scale * 1.4426950408889634f;
    P.q = (const bf16*)a.q; P.k_new = (const bf16*)a.k_new; P.v_new = (const bf16*)a.v_new;
    P.q_I = (const bf16*)a.q_I; P.k_I_new = (const bf16*)a.k_I_new; P.w = a.w;
    P.q_L = (const bf16*)a.q_L; P.k_L = (const bf16*)a.k_L; P.v_L = (const bf16*)a.v_L;
    P.gate = (const bf16*)a.gate_logit_lin;
    P.k_cache = (bf16*)a.k_cache; P.v_cache = (bf16*)a.v_cache; P.k_I_cache = (bf16*)a.k_I_cache;
    P.S = a.S; P.z = a.z; P.o = (bf16*)a.o; P.idx = a.idx; P.count = a.count;
    char* w8 = (char*)ws;
    P.status = (unsigned*)ws;
    P.ghist = (unsigned*)(w8 + decode_hist_offset());
    P.ghist2 = (unsigned*)(w8 + decode_hist2_offset(s.B));
    P.sync = (unsigned*)(w8 + decode_sync_offset(s.B));
    P.olin = (float*)(w8 + pl.olin);
    P.part = (float*)(w8 + pl.part);
    P.cand = (uint2*)(w8 + pl.cand);
    P.gsel = (int*)(w8 + pl.gsel);

    CUtensorMap tmap_slot, tmap_tail;  // unused by the window step (it scans no keys)
    memset(&tmap_slot, 0, sizeof(tmap_slot));
    memset(&tmap_tail, 0, sizeof(tmap_tail));
    const uint64_t kI_rows = (uint64_t)s.B * s.N_max * s.H_Ik;
    if (!window && (!make_tmap_bf16_rows(&tmap_slot, a.k_I_cache, kDI, kI_rows, kSlotRows) ||
                    !make_tmap_bf16_rows(&tmap_tail, a.k_I_cache, kDI, kI_rows, kBoxRows)))
        return cudaErrorInvalidValue;

    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(k_decode_coop, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident: the exchanges wait on peers
    attr[0].val.cooperative = 1;
    // a programmatic dependent of the previous kernel on the stream: its launch
    // and shared-memory set-up overlap that kernel's end (the kernel waits for
    // it to complete before touching global memory)
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(s.B * pl.ncta);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_decode_coop, tmap_slot, tmap_tail, P);
    if (e == cudaErrorInvalidValue || e == cudaErrorNotSupported) {
        // a driver that takes no programmatic dependency with a cooperative grid
        (void)cudaGetLastError();
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, k_decode_coop, tmap_slot, tmap_tail, P);
    }
    return e;
}

}  // namespace lisa
