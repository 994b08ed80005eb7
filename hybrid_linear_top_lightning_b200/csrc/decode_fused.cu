// Fused LISA decode step for B200 (sm_100a): one kernel launch per step.
//
// One thread-block cluster of C CTAs serves one sequence.  CTA r of the
// cluster owns the key slice [r*KPC, (r+1)*KPC) of the context and the slice
// of linear-state columns that its (KV head, column block) names.  The step
// (LISA, arXiv 2607.19358v1: Sec. 3.2 generation step and Eq. 1; Sec. 3.1 and
// Sec. 3.3 Eq. 3-4 for the linear branch):
//
//  A  indexer scan: the CTA's k_I rows stream in by TMA (128-row boxes,
//     128-byte swizzle, a ring of stages); each warp scores 16 keys at a time
//     on the tensor cores (mma m16n8k16: keys x indexer heads, K = d_I = 64),
//     then ReLU, head weights and the head sum give the score, kept in shared
//     memory.  The new token's row comes from k_I_new.  Meanwhile the CTA's
//     linear-state slice arrives by cp.async.
//  A' linear branch: S[:, cols] += phi(k)^T v[cols]; o_lin = phi(q) S[:, cols]
//     (divided by phi(q).z in elu+1 mode) for the query heads of the group.
//  B  top-M: an exact radix select over the cluster (11/11/10-bit passes on the
//     order-preserving integer key of each score).  Each CTA histograms its own
//     keys and adds the non-zero bins into the bin owner's shared memory
//     (distributed shared memory); after a cluster barrier every CTA reads the
//     whole histogram and finds the same digit.  Ties at the threshold keep the
//     lowest positions.  The selected positions are then spread evenly over
//     the CTAs (each CTA writes its picks straight into the owner's list).
//  C  sparse attention: each CTA gathers its share of the selected K and V rows
//     (all KV heads of a position are one contiguous row) with 1D bulk copies
//     into padded shared-memory rows, and runs an online softmax on the tensor
//     cores: query heads of a group on the M side (16 rows), keys on N.
//  D  combine: per-CTA partial (max, sum, output) triples are merged across the
//     cluster through distributed shared memory; the gate mixes the linear and
//     sparse outputs and writes o.
//
// Every wait on an mbarrier is bounded; a wait that gives up records
// LISA_ERR_TIMEOUT in the status word, skips the dependent work and still
// takes part in every cluster barrier, so no CTA is left waiting.  There are no
// inter-cluster dependencies and no spin loops on global memory.
#include <cuda.h>
#include <math.h>

#include "lisa_fast.cuh"
#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kD = 128;             // head dimension of this path
constexpr int kDI = 64;             // indexer dimension of this path
constexpr int kScanRows = 128;      // keys per TMA box (16 per warp)
constexpr int kScanStages = 4;      // TMA ring depth (64 KB in flight)
constexpr int kScanBoxBytes = kScanRows * kDI * 2;
constexpr int kGKeys = 32;          // keys per gather stage
constexpr int kGStages = 2;
constexpr int kMaxKPC = 8192;       // keys per CTA (scores kept in shared memory)
constexpr int kMaxPer = 512;        // selected positions per CTA after balancing
constexpr int kMaxBins = 2048;
constexpr uint32_t kWaitTries = 1u << 22;  // bounded mbarrier polls

struct Params {
    int B, n, N_max, H_q, H_kv, group, H_I, M, phi;
    int KPC;           // keys per CTA (multiple of 16)
    int ncols;         // linear-state columns per CTA
    int rowbytes;      // bytes of one cached K (or V) row: H_kv * d * 2
    float scale_log2;  // sm_scale * log2(e)
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
};

// Shared-memory plan (offsets in bytes from a 1024-byte aligned base).
struct Smem {
    int region_a;   // TMA ring for the scan, then the K/V gather stages, then partials
    int scores;     // float[KPC]
    int hist;       // u32[kMaxBins]    local histogram
    int bins;       // u32[3][kMaxBins / C]  bin slices this CTA owns, one per pass
    int s_slice;    // float[128][ncols]
    int fk;         // float[128]       phi(k_L) of the group's KV head
    int fq;         // float[16][128]   phi(q_L) of the group's query heads
    int vcol;       // float[ncols]
    int zloc;       // float[128]
    int olin;       // float[16][ncols]
    int den;        // float[16]
    int mypos;      // int[kMaxPer]
    int xchg;       // int[4]   n_gt, n_eq published to the cluster
    int misc;       // int[64]  broadcasts and per-CTA tables
    int ctab;       // int[2 * 16 + 16 + 16]
    int bars;       // uint64[kScanStages + kGStages]
    int total;
};

__host__ __device__ inline int align_up(int x, int a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Smem smem_plan(int C, int KPC, int ncols, int rowbytes, int H_kv) {
    Smem s;
    const int scan_bytes = kScanStages * kScanBoxBytes;
    const int krow = rowbytes + 16;
    const int gather_bytes = kGStages * kGKeys * 2 * krow;
    const int part_bytes = H_kv * 16 * (kD + 2) * 4;
    int a = scan_bytes;
    if (gather_bytes > a) a = gather_bytes;
    if (part_bytes > a) a = part_bytes;
    int off = 0;
    s.region_a = off; off += align_up(a, 1024);
    s.scores = off;   off += align_up(KPC * 4, 16);
    s.hist = off;     off += kMaxBins * 4;
    s.bins = off;     off += 3 * (kMaxBins / C) * 4;
    s.s_slice = off;  off += align_up(kD * ncols * 4, 16);
    s.fk = off;       off += kD * 4;
    s.fq = off;       off += 16 * kD * 4;
    s.vcol = off;     off += align_up(ncols * 4, 16);
    s.zloc = off;     off += kD * 4;
    s.olin = off;     off += align_up(16 * ncols * 4, 16);
    s.den = off;      off += 16 * 4;
    s.mypos = off;    off += kMaxPer * 4;
    s.xchg = off;     off += 16;
    s.misc = off;     off += 64 * 4;
    s.ctab = off;     off += 64 * 4;
    s.bars = off;     off += (kScanStages + kGStages) * 8;
    s.total = align_up(off, 16) + 1024;  // slack for aligning the base
    return s;
}

__device__ __forceinline__ float feat(int phi, float x) {
    if (phi == LISA_PHI_IDENTITY) return x;
    return x > 0.0f ? x + 1.0f : __expf(x);
}

// Exclusive scan over the 256 threads of the block.
__device__ __forceinline__ int block_scan_excl(int v, int* scratch, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    int off = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const int x = scratch[w];
        if (w < warp) off += x;
        total += x;
    }
    __syncthreads();
    return off + incl - v;
}

template <int C>
__global__ void __launch_bounds__(kThreads, 1)
    k_decode_fused(const __grid_constant__ CUtensorMap tmap_kI, const Params P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Smem L = smem_plan(C, P.KPC, P.ncols, P.rowbytes, P.H_kv);
    uint8_t* region_a = base + L.region_a;
    float* scores = reinterpret_cast<float*>(base + L.scores);
    uint32_t* hist = reinterpret_cast<uint32_t*>(base + L.hist);
    uint32_t* bins = reinterpret_cast<uint32_t*>(base + L.bins);
    float* s_slice = reinterpret_cast<float*>(base + L.s_slice);
    float* fk = reinterpret_cast<float*>(base + L.fk);
    float* fq = reinterpret_cast<float*>(base + L.fq);
    float* vcol = reinterpret_cast<float*>(base + L.vcol);
    float* zloc = reinterpret_cast<float*>(base + L.zloc);
    float* olin = reinterpret_cast<float*>(base + L.olin);
    float* den = reinterpret_cast<float*>(base + L.den);
    int* mypos = reinterpret_cast<int*>(base + L.mypos);
    int* xchg = reinterpret_cast<int*>(base + L.xchg);
    int* misc = reinterpret_cast<int*>(base + L.misc);
    int* ctab = reinterpret_cast<int*>(base + L.ctab);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + L.bars);
    uint64_t* scan_bar = bars;
    uint64_t* gath_bar = bars + kScanStages;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const int r = (int)ptx::cluster_ctarank();
    const int b = blockIdx.x / C;
    const int n = P.n, p = n - 1;
    const int k0 = r * P.KPC;
    const int k1 = min(n, k0 + P.KPC);
    const int nk = max(0, k1 - k0);
    const int n_scan_stages = (nk + kScanRows - 1) / kScanRows;
    const int per_owner = kMaxBins / C;
    bool ok = true;  // false once a bounded wait gave up

    // ---------------------------------------------------------------- set-up
    if (tid == 0) {
        for (int i = 0; i < kScanStages + kGStages; ++i) ptx::mbar_init(&bars[i], 1);
        ptx::fence_mbar_init();
    }
    for (int i = tid; i < 3 * per_owner; i += kThreads) bins[i] = 0;
    __syncthreads();
    // First cluster barrier: every CTA's bins are zero and its shared memory is
    // live before anyone touches it remotely.  Waited on before the first
    // remote access, so the scan overlaps it.
    ptx::cluster_arrive();

    if (tid == 0) {
        const int first = min(n_scan_stages, kScanStages);
        for (int st = 0; st < first; ++st) {
            ptx::mbar_arrive_expect_tx(&scan_bar[st], kScanBoxBytes);
            ptx::tma_load_2d(region_a + st * kScanBoxBytes, &tmap_kI, 0,
                             b * P.N_max + k0 + st * kScanRows, &scan_bar[st]);
        }
    }
    // Linear-state slice of this CTA: KV head g_r, columns [c0, c0 + ncols).
    const int cta_per_head = C / P.H_kv;
    const int g_r = r / cta_per_head;
    const int c0 = (r % cta_per_head) * P.ncols;
    float* Sg = P.S + ((int64_t)b * P.H_kv + g_r) * kD * kD;
    {
        const int chunks_per_row = P.ncols / 4;
        for (int e = tid; e < kD * chunks_per_row; e += kThreads) {
            const int i = e / chunks_per_row, c = (e % chunks_per_row) * 4;
            ptx::cp_async_16(s_slice + i * P.ncols + c, Sg + (int64_t)i * kD + c0 + c);
        }
        ptx::cp_async_commit();
    }
    // Cache append of the new token (nobody in this launch reads row p of the
    // caches: the scan and the gather take it from the inputs).
    if (r == 0) {
        const int kv_chunks = P.rowbytes / 16;
        const uint4* kn = reinterpret_cast<const uint4*>(P.k_new + (int64_t)b * P.H_kv * kD);
        const uint4* vn = reinterpret_cast<const uint4*>(P.v_new + (int64_t)b * P.H_kv * kD);
        uint4* kd = reinterpret_cast<uint4*>(P.k_cache + ((int64_t)b * P.N_max + p) * P.H_kv * kD);
        uint4* vd = reinterpret_cast<uint4*>(P.v_cache + ((int64_t)b * P.N_max + p) * P.H_kv * kD);
        for (int i = tid; i < kv_chunks; i += kThreads) {
            kd[i] = kn[i];
            vd[i] = vn[i];
        }
        if (tid < kDI / 8) {
            const uint4* kin = reinterpret_cast<const uint4*>(P.k_I_new + (int64_t)b * kDI);
            uint4* kid = reinterpret_cast<uint4*>(P.k_I_cache + ((int64_t)b * P.N_max + p) * kDI);
            kid[tid] = kin[tid];
        }
    }

    // ---------------------------------------------------------------- A: indexer scan
    // Fragment layout (mma m16n8k16, A = 16 keys x 16 dims, B = 16 dims x 8 heads):
    // the thread (gid, tq) holds dims [16 tq, 16 tq + 16) of its rows; k-step s
    // uses dims 16 tq + 4 s + {0,1} and {2,3}.  A and B use the same dim order,
    // so the dot products are unchanged.
    uint32_t qb[8];
    float w_lo = 0.0f, w_hi = 0.0f;
    {
        if (gid < P.H_I) {
            const uint4* src = reinterpret_cast<const uint4*>(
                P.q_I + ((int64_t)b * P.H_I + gid) * kDI + 16 * tq);
            const uint4 u0 = src[0], u1 = src[1];
            qb[0] = u0.x; qb[1] = u0.y; qb[2] = u0.z; qb[3] = u0.w;
            qb[4] = u1.x; qb[5] = u1.y; qb[6] = u1.z; qb[7] = u1.w;
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) qb[i] = 0u;
        }
        const float* wb = P.w + (int64_t)b * P.H_I;
        if (2 * tq < P.H_I) w_lo = wb[2 * tq];
        if (2 * tq + 1 < P.H_I) w_hi = wb[2 * tq + 1];
    }
    for (int st = 0; st < n_scan_stages; ++st) {
        const int buf = st % kScanStages;
        const uint32_t parity = (st / kScanStages) & 1;
        if (ok && !ptx::mbar_wait_bounded(&scan_bar[buf], parity, kWaitTries)) {
            ok = false;
            if (tid == 0) record_error(P.status, kDevTimeout);
        }
        if (ok) {
            const uint8_t* tile = region_a + buf * kScanBoxBytes;
            const int row0 = warp * 16 + gid;
            uint32_t ra[2][8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = row0 + 8 * h;
                const int pos = k0 + st * kScanRows + row;
                if (pos == p) {
                    const uint4* src = reinterpret_cast<const uint4*>(
                        P.k_I_new + (int64_t)b * kDI + 16 * tq);
                    const uint4 u0 = src[0], u1 = src[1];
                    ra[h][0] = u0.x; ra[h][1] = u0.y; ra[h][2] = u0.z; ra[h][3] = u0.w;
                    ra[h][4] = u1.x; ra[h][5] = u1.y; ra[h][6] = u1.z; ra[h][7] = u1.w;
                } else {
                    const uint8_t* rp = tile + row * 128;
                    const int sw = row & 7;
                    const uint4 u0 = *reinterpret_cast<const uint4*>(rp + (((2 * tq) ^ sw) << 4));
                    const uint4 u1 = *reinterpret_cast<const uint4*>(rp + (((2 * tq + 1) ^ sw) << 4));
                    ra[h][0] = u0.x; ra[h][1] = u0.y; ra[h][2] = u0.z; ra[h][3] = u0.w;
                    ra[h][4] = u1.x; ra[h][5] = u1.y; ra[h][6] = u1.z; ra[h][7] = u1.w;
                }
            }
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                const uint32_t a[4] = {ra[0][2 * s], ra[1][2 * s], ra[0][2 * s + 1], ra[1][2 * s + 1]};
                ptx::mma_bf16(acc, a, qb[2 * s], qb[2 * s + 1]);
            }
            float s0 = w_lo * fmaxf(acc[0], 0.0f) + w_hi * fmaxf(acc[1], 0.0f);
            float s1 = w_lo * fmaxf(acc[2], 0.0f) + w_hi * fmaxf(acc[3], 0.0f);
            s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
            s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
            s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
            const int lr0 = st * kScanRows + row0;  // local key index
            if (tq == 0 && lr0 < nk) scores[lr0] = s0;
            if (tq == 1 && lr0 + 8 < nk) scores[lr0 + 8] = s1;
        }
        __syncthreads();  // every warp is done with this buffer
        if (tid == 0 && ok && st + kScanStages < n_scan_stages) {
            ptx::mbar_arrive_expect_tx(&scan_bar[buf], kScanBoxBytes);
            ptx::tma_load_2d(region_a + buf * kScanBoxBytes, &tmap_kI, 0,
                             b * P.N_max + k0 + (st + kScanStages) * kScanRows, &scan_bar[buf]);
        }
    }

    // ---------------------------------------------------------------- A': linear branch
    ptx::cp_async_wait_all();
    {
        const bf16* kl = P.k_L + ((int64_t)b * P.H_kv + g_r) * kD;
        const bf16* vl = P.v_L + ((int64_t)b * P.H_kv + g_r) * kD;
        for (int i = tid; i < kD; i += kThreads) {
            fk[i] = feat(P.phi, __bfloat162float(kl[i]));
        }
        for (int c = tid; c < P.ncols; c += kThreads) vcol[c] = __bfloat162float(vl[c0 + c]);
        for (int e = tid; e < P.group * kD; e += kThreads) {
            const int h = e / kD, i = e % kD;
            fq[h * kD + i] =
                feat(P.phi, __bfloat162float(P.q_L[((int64_t)b * P.H_q + g_r * P.group + h) * kD + i]));
        }
    }
    __syncthreads();
    const bool norm = P.phi == LISA_PHI_ELU1_NORM;
    if (norm) {
        const float* zg = P.z + ((int64_t)b * P.H_kv + g_r) * kD;
        for (int i = tid; i < kD; i += kThreads) zloc[i] = zg[i] + fk[i];
    }
    for (int e = tid; e < kD * P.ncols; e += kThreads) {
        const int i = e / P.ncols, c = e % P.ncols;
        const float nv = fmaf(fk[i], vcol[c], s_slice[e]);
        s_slice[e] = nv;
        Sg[(int64_t)i * kD + c0 + c] = nv;
    }
    __syncthreads();
    if (norm) {
        if (c0 == 0)
            for (int i = tid; i < kD; i += kThreads)
                P.z[((int64_t)b * P.H_kv + g_r) * kD + i] = zloc[i];
        for (int h = warp; h < P.group; h += kWarps) {
            float dz = 0.0f;
            for (int i = lane; i < kD; i += 32) dz = fmaf(fq[h * kD + i], zloc[i], dz);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dz += __shfl_xor_sync(0xffffffffu, dz, o);
            if (lane == 0) den[h] = dz;
        }
        __syncthreads();
    }
    for (int e = tid; e < P.group * P.ncols; e += kThreads) {
        const int h = e / P.ncols, c = e % P.ncols;
        float acc = 0.0f;
        for (int i = 0; i < kD; ++i) acc = fmaf(fq[h * kD + i], s_slice[i * P.ncols + c], acc);
        olin[h * P.ncols + c] = norm ? acc / den[h] : acc;
    }

    // ---------------------------------------------------------------- B: top-M
    ptx::cluster_wait();  // matches the set-up arrive
    const int cnt = min(P.M, n);
    int* scan_scratch = misc;       // [kWarps]
    int* bc = misc + 16;            // broadcasts
    int sel_offset = 0, n_sel = 0;  // this CTA's selected positions and their global offset
    uint32_t tau = 0;
    int krem = 0;
    int my_take_eq = 0;  // keys equal to the threshold this CTA keeps (lowest positions first)
    const bool select_all = n <= P.M;
    if (!select_all) {
        uint32_t prefix = 0, mask = 0;
        krem = P.M;
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const int nb = pass == 2 ? 1024 : 2048;
            const int owner_span = nb / C;
            for (int i = tid; i < nb; i += kThreads) hist[i] = 0;
            __syncthreads();
            for (int i = tid; i < nk; i += kThreads) {
                const uint32_t key = order_key(scores[i]);
                if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
            }
            __syncthreads();
            uint32_t* pass_bins = bins + pass * per_owner;
            for (int i = tid; i < nb; i += kThreads) {
                const uint32_t v = hist[i];
                if (v) {
                    const uint32_t owner = i / owner_span;
                    const uint32_t addr = ptx::mapa(ptx::smem_u32(pass_bins + (i % owner_span)), owner);
                    ptx::red_add_dsmem_u32(addr, v);
                }
            }
            ptx::cluster_sync();
            // Every CTA reads the whole histogram: thread t owns bins [t*bpt, (t+1)*bpt).
            const int bpt = nb / kThreads;  // 8 or 4
            uint32_t hv[8];
            int tsum = 0;
            for (int j = 0; j < bpt; ++j) {
                const int i = tid * bpt + j;
                const uint32_t owner = i / owner_span;
                hv[j] = ptx::ld_dsmem_u32(ptx::mapa(ptx::smem_u32(pass_bins + (i % owner_span)), owner));
                tsum += (int)hv[j];
            }
            // suffix sum over threads (bins above this thread's range)
            int total;
            const int below = block_scan_excl(tsum, scan_scratch, total);
            const int above = total - below - tsum;
            if (above < krem && krem <= above + tsum) {
                int acc = above;
                for (int j = bpt - 1; j >= 0; --j) {
                    if (acc + (int)hv[j] >= krem) {
                        bc[0] = tid * bpt + j;
                        bc[1] = krem - acc;
                        break;
                    }
                    acc += (int)hv[j];
                }
            }
            __syncthreads();
            prefix |= (uint32_t)bc[0] << shift;
            krem = bc[1];
            mask |= (uint32_t)(nb - 1) << shift;
            __syncthreads();
        }
        tau = prefix;
        // local counts above and equal to the threshold
        if (tid == 0) { bc[2] = 0; bc[3] = 0; }
        __syncthreads();
        int gt = 0, eq = 0;
        for (int i = tid; i < nk; i += kThreads) {
            const uint32_t key = order_key(scores[i]);
            gt += key > tau;
            eq += key == tau;
        }
        if (gt) atomicAdd(&bc[2], gt);
        if (eq) atomicAdd(&bc[3], eq);
        __syncthreads();
        if (tid == 0) { xchg[0] = bc[2]; xchg[1] = bc[3]; }
        ptx::cluster_sync();
        if (tid < C) {
            ctab[tid] = (int)ptx::ld_dsmem_u32(ptx::mapa(ptx::smem_u32(xchg), tid));
            ctab[16 + tid] = (int)ptx::ld_dsmem_u32(ptx::mapa(ptx::smem_u32(xchg + 1), tid));
        }
        __syncthreads();
        // ties: the lowest positions win, so CTAs take their equal keys in rank order
        int eq_before = 0, off = 0;
        for (int c = 0; c < C; ++c) {
            const int take = max(0, min(ctab[16 + c], krem - eq_before));
            const int sel = ctab[c] + take;
            if (c == r) { sel_offset = off; n_sel = sel; my_take_eq = take; }
            eq_before += ctab[16 + c];
            off += sel;
        }
    } else {
        sel_offset = k0;
        n_sel = nk;
    }

    // Ordered compaction of this CTA's selected keys into the owners' lists.
    const int per = (cnt + C - 1) / C;
    {
        const int kpt = (nk + kThreads - 1) / kThreads;
        const int i0 = tid * kpt, i1 = min(nk, i0 + kpt);
        const int take_eq = my_take_eq;
        int eq_rank0 = 0;
        // rank of this thread's first equal key among the CTA's equal keys
        int my_eq = 0;
        if (!select_all)
            for (int i = i0; i < i1; ++i) my_eq += order_key(scores[i]) == tau;
        int tot_eq;
        eq_rank0 = block_scan_excl(my_eq, scan_scratch, tot_eq);
        int my_sel = 0;
        {
            int er = eq_rank0;
            for (int i = i0; i < i1; ++i) {
                if (select_all) { ++my_sel; continue; }
                const uint32_t key = order_key(scores[i]);
                if (key > tau) ++my_sel;
                else if (key == tau) { if (er < take_eq) ++my_sel; ++er; }
            }
        }
        int tot_sel;
        int rank = block_scan_excl(my_sel, scan_scratch, tot_sel);
        int er = eq_rank0;
        for (int i = i0; i < i1; ++i) {
            bool sel;
            if (select_all) {
                sel = true;
            } else {
                const uint32_t key = order_key(scores[i]);
                sel = key > tau;
                if (key == tau) { sel = er < take_eq; ++er; }
            }
            if (!sel) continue;
            const int gi = sel_offset + rank++;
            const int pos = k0 + i;
            const int dest = gi / per, slot = gi - dest * per;
            ptx::st_dsmem_u32(ptx::mapa(ptx::smem_u32(mypos + slot), dest), (uint32_t)pos);
            if (P.idx) P.idx[(int64_t)b * P.M + gi] = pos;
        }
        (void)n_sel;
        if (P.idx && r == 0)
            for (int i = cnt + tid; i < P.M; i += kThreads) P.idx[(int64_t)b * P.M + i] = -1;
        if (P.count && r == 0 && tid == 0) P.count[b] = cnt;
    }
    ptx::cluster_sync();  // every CTA's list is complete

    // ---------------------------------------------------------------- C: gather + attention
    const int my_cnt = max(0, min(cnt - r * per, per));
    const int wph = kWarps / P.H_kv;  // warps per KV head
    const int g_w = warp / wph;
    const int part = warp % wph;
    const int dw = kD / wph;          // output dims of this warp
    const int krow = P.rowbytes + 16;
    const int stage_bytes = kGKeys * 2 * krow;
    // query fragments of head group g_w: rows = query heads (group <= 16), 8 k-steps
    uint32_t qa[8][4];
    {
        const int h0 = g_w * P.group;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = gid + 8 * hh;
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    uint32_t v = 0u;
                    if (row < P.group)
                        v = *reinterpret_cast<const uint32_t*>(
                            P.q + ((int64_t)b * P.H_q + h0 + row) * kD + ks * 16 + 2 * tq + 8 * kk);
                    qa[ks][hh + 2 * kk] = v;
                }
            }
        }
    }
    const int n_gst = (my_cnt + kGKeys - 1) / kGKeys;
    auto issue_stage = [&](int st) {
        // warp 0: lane j copies the K and V rows of the stage's key j
        if (warp == 0) {
            const int buf = st % kGStages;
            uint8_t* kb = region_a + buf * stage_bytes;
            uint8_t* vb = kb + kGKeys * krow;
            if (lane == 0) ptx::mbar_arrive_expect_tx(&gath_bar[buf], kGKeys * 2 * P.rowbytes);
            __syncwarp();
            int j = st * kGKeys + lane;
            if (j >= my_cnt) j = st * kGKeys;  // pad with a valid row; masked below
            const int pos = mypos[j];
            const bf16* ks;
            const bf16* vs;
            if (pos == p) {
                ks = P.k_new + (int64_t)b * P.H_kv * kD;
                vs = P.v_new + (int64_t)b * P.H_kv * kD;
            } else {
                ks = P.k_cache + ((int64_t)b * P.N_max + pos) * P.H_kv * kD;
                vs = P.v_cache + ((int64_t)b * P.N_max + pos) * P.H_kv * kD;
            }
            ptx::bulk_load(kb + lane * krow, ks, P.rowbytes, &gath_bar[buf]);
            ptx::bulk_load(vb + lane * krow, vs, P.rowbytes, &gath_bar[buf]);
        }
    };
    if (ok)
        for (int st = 0; st < min(n_gst, kGStages); ++st) issue_stage(st);

    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.0f, 0.0f};
    float oacc[8][4];  // up to 8 n-tiles of 8 dims (dw <= 64)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[j][e] = 0.0f;
    const int ntile_o = dw / 8;

    for (int st = 0; st < n_gst; ++st) {
        const int buf = st % kGStages;
        const uint32_t parity = (st / kGStages) & 1;
        if (ok && !ptx::mbar_wait_bounded(&gath_bar[buf], parity, kWaitTries)) {
            ok = false;
            if (tid == 0) record_error(P.status, kDevTimeout);
        }
        if (ok) {
            const uint32_t kb = ptx::smem_u32(region_a + buf * stage_bytes);
            const uint32_t vb = kb + kGKeys * krow;
            const uint32_t head_off = (uint32_t)(g_w * kD * 2);
            // S = Q K^T for 32 keys: 4 n-tiles of 8 keys
            float sc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sc[nt][e] = 0.0f;
#pragma unroll
                for (int ks = 0; ks < 8; ks += 2) {
                    uint32_t kr[4];
                    const int key = nt * 8 + (lane & 7);
                    const int dim0 = ks * 16 + (lane >> 3) * 8;
                    ptx::ldmatrix_x4(kr, kb + key * krow + head_off + dim0 * 2);
                    ptx::mma_bf16(sc[nt], qa[ks], kr[0], kr[1]);
                    ptx::mma_bf16(sc[nt], qa[ks + 1], kr[2], kr[3]);
                }
            }
            // scale, mask, online softmax (rows gid and gid + 8)
            float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = st * kGKeys + nt * 8 + 2 * tq + (e & 1);
                    float v = sc[nt][e] * P.scale_log2;
                    if (key >= my_cnt) v = -INFINITY;
                    sc[nt][e] = v;
                    mt[e >> 1] = fmaxf(mt[e >> 1], v);
                }
            }
            float corr[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], 1));
                mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], 2));
                const float m_new = fmaxf(m_run[h], mt[h]);
                corr[h] = (m_new == -INFINITY) ? 1.0f : exp2f(m_run[h] - m_new);
                m_run[h] = m_new;
                l_run[h] *= corr[h];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                oacc[j][0] *= corr[0]; oacc[j][1] *= corr[0];
                oacc[j][2] *= corr[1]; oacc[j][3] *= corr[1];
            }
            uint32_t pa[2][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                float pv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float m = m_run[e >> 1];
                    pv[e] = (m == -INFINITY) ? 0.0f : exp2f(sc[nt][e] - m);
                    l_run[e >> 1] += pv[e];
                }
                // A fragment of P for k-step nt/2: n-tile 2k -> regs 0,1; 2k+1 -> regs 2,3
                const int kk = nt >> 1, hi = nt & 1;
                pa[kk][0 + 2 * hi] = ptx::pack_bf16(pv[0], pv[1]);
                pa[kk][1 + 2 * hi] = ptx::pack_bf16(pv[2], pv[3]);
            }
            // O += P V over this warp's dims
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    if (j < ntile_o) {
                        uint32_t vr[4];
                        const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                        const int dim0 = part * dw + (j + (lane >> 4)) * 8;
                        ptx::ldmatrix_x4_trans(vr, vb + key * krow + head_off + dim0 * 2);
                        ptx::mma_bf16(oacc[j], pa[kk], vr[0], vr[1]);
                        ptx::mma_bf16(oacc[j + 1], pa[kk], vr[2], vr[3]);
                    }
                }
            }
        }
        __syncthreads();  // buffer free
        if (ok && st + kGStages < n_gst) issue_stage(st + kGStages);
    }
    // reduce the row sums across the quad
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
    }
    // partials into region A: m, l per (g, row); O per (g, row, dim)
    __syncthreads();
    float* part_m = reinterpret_cast<float*>(region_a);
    float* part_l = part_m + P.H_kv * 16;
    float* part_o = part_l + P.H_kv * 16;
    {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = gid + 8 * h;
            if (part == 0 && tq == 0) {
                part_m[g_w * 16 + row] = m_run[h];
                part_l[g_w * 16 + row] = l_run[h];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (j < ntile_o) {
                    const int dim = part * dw + j * 8 + 2 * tq;
                    float* dst = part_o + (g_w * 16 + row) * kD + dim;
                    dst[0] = oacc[j][2 * h];
                    dst[1] = oacc[j][2 * h + 1];
                }
            }
        }
    }
    ptx::cluster_sync();  // partials visible cluster-wide

    // ---------------------------------------------------------------- D: combine + gate
    for (int e = tid; e < P.group * P.ncols; e += kThreads) {
        const int h = e / P.ncols, c = e % P.ncols;
        const int prow = g_r * 16 + h;
        float mx = -INFINITY;
        float mc[16], lc[16];
        for (int cc = 0; cc < C; ++cc) {
            mc[cc] = ptx::ld_dsmem_f32(ptx::mapa(ptx::smem_u32(part_m + prow), cc));
            lc[cc] = ptx::ld_dsmem_f32(ptx::mapa(ptx::smem_u32(part_l + prow), cc));
            mx = fmaxf(mx, mc[cc]);
        }
        float num = 0.0f, dsum = 0.0f;
        for (int cc = 0; cc < C; ++cc) {
            if (mc[cc] == -INFINITY) continue;
            const float f = exp2f(mc[cc] - mx);
            dsum = fmaf(lc[cc], f, dsum);
            num = fmaf(ptx::ld_dsmem_f32(ptx::mapa(ptx::smem_u32(part_o + prow * kD + c0 + c), cc)),
                       f, num);
        }
        const float o_sp = dsum > 0.0f ? num / dsum : 0.0f;
        const int hq = g_r * P.group + h;
        const float x = __bfloat162float(P.gate[(int64_t)b * P.H_q + hq]);
        const float g = 1.0f / (1.0f + __expf(-x));
        const float out = g * olin[h * P.ncols + c] + (1.0f - g) * o_sp;
        P.o[((int64_t)b * P.H_q + hq) * kD + c0 + c] = __float2bfloat16_rn(out);
    }
    ptx::cluster_sync();  // nobody exits while others still read its shared memory
    if (!ok && tid == 0) {
        // A bounded wait gave up: give the copies still in flight another bounded
        // chance to land before the shared memory they target is released.
        for (int i = 0; i < kScanStages + kGStages; ++i)
            for (uint32_t par = 0; par < 2; ++par) ptx::mbar_wait_bounded(&bars[i], par, 1u << 16);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

int pick_cluster(const Shape& s) {
    // 16 CTAs per sequence when the GPU can hold such clusters and there is
    // not already enough work to fill it with clusters of 8.
    static int can16 = -1;
    if (can16 < 0) {
        can16 = 0;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 16;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(16);
        cfg.blockDim = dim3(kThreads);
        const Smem L = smem_plan(16, kMaxKPC, 64, 1024, 4);
        cfg.dynamicSmemBytes = L.total;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        auto kern = k_decode_fused<16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) == cudaSuccess && nclusters >= 1)
            can16 = 1;
        cudaGetLastError();
    }
    if (!can16) return 8;
    return s.B * 8 >= 2 * 148 ? 8 : 16;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

size_t fast_decode_ws_bytes(const Shape&) { return kStatusBytes; }

bool fast_decode_supported(const Shape& s, const lisa_decode_args& a) {
    if (s.dtype != LISA_BF16 || s.T != 1 || s.d != kD || s.d_I != kDI || s.H_Ik != 1) return false;
    if (s.H_I > 8 || s.group > 16 || !(s.H_kv == 1 || s.H_kv == 2 || s.H_kv == 4)) return false;
    if (s.L < 1 || s.M < 1) return false;
    const int C = pick_cluster(s);
    const int KPC = align_up((s.L + C - 1) / C, 16);
    if (KPC > kMaxKPC) return false;
    const int cnt = s.M < s.L ? s.M : s.L;
    if ((cnt + C - 1) / C > kMaxPer) return false;
    const Smem L = smem_plan(C, KPC, s.H_kv * kD / C, s.H_kv * kD * 2, s.H_kv);
    if (L.total > 227 * 1024) return false;
    const void* ptrs[] = {a.q, a.k_new, a.v_new, a.q_I, a.k_I_new, a.q_L, a.k_L, a.v_L,
                          a.k_cache, a.v_cache, a.k_I_cache, a.S, a.o};
    for (const void* p : ptrs)
        if (!aligned16(p)) return false;
    if (s.phi == LISA_PHI_ELU1_NORM && !aligned16(a.z)) return false;
    if (!encode_fn()) return false;
    return true;
}

template <int C>
cudaError_t launch_decode(const Shape& s, const lisa_decode_args& a, void* ws, cudaStream_t st) {
    Params P;
    P.B = s.B; P.n = s.L; P.N_max = s.N_max; P.H_q = s.H_q; P.H_kv = s.H_kv; P.group = s.group;
    P.H_I = s.H_I; P.M = s.M; P.phi = s.phi;
    P.KPC = align_up((s.L + C - 1) / C, 16);
    P.ncols = s.H_kv * kD / C;
    P.rowbytes = s.H_kv * kD * 2;
    P.scale_log2 = s.sm_scale * 1.4426950408889634f;
    P.q = (const bf16*)a.q; P.k_new = (const bf16*)a.k_new; P.v_new = (const bf16*)a.v_new;
    P.q_I = (const bf16*)a.q_I; P.k_I_new = (const bf16*)a.k_I_new; P.w = a.w;
    P.q_L = (const bf16*)a.q_L; P.k_L = (const bf16*)a.k_L; P.v_L = (const bf16*)a.v_L;
    P.gate = (const bf16*)a.gate_logit_lin;
    P.k_cache = (bf16*)a.k_cache; P.v_cache = (bf16*)a.v_cache; P.k_I_cache = (bf16*)a.k_I_cache;
    P.S = a.S; P.z = a.z; P.o = (bf16*)a.o; P.idx = a.idx; P.count = a.count;
    P.status = (unsigned*)ws;

    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)kDI, (cuuint64_t)s.B * (cuuint64_t)s.N_max};
    const cuuint64_t gstride[1] = {(cuuint64_t)kDI * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kDI, (cuuint32_t)kScanRows};
    const cuuint32_t estride[2] = {1, 1};
    if (encode_fn()(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.k_I_cache, gdim, gstride, box,
                    estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    const Smem L = smem_plan(C, P.KPC, P.ncols, P.rowbytes, P.H_kv);
    auto kern = k_decode_fused<C>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (e != cudaSuccess) return e;
    if (C > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(s.B * C);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, P);
}

cudaError_t fast_decode_step(const Shape& s, const lisa_decode_args& a, void* ws, cudaStream_t st) {
    const int C = pick_cluster(s);
    if (C == 16) return launch_decode<16>(s, a, ws, st);
    return launch_decode<8>(s, a, ws, st);
}

}  // namespace lisa
