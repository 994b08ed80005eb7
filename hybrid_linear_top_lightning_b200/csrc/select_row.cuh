// Exact top-M of one score row by one CTA of kSelThreads threads: the
// selection step of the Lightning Indexer (LISA, arXiv 2607.19358v1, Sec. 3.2:
// the M highest summed scores are kept).  Order (score desc, position asc);
// positions are emitted by rank, i.e. in ascending position order.
//
// Radix select on the 32-bit order-preserving key of each score:
//  1. first digit = key bits [31:20] (4096 bins), from a histogram given by the
//     caller (built while the scores were produced) or computed here;
//  2. one ordered pass over the row: keys whose first digit is above the
//     threshold digit are selected; keys equal to it are candidates, appended
//     to per-warp lists in position order;
//  3. two 10-bit refinements over the candidates only (or over the whole row
//     when a warp's candidate list overflows);
//  4. every warp knows how many of its positions are selected (ties at the
//     threshold key go to the lowest positions); warps whose rank range meets
//     [lo, hi) walk their positions and write out[rank - lo] = position.
#pragma once

#include "lisa_internal.cuh"

namespace lisa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kCandCap = 256;  // candidates per warp kept in shared memory

struct SelectSmem {
    unsigned* hist;   // 4096 u32
    int* bc;          // >= 64 ints: broadcasts and per-warp counts
    uint2* cand;      // kSelWarps * kCandCap (key, position)
};

__device__ __forceinline__ int sel_block_excl_scan(int v, int* scratch, int& total) {
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
    for (int w = 0; w < kSelWarps; ++w) {
        const int x = scratch[w];
        if (w < warp) off += x;
        total += x;
    }
    __syncthreads();
    return off + incl - v;
}

// Finds the bin holding the `need`-th largest key: thread t owns bins
// [t*bpt, (t+1)*bpt) with counts hv[].  Result in bc[0] (bin) and bc[1] (rank
// of the wanted key inside that bin, counted from its top).
__device__ __forceinline__ void sel_find_bin(const unsigned* hv, int bpt, int need, int* bc) {
    const int tid = threadIdx.x;
    int tsum = 0;
    for (int q = 0; q < bpt; ++q) tsum += (int)hv[q];
    int total;
    const int below = sel_block_excl_scan(tsum, bc + 32, total);
    const int above = total - below - tsum;
    if (tid == 0) { bc[0] = 0; bc[1] = 1; }
    __syncthreads();
    if (above < need && need <= above + tsum) {
        int acc = above;
        for (int q = bpt - 1; q >= 0; --q) {
            if (acc + (int)hv[q] >= need) {
                bc[0] = tid * bpt + q;
                bc[1] = need - acc;
                break;
            }
            acc += (int)hv[q];
        }
    }
    __syncthreads();
}

// row: n scores, resident in shared memory (`resident`) or in global memory
// (read through L2); the row buffer holds at least round_up(n, 8) floats.
// M < n.  first_hist: 4096-bin histogram of key >> 20 over the row, or null.
// row_bar: if not null, an mbarrier (phase 0) that completes when a TMA copy
// of the row into shared memory has landed; it is waited on (bounded) after
// the first digit is known, so the copy overlaps the histogram work.
static __device__ void row_topm(const float* row, bool resident, int n, int M, const unsigned* first_hist,
                         const SelectSmem& sm, int lo, int hi, int* out, uint64_t* row_bar,
                         unsigned* status) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto keys8 = [&](int base, uint32_t (&k)[8]) {
        const float4* src = reinterpret_cast<const float4*>(row) + base / 4;
        float4 v0, v1;
        if (resident) { v0 = src[0]; v1 = src[1]; }
        else { v0 = __ldcg(src); v1 = __ldcg(src + 1); }
        k[0] = order_key(v0.x); k[1] = order_key(v0.y); k[2] = order_key(v0.z); k[3] = order_key(v0.w);
        k[4] = order_key(v1.x); k[5] = order_key(v1.y); k[6] = order_key(v1.z); k[7] = order_key(v1.w);
    };
    auto warp_excl = [&](int v, int& tot) {
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        tot = __shfl_sync(0xffffffffu, incl, 31);
        return incl - v;
    };
    int* bc = sm.bc;
    auto wait_row = [&]() {
        if (!row_bar) return;
        bool ok = false;
        for (uint32_t i = 0; i < (1u << 22) && !ok; ++i) {
            uint32_t r;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(r)
                : "r"((uint32_t)__cvta_generic_to_shared(row_bar))
                : "memory");
            ok = r != 0;
        }
        // a copy that never landed leaves the row unread: the selection then
        // works on stale shared memory, and the status word says so
        if (!ok && tid == 0) record_error(status, kDevTimeout);
    };
    // ---- 1. first digit
    uint32_t b1;
    int krem;
    {
        unsigned hv[16];
        if (first_hist) {
            const uint4* g4 = reinterpret_cast<const uint4*>(first_hist) + tid * 4;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 u = __ldcg(g4 + q);
                hv[4 * q] = u.x; hv[4 * q + 1] = u.y; hv[4 * q + 2] = u.z; hv[4 * q + 3] = u.w;
            }
        } else {
            wait_row();
            for (int i = tid; i < 4096; i += kSelThreads) sm.hist[i] = 0u;
            __syncthreads();
            for (int i8 = tid * 8; i8 < n; i8 += kSelThreads * 8) {
                uint32_t k[8];
                keys8(i8, k);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (i8 + e < n) atomicAdd(&sm.hist[k[e] >> 20], 1u);
            }
            __syncthreads();
#pragma unroll
            for (int q = 0; q < 16; ++q) hv[q] = sm.hist[tid * 16 + q];
        }
        sel_find_bin(hv, 16, M, bc);
        b1 = (uint32_t)bc[0];
        krem = bc[1];
    }
    if (first_hist) wait_row();
    // ---- 2. ordered candidate pass.  Warp w owns positions [w*seg, (w+1)*seg),
    // walked in blocks of 256 with lane l on positions blk + 8l .. blk + 8l + 7.
    const int seg = ((n + kSelWarps - 1) / kSelWarps + 255) / 256 * 256;
    const int s0 = warp * seg, s1 = min(n, s0 + seg);
    uint2* clist = sm.cand + warp * kCandCap;
    int n_above = 0, ncand = 0;
#pragma unroll 1
    for (int blk = s0; blk < s1; blk += 256) {
        const int base = blk + lane * 8;
        uint32_t k[8];
        unsigned cm = 0;
        if (base < s1) {
            keys8(base, k);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const bool v = base + e < s1;
                n_above += v && (k[e] >> 20) > b1;
                cm |= (unsigned)(v && (k[e] >> 20) == b1) << e;
            }
        }
        int ctot;
        int w = ncand + warp_excl(__popc(cm), ctot);
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if ((cm >> e) & 1u) {
                if (w < kCandCap) clist[w] = make_uint2(k[e], (uint32_t)(base + e));
                ++w;
            }
        ncand += ctot;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n_above += __shfl_xor_sync(0xffffffffu, n_above, o);
    int* above_w = bc + 8;   // [kSelWarps]
    int* ncand_w = bc + 16;  // [kSelWarps]
    int* gt_w = bc + 24;     // [kSelWarps]
    int* eq_w = bc + 48;     // [kSelWarps]  (bc + 32 .. 39 is the scan scratch)
    if (lane == 0) { above_w[warp] = n_above; ncand_w[warp] = ncand; }
    __syncthreads();
    bool overflow = false;
    for (int w = 0; w < kSelWarps; ++w) overflow |= ncand_w[w] > kCandCap;
    // ---- 3. refinements
    uint32_t prefix = b1 << 20, mask = 0xFFFu << 20;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        for (int i = tid; i < 1024; i += kSelThreads) sm.hist[i] = 0u;
        __syncthreads();
        if (!overflow) {
            for (int i = tid; i < kSelWarps * kCandCap; i += kSelThreads) {
                const int w = i / kCandCap, c = i % kCandCap;
                if (c < ncand_w[w]) {
                    const uint32_t k = sm.cand[i].x;
                    if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & 1023u], 1u);
                }
            }
        } else {
            for (int i8 = tid * 8; i8 < n; i8 += kSelThreads * 8) {
                uint32_t k[8];
                keys8(i8, k);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (i8 + e < n && (k[e] & mask) == prefix)
                        atomicAdd(&sm.hist[(k[e] >> shift) & 1023u], 1u);
            }
        }
        __syncthreads();
        unsigned hv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) hv[q] = sm.hist[tid * 4 + q];
        sel_find_bin(hv, 4, krem, bc);
        prefix |= (uint32_t)bc[0] << shift;
        krem = bc[1];
        mask |= 1023u << shift;
        __syncthreads();
    }
    const uint32_t tau = prefix;  // the M-th largest key; krem of its ties are kept
    // ---- 4. per-warp selected counts, then the ranked walk
    int gt_c = 0, eq_c = 0;
    if (!overflow) {
        for (int c = lane; c < ncand_w[warp]; c += 32) {
            const uint32_t k = clist[c].x;
            gt_c += k > tau;
            eq_c += k == tau;
        }
    } else {
        for (int blk = s0; blk < s1; blk += 256) {
            const int base = blk + lane * 8;
            if (base >= s1) continue;
            uint32_t k[8];
            keys8(base, k);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if (base + e < s1 && (k[e] >> 20) == b1) { gt_c += k[e] > tau; eq_c += k[e] == tau; }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt_c += __shfl_xor_sync(0xffffffffu, gt_c, o);
        eq_c += __shfl_xor_sync(0xffffffffu, eq_c, o);
    }
    if (lane == 0) { gt_w[warp] = gt_c; eq_w[warp] = eq_c; }
    __syncthreads();
    int eq_before = 0, sel_before = 0;
    for (int w = 0; w < warp; ++w) {
        const int eqw = eq_w[w];
        sel_before += above_w[w] + gt_w[w] + max(0, min(eqw, krem - eq_before));
        eq_before += eqw;
    }
    const int sel_mine = n_above + gt_c + max(0, min(eq_c, krem - eq_before));
    if (sel_before < hi && sel_before + sel_mine > lo) {
#pragma unroll 1
        for (int blk = s0; blk < s1; blk += 256) {
            const int base = blk + lane * 8;
            uint32_t k[8];
            unsigned eqm = 0, selm = 0;
            if (base < s1) {
                keys8(base, k);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const bool v = base + e < s1;
                    const bool above = v && (k[e] >> 20) > b1;
                    const bool cand = v && (k[e] >> 20) == b1;
                    eqm |= (unsigned)(cand && k[e] == tau) << e;
                    selm |= (unsigned)(above || (cand && k[e] > tau)) << e;
                }
            }
            int eq_tot;
            int er = eq_before + warp_excl(__popc(eqm), eq_tot);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if ((eqm >> e) & 1u) { selm |= (unsigned)(er < krem) << e; ++er; }
            int sel_tot;
            int rank = sel_before + warp_excl(__popc(selm), sel_tot);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                if ((selm >> e) & 1u) {
                    if (rank >= lo && rank < hi) out[rank - lo] = base + e;
                    ++rank;
                }
            eq_before += eq_tot;
            sel_before += sel_tot;
            if (sel_before >= hi) break;  // warp-uniform
        }
    }
    __syncthreads();
}

}  // namespace lisa
