// Exact top-M of one score row by one CTA of kSelThreads threads: the
// selection step of the Lightning Indexer (LISA, arXiv 2607.19358v1, Sec. 3.2:
// the M highest summed scores are kept).  Order (score desc, position asc);
// positions are emitted by rank, i.e. in ascending position order.
//
// Radix select on the 32-bit order-preserving key of each score, with every
// thread working on its own contiguous chunk of 64 positions per round of
// kSelThreads * 64 positions (no warp walks a range serially):
//  1. first digit = key bits [31:20] (4096 bins), from a histogram given by the
//     caller (built while the scores were produced) or computed here;
//  2. the keys whose first digit equals the threshold digit are the
//     candidates: counted per thread, then written in position order at
//     block-scanned offsets;
//  3. two 10-bit refinements over the candidates (or over the whole row when
//     there are more than the candidate buffer holds) give the exact M-th
//     largest key tau and how many keys equal to tau are kept;
//  4. per thread, bit masks of its keys above tau and equal to tau; a block
//     scan of the tie counts gives each tie its rank in position order (ties
//     go to the lowest positions), a block scan of the selected counts gives
//     each selected position its rank; positions whose rank falls in
//     [lo, hi) are written to out[rank - lo].
#pragma once

#include "lisa_internal.cuh"

namespace lisa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kCandCap = 256;                         // candidate slots per warp
constexpr int kCandTotal = kSelWarps * kCandCap;      // candidate buffer (entries)
constexpr int kSelChunk = 64;                         // positions per thread per round
constexpr int kSelRound = kSelThreads * kSelChunk;    // positions per round

struct SelectSmem {
    unsigned* hist;   // 4096 u32
    int* bc;          // >= 64 ints: broadcasts and scan scratch
    uint2* cand;      // kCandTotal (key, position)
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

// Keeps the `keep` lowest set bits of m.
__device__ __forceinline__ uint64_t sel_lowest_bits(uint64_t m, int keep) {
    uint64_t r = 0;
    for (int i = 0; i < keep && m; ++i) {
        const uint64_t b = m & (~m + 1);
        r |= b;
        m ^= b;
    }
    return r;
}

// row: n scores, resident in shared memory (`resident`) or in global memory;
// the row buffer holds at least round_up(n, 4) floats.  M < n.  first_hist:
// 4096-bin histogram of key >> 20 over the row, or null.  row_bar: if not
// null, an mbarrier (phase 0) that completes when a TMA copy of the row into
// shared memory has landed; it is waited on (bounded) before the row is read,
// after the first digit when that comes from first_hist.
static __device__ void row_topm(const float* row, bool resident, int n, int M, const unsigned* first_hist,
                                const SelectSmem& sm, int lo, int hi, int* out, uint64_t* row_bar,
                                unsigned* status) {
    const int tid = threadIdx.x;
    int* bc = sm.bc;
    const int rounds = (n + kSelRound - 1) / kSelRound;
    // float4 j (0..15) of this thread's chunk in round r, visited in a rotated
    // order so that the lanes of a quarter warp hit distinct shared-memory banks
    auto chunk_q = [&](int r, int j) { return (r * kSelRound + tid * kSelChunk) / 4 + ((j + tid) & 15); };
    auto load4 = [&](int q, uint32_t (&k)[4]) {
        const float4* src = reinterpret_cast<const float4*>(row) + q;
        const float4 v = resident ? *src : __ldg(src);
        k[0] = order_key(v.x); k[1] = order_key(v.y); k[2] = order_key(v.z); k[3] = order_key(v.w);
    };
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
            for (int r = 0; r < rounds; ++r)
#pragma unroll 4
                for (int j = 0; j < 16; ++j) {
                    const int q = chunk_q(r, j);
                    if (4 * q >= n) continue;
                    uint32_t k[4];
                    load4(q, k);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * q + e < n) atomicAdd(&sm.hist[k[e] >> 20], 1u);
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

    // ---- 2. candidates (first digit == b1), in position order
    int ncand;
    {
        int mine = 0;
        for (int r = 0; r < rounds; ++r)
#pragma unroll 4
            for (int j = 0; j < 16; ++j) {
                const int q = chunk_q(r, j);
                if (4 * q >= n) continue;
                uint32_t k[4];
                load4(q, k);
#pragma unroll
                for (int e = 0; e < 4; ++e) mine += (4 * q + e < n) && (k[e] >> 20) == b1;
            }
        int off = sel_block_excl_scan(mine, bc + 32, ncand);
        if (ncand <= kCandTotal && mine > 0) {
            for (int r = 0; r < rounds; ++r)
                for (int j = 0; j < 16; ++j) {
                    const int q = (r * kSelRound + tid * kSelChunk) / 4 + j;  // position order
                    if (4 * q >= n) continue;
                    uint32_t k[4];
                    load4(q, k);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if ((4 * q + e < n) && (k[e] >> 20) == b1)
                            sm.cand[off++] = make_uint2(k[e], (uint32_t)(4 * q + e));
                }
        }
        __syncthreads();
    }
    const bool overflow = ncand > kCandTotal;

    // ---- 3. refinements
    uint32_t prefix = b1 << 20, mask = 0xFFFu << 20;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        for (int i = tid; i < 1024; i += kSelThreads) sm.hist[i] = 0u;
        __syncthreads();
        if (!overflow) {
            for (int i = tid; i < ncand; i += kSelThreads) {
                const uint32_t k = sm.cand[i].x;
                if ((k & mask) == prefix) atomicAdd(&sm.hist[(k >> shift) & 1023u], 1u);
            }
        } else {
            for (int r = 0; r < rounds; ++r)
                for (int j = 0; j < 16; ++j) {
                    const int q = chunk_q(r, j);
                    if (4 * q >= n) continue;
                    uint32_t k[4];
                    load4(q, k);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * q + e < n && (k[e] & mask) == prefix)
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
    }
    const uint32_t tau = prefix;  // the M-th largest key; krem of its ties are kept

    // ---- 4. ranks in position order, round by round
    int rank_base = 0, tie_base = 0;
#pragma unroll 1
    for (int r = 0; r < rounds && rank_base < hi; ++r) {
        uint64_t gtm = 0, eqm = 0;
#pragma unroll 4
        for (int j = 0; j < 16; ++j) {
            const int q = chunk_q(r, j);
            if (4 * q >= n) continue;
            uint32_t k[4];
            load4(q, k);
            const int bit = ((j + tid) & 15) * 4;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool v = 4 * q + e < n;
                gtm |= (uint64_t)(v && k[e] > tau) << (bit + e);
                eqm |= (uint64_t)(v && k[e] == tau) << (bit + e);
            }
        }
        const int eq_t = __popcll(eqm);
        int eq_tot;
        const int tie_before = tie_base + sel_block_excl_scan(eq_t, bc + 32, eq_tot);
        tie_base += eq_tot;
        const int keep = max(0, min(eq_t, krem - tie_before));
        const uint64_t selm = gtm | sel_lowest_bits(eqm, keep);
        const int sel_t = __popcll(selm);
        int sel_tot;
        int rank = rank_base + sel_block_excl_scan(sel_t, bc + 32, sel_tot);
        rank_base += sel_tot;
        if (rank < hi && rank + sel_t > lo) {
            const int pos0 = r * kSelRound + tid * kSelChunk;
            uint64_t m = selm;
            while (m) {
                const int b = __ffsll((long long)m) - 1;
                m &= m - 1;
                if (rank >= lo && rank < hi) out[rank - lo] = pos0 + b;
                ++rank;
            }
        }
    }
    __syncthreads();
}

}  // namespace lisa
