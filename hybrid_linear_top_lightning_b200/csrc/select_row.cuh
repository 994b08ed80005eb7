// Exact top-M of one score row by one CTA of NT threads: the
// selection step of the Lightning Indexer (LISA, arXiv 2607.19358v1, Sec. 3.2:
// the M highest summed scores are kept).  Order (score desc, position asc);
// positions are emitted by rank, i.e. in ascending position order.
//
// Radix select on the 32-bit order-preserving key of each score (the row holds
// the keys, written by the kernel that produced the scores), with every thread
// working on its own contiguous chunk of 16384 / NT positions per round of
// 16384 positions (no warp walks a range serially):
//  1. first digit = key bits [31:20] (4096 bins), from a histogram given by the
//     caller (built while the scores were produced) or computed here;
//  2. the keys whose first digit equals the threshold digit are the
//     candidates: counted per thread, then written at block-scanned offsets;
//  3. two 10-bit refinements over the candidates (or over the whole row when
//     there are more than the candidate buffer holds) give the exact M-th
//     largest key tau and how many keys equal to tau are kept;
//  4. per thread, the count of its keys above tau and equal to tau (in one
//     round: from the first-digit pass and its own candidates); unless every
//     key equal to tau is kept, a block scan of the tie counts gives each tie
//     its rank in position order (ties go to the lowest positions); a block
//     scan of the selected counts gives each thread the rank of its first
//     selected position; threads whose ranks meet [lo, hi) rebuild bit masks
//     of their chunk and write out[rank - lo] = position (in one round through
//     shared memory, so that the index row leaves in coalesced stores).
#pragma once

#include "lisa_internal.cuh"

namespace lisa {

constexpr int kCandTotal = 2048;    // candidate buffer (entries)
constexpr int kSelRound = 16384;    // positions per round

struct SelectSmem {
    unsigned* hist;   // 4096 u32
    int* bc;          // >= 64 ints: broadcasts and scan scratch
    uint2* cand;      // kCandTotal (key, position)
    // the candidate buffer once the ranks are known: the index row is
    // scattered here by rank and leaves in coalesced stores
    __device__ int* stage() const { return reinterpret_cast<int*>(cand); }
    static constexpr int kStageCap = kCandTotal * 2;
};

// Exclusive block scan of v; `total` gets the block sum.  Two barriers: the
// warp sums go through shared memory and every warp scans them by shuffles.
template <int NT>
__device__ __forceinline__ int sel_block_excl_scan(int v, int* scratch, int& total) {
    constexpr int kWarps = NT / 32;
    static_assert(kWarps <= 32, "one warp scans the warp sums");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    const int ws = lane < kWarps ? scratch[lane] : 0;
    int wincl = ws;
#pragma unroll
    for (int o = 1; o < kWarps; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wincl, o);
        if (lane >= o) wincl += y;
    }
    total = __shfl_sync(0xffffffffu, wincl, kWarps - 1);
    const int woff = __shfl_sync(0xffffffffu, wincl - ws, warp);
    __syncthreads();
    return woff + incl - v;
}

// Finds the bin holding the `need`-th largest key: thread t owns bins
// [t*bpt, (t+1)*bpt) with counts hv[].  Result in bc[0] (bin), bc[1] (rank
// of the wanted key inside that bin, counted from its top) and bc[2] (the
// bin's count).
template <int NT>
__device__ __forceinline__ void sel_find_bin(const unsigned* hv, int bpt, int need, int* bc) {
    const int tid = threadIdx.x;
    int tsum = 0;
    for (int q = 0; q < bpt; ++q) tsum += (int)hv[q];
    int total;
    const int below = sel_block_excl_scan<NT>(tsum, bc + 32, total);
    const int above = total - below - tsum;
    if (tid == 0) { bc[0] = 0; bc[1] = 1; bc[2] = 0; }
    __syncthreads();
    if (above < need && need <= above + tsum) {
        int acc = above;
        for (int q = bpt - 1; q >= 0; --q) {
            if (acc + (int)hv[q] >= need) {
                bc[0] = tid * bpt + q;
                bc[1] = need - acc;
                bc[2] = (int)hv[q];
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

// row: the order-preserving keys (order_key) of n scores, resident in shared
// memory (`resident`) or in global memory; the row buffer holds at least
// round_up(n, 4) entries.  With REG (one round: n <= kSelRound), each thread
// reads its chunk once into registers and every pass works from there.
// M < n.  first_hist:
// 4096-bin histogram of key >> 20 over the row, or null.  row_bar: if not
// null, an mbarrier (phase 0) that completes when a TMA copy of the row into
// shared memory has landed; it is waited on (bounded) before the row is read,
// after the first digit when that comes from first_hist.
template <int NT, bool REG = false>
__device__ void row_topm(const uint32_t* row, bool resident, int n, int M, const unsigned* first_hist,
                         const SelectSmem& sm, int lo, int hi, int* out, uint64_t* row_bar,
                         unsigned* status) {
    constexpr int kChunk = kSelRound / NT;  // positions per thread per round
    constexpr int kQ = kChunk / 4;          // 16-byte words per thread per round
    constexpr int kHb = 4096 / NT;          // first-digit bins per thread
    constexpr int kRb = 1024 / NT;          // refinement bins per thread
    static_assert(kQ >= 1 && (kQ & (kQ - 1)) == 0 && kHb >= 1 && kRb >= 1, "thread count");
    const int tid = threadIdx.x;
    int* bc = sm.bc;
    const int rounds = (n + kSelRound - 1) / kSelRound;
    // word j of this thread's chunk in round r, visited in a rotated order so
    // that the lanes of a quarter warp spread over the shared-memory banks
    auto chunk_q = [&](int r, int j) { return (r * kSelRound + tid * kChunk) / 4 + ((j + tid) & (kQ - 1)); };
    auto load4 = [&](int q, uint32_t (&k)[4]) {
        const uint4* src = reinterpret_cast<const uint4*>(row) + q;
        const uint4 v = resident ? *src : __ldg(src);
        k[0] = v.x; k[1] = v.y; k[2] = v.z; k[3] = v.w;
    };
    // REG: the thread's chunk of round 0, read once (words in natural order)
    uint32_t kr[REG ? kChunk : 1];
    if (REG) {
#pragma unroll
        for (int j = 0; j < kQ; ++j) {
            const int q = tid * kQ + j;
            uint32_t k[4] = {0u, 0u, 0u, 0u};
            if (4 * q < n) load4(q, k);
#pragma unroll
            for (int e = 0; e < 4; ++e) kr[(4 * j + e) % (REG ? kChunk : 1)] = k[e];
        }
    }
    // word j of round r: its index q and its four keys
    auto word = [&](int r, int j, uint32_t (&k)[4]) -> int {
        if (REG) {
#pragma unroll
            for (int e = 0; e < 4; ++e) k[e] = kr[(4 * j + e) % (REG ? kChunk : 1)];
            return tid * kQ + j;
        }
        const int q = chunk_q(r, j);
        if (4 * q < n) load4(q, k);
        return q;
    };
    // bit of word j's first key in the thread's chunk masks
    auto word_bit = [&](int j) { return (REG ? j : ((j + tid) & (kQ - 1))) * 4; };
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
        unsigned hv[kHb];
        if (first_hist) {
            const uint4* g4 = reinterpret_cast<const uint4*>(first_hist) + tid * (kHb / 4);
#pragma unroll
            for (int q = 0; q < kHb / 4; ++q) {
                const uint4 u = __ldcg(g4 + q);
                hv[4 * q] = u.x; hv[4 * q + 1] = u.y; hv[4 * q + 2] = u.z; hv[4 * q + 3] = u.w;
            }
        } else {
            wait_row();
            for (int i = tid; i < 4096; i += NT) sm.hist[i] = 0u;
            __syncthreads();
            for (int r = 0; r < rounds; ++r)
#pragma unroll
                for (int j = 0; j < kQ; ++j) {
                    uint32_t k[4];
                    const int q = word(r, j, k);
                    if (4 * q >= n) continue;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * q + e < n) atomicAdd(&sm.hist[k[e] >> 20], 1u);
                }
            __syncthreads();
#pragma unroll
            for (int q = 0; q < kHb; ++q) hv[q] = sm.hist[tid * kHb + q];
        }
        sel_find_bin<NT>(hv, kHb, M, bc);
        b1 = (uint32_t)bc[0];
        krem = bc[1];
    }
    // the two refinement histograms: [0, 1024) and [1024, 2048)
    for (int i = tid; i < 2048; i += NT) sm.hist[i] = 0u;
    if (first_hist) wait_row();

    // ---- 2. candidates (first digit == b1); keys with a higher first digit are
    // selected whatever the lower digits, and counted per thread
    int ncand, above = 0, mine = 0, off;
    {
        for (int r = 0; r < rounds; ++r)
#pragma unroll
            for (int j = 0; j < kQ; ++j) {
                uint32_t k[4];
                const int q = word(r, j, k);
                if (4 * q >= n) continue;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool v = 4 * q + e < n;
                    mine += v && (k[e] >> 20) == b1;
                    above += v && (k[e] >> 20) > b1;
                }
            }
        off = sel_block_excl_scan<NT>(mine, bc + 32, ncand);
        if (ncand <= kCandTotal && mine > 0) {
            int w = off;
            for (int r = 0; r < rounds; ++r)
#pragma unroll
                for (int j = 0; j < kQ; ++j) {
                    uint32_t k[4];
                    const int q = word(r, j, k);
                    if (4 * q >= n) continue;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if ((4 * q + e < n) && (k[e] >> 20) == b1)
                            sm.cand[w++] = make_uint2(k[e], (uint32_t)(4 * q + e));
                }
        }
        __syncthreads();
    }
    const bool overflow = ncand > kCandTotal;

    // ---- 3. refinements (the histograms were cleared before the candidate pass)
    uint32_t prefix = b1 << 20, mask = 0xFFFu << 20;
    int ties = 0;  // keys equal to tau
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        unsigned* h = sm.hist + pass * 1024;
        if (!overflow) {
            for (int i = tid; i < ncand; i += NT) {
                const uint32_t k = sm.cand[i].x;
                if ((k & mask) == prefix) atomicAdd(&h[(k >> shift) & 1023u], 1u);
            }
        } else {
            for (int r = 0; r < rounds; ++r)
#pragma unroll
                for (int j = 0; j < kQ; ++j) {
                    uint32_t k[4];
                    const int q = word(r, j, k);
                    if (4 * q >= n) continue;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * q + e < n && (k[e] & mask) == prefix)
                            atomicAdd(&h[(k[e] >> shift) & 1023u], 1u);
                }
        }
        __syncthreads();
        unsigned hv[kRb];
#pragma unroll
        for (int q = 0; q < kRb; ++q) hv[q] = h[tid * kRb + q];
        sel_find_bin<NT>(hv, kRb, krem, bc);
        prefix |= (uint32_t)bc[0] << shift;
        krem = bc[1];
        ties = bc[2];
        mask |= 1023u << shift;
        if (pass == 0 && ties == 1 && !overflow) {
            // one key left with these 22 bits: it is the M-th largest
            for (int i = tid; i < ncand; i += NT) {
                const uint32_t k = sm.cand[i].x;
                if ((k & mask) == prefix) bc[3] = (int)k;
            }
            __syncthreads();
            prefix = (uint32_t)bc[3];
            break;
        }
    }
    const uint32_t tau = prefix;  // the M-th largest key; krem of its ties are kept

    // emits this thread's selected positions of round r with ranks in [lo, hi)
    // to dst[rank - lo]; `keep` = how many of its keys equal to tau are kept
    // (its lowest ones)
    auto emit = [&](int* dst, int r, int rank, int keep) {
        if (REG) {
            // the thread's keys are in registers in position order: one pass
            int eq_seen = 0;
#pragma unroll
            for (int j = 0; j < kQ; ++j) {
                uint32_t k[4];
                const int q = word(r, j, k);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool v = 4 * q + e < n;
                    const bool eq = v && k[e] == tau;
                    const bool take = (v && k[e] > tau) || (eq && eq_seen < keep);
                    eq_seen += eq;
                    if (take) {
                        if (rank >= lo && rank < hi) dst[rank - lo] = 4 * q + e;
                        ++rank;
                    }
                }
            }
            return;
        }
        uint64_t gtm = 0, eqm = 0;
#pragma unroll
        for (int j = 0; j < kQ; ++j) {
            uint32_t k[4];
            const int q = word(r, j, k);
            if (4 * q >= n) continue;
            const int nv = min(4, n - 4 * q);
            uint32_t g = 0, e4 = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                g |= (uint32_t)(e < nv && k[e] > tau) << e;
                e4 |= (uint32_t)(e < nv && k[e] == tau) << e;
            }
            const int bit = word_bit(j);
            gtm |= (uint64_t)g << bit;
            eqm |= (uint64_t)e4 << bit;
        }
        uint64_t m = gtm | sel_lowest_bits(eqm, keep);
        const int pos0 = r * kSelRound + tid * kChunk;
        while (m) {
            const int b = __ffsll((long long)m) - 1;
            m &= m - 1;
            if (rank >= lo && rank < hi) dst[rank - lo] = pos0 + b;
            ++rank;
        }
    };

    if (rounds == 1 && !overflow) {
        // ---- 4'. one round: per-thread counts from the first-digit pass and the
        // thread's own candidates; only threads whose ranks meet [lo, hi) re-read
        // their chunk
        int gt_c = 0, eq_c = 0;
        for (int i = off; i < off + mine; ++i) {
            const uint32_t k = sm.cand[i].x;
            gt_c += k > tau;
            eq_c += k == tau;
        }
        int keep = eq_c;
        if (krem < ties) {
            int eq_tot;
            const int tie_before = sel_block_excl_scan<NT>(eq_c, bc + 32, eq_tot);
            keep = max(0, min(eq_c, krem - tie_before));
        }
        const int sel_t = above + gt_c + keep;
        int sel_tot;
        // the scan's barriers also end every read of the candidate buffer
        const int rank = sel_block_excl_scan<NT>(sel_t, bc + 32, sel_tot);
        const int nout = min(hi, sel_tot) - lo;
        if (nout > SelectSmem::kStageCap) {
            if (rank < hi && rank + sel_t > lo) emit(out, 0, rank, keep);
        } else if (nout > 0) {
            int* stage = sm.stage();
            if (rank < hi && rank + sel_t > lo) emit(stage, 0, rank, keep);
            __syncthreads();
            for (int i = tid; i < nout; i += NT) out[i] = stage[i];
        }
        __syncthreads();
        return;
    }

    // ---- 4. ranks in position order, round by round
    int rank_base = 0, tie_base = 0;
#pragma unroll 1
    for (int r = 0; r < rounds && rank_base < hi; ++r) {
        int gt_t = 0, eq_t = 0;
#pragma unroll
        for (int j = 0; j < kQ; ++j) {
            uint32_t k[4];
            const int q = word(r, j, k);
            if (4 * q >= n) continue;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool v = 4 * q + e < n;
                gt_t += v && k[e] > tau;
                eq_t += v && k[e] == tau;
            }
        }
        int keep = eq_t;
        if (krem < ties) {
            // only the krem lowest-positioned keys equal to tau are kept
            int eq_tot;
            const int tie_before = tie_base + sel_block_excl_scan<NT>(eq_t, bc + 32, eq_tot);
            tie_base += eq_tot;
            keep = max(0, min(eq_t, krem - tie_before));
        }
        const int sel_t = gt_t + keep;
        int sel_tot;
        const int rank = rank_base + sel_block_excl_scan<NT>(sel_t, bc + 32, sel_tot);
        rank_base += sel_tot;
        if (rank < hi && rank + sel_t > lo) emit(out, r, rank, keep);
    }
    __syncthreads();
}

}  // namespace lisa
