// Sparse softmax attention of one query row over a list of cached positions,
// for one CTA of kAttThreads threads (LISA, arXiv 2607.19358v1, Sec. 3.2 Eq. 1:
// SA_M over the selected rows; GQA: query head h reads KV head h / group).
//
// The K and V rows of the positions (all KV heads of a position are one
// contiguous row) are gathered in stages of 32 with 128-bit loads into
// registers, one stage ahead of the math, and stored into padded shared-memory
// rows.  Warp w serves KV head w / (8 / HKV) and a slice of the value dims;
// the query heads of the group sit on the M side of mma m16n8k16 (rows past
// the group are zero), keys on N for Q.K^T, keys on K for P.V; the softmax is
// online (running max and sum per query head, base 2).
#pragma once

#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"

namespace lisa {

constexpr int kAttThreads = 256;
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kGKeys = 32;             // keys per gather stage
constexpr int kQRow = 128 * 2 + 16;    // padded shared-memory row of one query head (bytes)

template <int HKV>
struct AttGeo {
    static constexpr int d = 128;
    static constexpr int rowbytes = HKV * d * 2;      // one cached K (or V) row
    static constexpr int krow = rowbytes + 16;        // padded shared-memory row
    static constexpr int rpc = rowbytes / 16;         // 16-byte chunks per row
    static constexpr int stage_bytes = kGKeys * 2 * krow;
    static constexpr int chunks_per_thread = kGKeys * 2 * rpc / kAttThreads;
    static constexpr int wph = kAttWarps / HKV;       // warps per KV head
    static constexpr int dw = d / wph;                // output dims per warp
    static constexpr int ntile_o = dw / 8;
    static constexpr int qbytes = ((HKV * 16 * kQRow + 127) / 128) * 128;
};

// Per-warp result: running max (base 2) and sum of query rows gid and gid + 8,
// and the un-normalised output tile of this warp's dims.
template <int HKV>
struct AttAcc {
    float m[2];
    float l[2];
    float o[AttGeo<HKV>::ntile_o][4];
};

// Loads the query heads of one row, [H_q][128] bf16 at q_row, into shared
// memory: group g at rows g*16 .. g*16+group-1, the rest zero.
template <int HKV>
__device__ __forceinline__ void attn_load_query(uint8_t* qs, const __nv_bfloat16* q_row, int group) {
    for (int e = threadIdx.x; e < HKV * 16 * 16; e += kAttThreads) {
        const int g = e / (16 * 16), r = (e / 16) % 16, c = e % 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < group) v = reinterpret_cast<const uint4*>(q_row + (int64_t)(g * group + r) * 128)[c];
        *reinterpret_cast<uint4*>(qs + (g * 16 + r) * kQRow + c * 16) = v;
    }
}

// pos[0..cnt): positions (shared memory).  Position `p_special` (if >= 0) is
// read from k_special / v_special instead of the caches.  Positions outside
// [0, p_max] are masked out and reported through `status`.
template <int HKV>
__device__ __forceinline__ void attn_core(const uint8_t* qs, uint8_t* stage, const int* pos, int cnt,
                                          const __nv_bfloat16* k_cache, const __nv_bfloat16* v_cache,
                                          int64_t row0,  // b * N_max
                                          int p_max, int p_special, const __nv_bfloat16* k_special,
                                          const __nv_bfloat16* v_special, float scale_log2,
                                          unsigned* status, AttAcc<HKV>& acc) {
    using A = AttGeo<HKV>;
    using bf16 = __nv_bfloat16;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tq = lane & 3;
    const int g_w = warp / A::wph, part = warp % A::wph;
    const int nst = (cnt + kGKeys - 1) / kGKeys;
    constexpr int kb_row = HKV * 128;

    uint4 rb[A::chunks_per_thread];
    auto load_stage = [&](int st) {
#pragma unroll
        for (int u = 0; u < A::chunks_per_thread; ++u) {
            const int c = tid + u * kAttThreads;
            const int kk = c / (2 * A::rpc), w2 = c % (2 * A::rpc);
            const int which = w2 / A::rpc, off = w2 % A::rpc;
            int jj = st * kGKeys + kk;
            if (jj >= cnt) jj = st * kGKeys;  // pad with a listed row; masked below
            int ps = pos[jj];
            if (ps < 0 || ps > p_max) ps = 0;  // never dereference an out-of-range position
            const bf16* src = (ps == p_special)
                                  ? (which ? v_special : k_special)
                                  : (which ? v_cache : k_cache) + (row0 + ps) * kb_row;
            rb[u] = __ldg(reinterpret_cast<const uint4*>(src) + off);
        }
    };
    auto store_stage = [&](int st) {
        uint8_t* dst = stage + (st & 1) * A::stage_bytes;
#pragma unroll
        for (int u = 0; u < A::chunks_per_thread; ++u) {
            const int c = tid + u * kAttThreads;
            const int kk = c / (2 * A::rpc), w2 = c % (2 * A::rpc);
            const int which = w2 / A::rpc, off = w2 % A::rpc;
            *reinterpret_cast<uint4*>(dst + which * kGKeys * A::krow + kk * A::krow + off * 16) = rb[u];
        }
    };

    acc.m[0] = acc.m[1] = -INFINITY;
    acc.l[0] = acc.l[1] = 0.0f;
#pragma unroll
    for (int t = 0; t < A::ntile_o; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc.o[t][e] = 0.0f;
    const uint32_t q_base = ptx::smem_u32(qs + g_w * 16 * kQRow);
    const uint32_t head_off = (uint32_t)(g_w * 128 * 2);

    __syncthreads();  // the stage area is free and the query rows are in place
    if (nst > 0) {
        load_stage(0);
        store_stage(0);
    }
    __syncthreads();
#pragma unroll 1
    for (int st = 0; st < nst; ++st) {
        if (st + 1 < nst) load_stage(st + 1);  // in flight while this stage computes
        const uint32_t kb = ptx::smem_u32(stage + (st & 1) * A::stage_bytes);
        const uint32_t vb = kb + kGKeys * A::krow;
        float sc[4][4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[t][e] = 0.0f;
#pragma unroll
        for (int ks = 0; ks < 8; ks += 2) {
            uint32_t qa0[4], qa1[4];
            {
                const int row = (lane & 7) + ((lane >> 3) & 1) * 8;
                const int col = ks * 16 + (lane >> 4) * 8;
                ptx::ldmatrix_x4(qa0, q_base + row * kQRow + col * 2);
                ptx::ldmatrix_x4(qa1, q_base + row * kQRow + (col + 16) * 2);
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                uint32_t kr[4];
                const int key = nt * 8 + (lane & 7);
                const int dim0 = ks * 16 + (lane >> 3) * 8;
                ptx::ldmatrix_x4(kr, kb + key * A::krow + head_off + dim0 * 2);
                ptx::mma_bf16(sc[nt], qa0, kr[0], kr[1]);
                ptx::mma_bf16(sc[nt], qa1, kr[2], kr[3]);
            }
        }
        float mt[2] = {-INFINITY, -INFINITY};
        bool bad = false;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = st * kGKeys + nt * 8 + 2 * tq + (e & 1);
                float v = sc[nt][e] * scale_log2;
                if (j >= cnt) {
                    v = -INFINITY;
                } else {
                    const int ps = pos[j];
                    if (ps < 0 || ps > p_max) { v = -INFINITY; bad = true; }
                }
                sc[nt][e] = v;
                mt[e >> 1] = fmaxf(mt[e >> 1], v);
            }
        if (bad) record_error(status, kDevBounds);
        float corr[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], 1));
            mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], 2));
            const float m_new = fmaxf(acc.m[h], mt[h]);
            corr[h] = (m_new == -INFINITY) ? 1.0f : exp2f(acc.m[h] - m_new);
            acc.m[h] = m_new;
            acc.l[h] *= corr[h];
        }
#pragma unroll
        for (int t = 0; t < A::ntile_o; ++t) {
            acc.o[t][0] *= corr[0]; acc.o[t][1] *= corr[0];
            acc.o[t][2] *= corr[1]; acc.o[t][3] *= corr[1];
        }
        uint32_t pa[2][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            float pv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float m = acc.m[e >> 1];
                pv[e] = (m == -INFINITY) ? 0.0f : exp2f(sc[nt][e] - m);
                acc.l[e >> 1] += pv[e];
            }
            const int kk = nt >> 1, hi2 = nt & 1;
            pa[kk][0 + 2 * hi2] = ptx::pack_bf16(pv[0], pv[1]);
            pa[kk][1 + 2 * hi2] = ptx::pack_bf16(pv[2], pv[3]);
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
            for (int t = 0; t < A::ntile_o; t += 2) {
                uint32_t vr[4];
                const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                const int dim0 = part * A::dw + (t + (lane >> 4)) * 8;
                ptx::ldmatrix_x4_trans(vr, vb + key * A::krow + head_off + dim0 * 2);
                ptx::mma_bf16(acc.o[t], pa[kk], vr[0], vr[1]);
                ptx::mma_bf16(acc.o[t + 1], pa[kk], vr[2], vr[3]);
            }
        }
        if (st + 1 < nst) store_stage(st + 1);
        __syncthreads();
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 1);
        acc.l[h] += __shfl_xor_sync(0xffffffffu, acc.l[h], 2);
    }
}

}  // namespace lisa
