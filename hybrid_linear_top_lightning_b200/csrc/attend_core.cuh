// Sparse softmax attention of one query row over a list of cached positions,
// for one CTA of kAttThreads threads (LISA, arXiv 2607.19358v1, Sec. 3.2 Eq. 1:
// SA_M over the selected rows; GQA: query head h reads KV head h / group).
//
// The K and V rows of the positions (all KV heads of a position are one
// contiguous row) are gathered in stages by 16-byte asynchronous copies
// (cp.async, through L2 only) into padded shared-memory rows, in a ring of
// kAttStages stages of which all but the one being computed are in flight.
//
// Tensor-core mapping (mma m16n8k16, bf16 in, fp32 accumulate): the keys sit
// on the M side and the (up to 8) query heads of a GQA group on N, so no MMA
// row is padding.  Scores: S^T[key][head] = K[key,:] . Q[head,:], with the
// query fragments held in registers for the whole row.  Output: the
// probabilities are transposed in registers (movmatrix) and O^T[dim][head] +=
// V^T[dim][key] P^T[key][head].  The warps serving one KV head split each
// stage's keys 16 apiece and keep their own online-softmax state (base 2);
// at the end the first warp of each KV head merges the others' states into
// its registers (one exchange through shared memory).
#pragma once

#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"

namespace lisa {

constexpr int kAttThreads = 256;
constexpr int kAttWarps = kAttThreads / 32;
constexpr int kAttStages = 3;  // gather stages in the shared-memory ring

template <int HKV>
struct AttGeo {
    static constexpr int d = 128;
    static constexpr int rowbytes = HKV * d * 2;          // one cached K (or V) row
    static constexpr int krow = rowbytes + 16;            // padded shared-memory row
    static constexpr int rpc = rowbytes / 16;             // 16-byte chunks per row
    static constexpr int wph = kAttWarps / HKV;           // warps per KV head
    static constexpr int keys = 16 * wph;                 // keys per stage
    static constexpr int tpk = kAttThreads / keys;        // copying threads per key
    static constexpr int cpt = 2 * rpc / tpk;             // chunks per copying thread
    static constexpr int stage_bytes = keys * 2 * krow;   // K rows, then V rows
    static constexpr int ring_bytes = kAttStages * stage_bytes;
    // merge exchange (in the ring after the loop): per warp 36 floats per lane
    static constexpr int xfer_bytes = kAttWarps * 36 * 32 * 4;
    static_assert(cpt * tpk == 2 * rpc, "chunk split");
    static_assert(xfer_bytes <= ring_bytes, "merge exchange fits in the ring");
};

// Query fragments of one row (B operand of the score MMA): per thread, head
// gid of the warp's KV-head group, dims ks*16 + 2tq (+1) and + 8 (+9); heads
// past the group are zero.  Loaded before the positions are known.
struct AttQ {
    uint32_t f[8][2];
};

template <int HKV>
__device__ __forceinline__ AttQ attn_load_q(const __nv_bfloat16* q_row, int group) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const int g_w = warp / AttGeo<HKV>::wph;
    const bool live = gid < group;
    const uint32_t* qh =
        reinterpret_cast<const uint32_t*>(q_row + (int64_t)(g_w * group + (live ? gid : 0)) * 128);
    AttQ q;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        q.f[ks][0] = live ? __ldg(qh + ks * 8 + tq) : 0u;
        q.f[ks][1] = live ? __ldg(qh + ks * 8 + 4 + tq) : 0u;
    }
    return q;
}

// Online-softmax state of one KV head's query heads, held by the first warp
// (part 0) of the head after attn_core: lane (gid, tq) has head slots
// r = 2tq + h (h = 0, 1) with base-2 running max m[h] and sum l[h], and the
// un-normalised output o[t][e] of slot 2tq + (e & 1), dim t*16 + gid + 8*(e >> 1).
struct AttOut {
    float m[2];
    float l[2];
    float o[8][4];
};

// Where the gathered K and V rows come from: the caches of one sequence
// (row0 = b * N_max), except position p_special (if >= 0), which is read from
// k_special / v_special; positions outside [0, p_max] are never dereferenced.
struct AttSrc {
    const __nv_bfloat16* k_cache;
    const __nv_bfloat16* v_cache;
    int64_t row0;
    int p_max;
    int p_special;
    const __nv_bfloat16* k_special;
    const __nv_bfloat16* v_special;
};

// The position this thread copies in stage st of the list pos[0..cnt) (the
// stage's first entry pads a short last stage; those keys are masked).  With
// pos == nullptr the list is the run of positions iota0, iota0 + 1, ...
template <int HKV>
__device__ __forceinline__ int attn_stage_pos(const int* pos, int cnt, int st, int iota0 = 0) {
    using A = AttGeo<HKV>;
    if (st * A::keys >= cnt) return 0;
    const int jj = st * A::keys + threadIdx.x / A::tpk;
    const int e = jj < cnt ? jj : st * A::keys;
    return pos ? pos[e] : iota0 + e;
}

// Issues this thread's 16-byte asynchronous copies of stage st into ring slot
// st % kAttStages and records the stage's positions (-1 past the list).  With
// SPLIT, the K row of each key instead goes by one 1-D bulk copy (from the
// key's first thread, arriving on kbar[slot]) and the threads copy the V rows
// only: the two copy paths of the SM share the gather (on the 7B prefill,
// 8.1 ms against 8.7 ms with 16-byte copies alone; 3/4 of K by bulk copy was
// no better than none).
template <int HKV, bool SPLIT = false>
__device__ __forceinline__ void attn_issue_stage(uint8_t* ring, int* spos, int cnt, int st, int raw,
                                                 const AttSrc& src, uint64_t* kbar = nullptr) {
    using A = AttGeo<HKV>;
    using bf16 = __nv_bfloat16;
    constexpr int GK = A::keys;
    constexpr int kb_row = HKV * 128;
    const int ck = threadIdx.x / A::tpk, sub = threadIdx.x % A::tpk;
    uint8_t* dst = ring + (st % kAttStages) * A::stage_bytes;
    if (sub == 0) spos[(st % kAttStages) * GK + ck] = (st * GK + ck < cnt) ? raw : -1;
    const int ps = (raw < 0 || raw > src.p_max) ? 0 : raw;  // never dereference out of range
    const bf16* ksrc = (ps == src.p_special) ? src.k_special : src.k_cache + (src.row0 + ps) * kb_row;
    const bf16* vsrc = (ps == src.p_special) ? src.v_special : src.v_cache + (src.row0 + ps) * kb_row;
    if (SPLIT) {
        if (sub == 0) {
            uint64_t* bar = kbar + st % kAttStages;
            ptx::fence_proxy_async_shared();  // the slot's earlier reads precede the copy
            ptx::mbar_arrive_expect_tx(bar, A::rowbytes);
            ptx::bulk_load(dst + ck * A::krow, ksrc, A::rowbytes, bar);
        }
#pragma unroll
        for (int u = 0; u < A::cpt / 2; ++u) {
            const int off = sub + u * A::tpk;
            ptx::cp_async_16(dst + GK * A::krow + ck * A::krow + off * 16,
                             reinterpret_cast<const uint4*>(vsrc) + off);
        }
        return;
    }
#pragma unroll
    for (int u = 0; u < A::cpt; ++u) {
        const int i = sub + u * A::tpk;
        const int which = i / A::rpc, off = i % A::rpc;
        const bf16* from = which ? vsrc : ksrc;
        ptx::cp_async_16(dst + which * GK * A::krow + ck * A::krow + off * 16,
                         reinterpret_cast<const uint4*>(from) + off);
    }
}

// One stage of 16 keys for one warp (the bulk-copy gathers of the decode and
// prefill kernels): K rows at shared address kb, V rows at vb, `krow` bytes
// apart, the warp's KV head `head_off` bytes into each row; qf are its query
// fragments (the layout of AttQ).  Key k of the stage counts iff bit k of
// `valid` is set (each lane reads bits gid and gid + 8).  Updates the warp's
// online-softmax state: m and l (base 2; l summed over this lane's keys only)
// and o, in the layout of AttOut.
__device__ __forceinline__ void attn_stage16(const uint32_t (&qf)[8][2], uint32_t kb, uint32_t vb,
                                             int krow, uint32_t head_off, unsigned valid,
                                             float scale_log2, float (&m)[2], float (&l)[2],
                                             float (&o)[8][4]) {
    const int lane = threadIdx.x & 31, gid = lane >> 2;
    // ldmatrix lane addressing: K as A (keys x dims), V as A^T (dims x keys)
    const int ka_key = (lane & 7) + ((lane >> 3) & 1) * 8, ka_dim = (lane >> 4) * 8;
    const int va_key = (lane & 7) + (lane >> 4) * 8, va_dim = ((lane >> 3) & 1) * 8;
    float s0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int ks = 0; ks < 8; ks += 2) {
        uint32_t a0[4], a1[4];
        ptx::ldmatrix_x4(a0, kb + ka_key * krow + head_off + (ks * 16 + ka_dim) * 2);
        ptx::ldmatrix_x4(a1, kb + ka_key * krow + head_off + ((ks + 1) * 16 + ka_dim) * 2);
        ptx::mma_bf16(s0, a0, qf[ks][0], qf[ks][1]);
        ptx::mma_bf16(s1, a1, qf[ks + 1][0], qf[ks + 1][1]);
    }
    // element e: key gid + 8 (e >> 1), head slot 2tq + (e & 1)
    float v[4];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const bool ok = (valid >> (gid + 8 * r)) & 1u;
#pragma unroll
        for (int h = 0; h < 2; ++h)
            v[2 * r + h] = ok ? (s0[2 * r + h] + s1[2 * r + h]) * scale_log2 : -INFINITY;
    }
    float corr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float mt = fmaxf(v[h], v[2 + h]);
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
        const float m_new = fmaxf(m[h], mt);
        corr[h] = (m_new == -INFINITY) ? 1.0f : ptx::ex2(m[h] - m_new);
        m[h] = m_new;
        l[h] *= corr[h];
    }
    float pr[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float mm = m[e & 1];
        pr[e] = (mm == -INFINITY) ? 0.0f : ptx::ex2(v[e] - mm);
        l[e & 1] += pr[e];
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        o[t][0] *= corr[0]; o[t][1] *= corr[1];
        o[t][2] *= corr[0]; o[t][3] *= corr[1];
    }
    // P^T fragments (keys x heads) -> B operand (k = keys, n = heads)
    const uint32_t b0 = ptx::movmatrix_trans(ptx::pack_bf16(pr[0], pr[1]));
    const uint32_t b1 = ptx::movmatrix_trans(ptx::pack_bf16(pr[2], pr[3]));
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        uint32_t va[4];
        ptx::ldmatrix_x4_trans(va, vb + va_key * krow + head_off + (t * 16 + va_dim) * 2);
        ptx::mma_bf16(o[t], va, b0, b1);
    }
}

// q: the row's query fragments (attn_load_q), `group` <= 8 heads per KV
// head.  pos[0..cnt): positions (shared or global memory; nullptr: the run
// iota0 .. iota0 + cnt - 1), gathered from `src`; positions outside [0, src.p_max] are masked out and reported through
// `status`.  `ring` holds AttGeo<HKV>::ring_bytes bytes, `spos` (shared
// memory) kAttStages * AttGeo<HKV>::keys ints; both are clobbered.  The
// result is valid in the warps with part == 0 (warp % wph == 0).
template <int HKV, bool SPLIT = false>
__device__ __forceinline__ void attn_core(const AttQ& q, uint8_t* ring, int* spos, const int* pos,
                                          int cnt, const AttSrc& src, float scale_log2,
                                          unsigned* status, AttOut& out, uint64_t* kbar = nullptr,
                                          int iota0 = 0) {
    using A = AttGeo<HKV>;
    constexpr int GK = A::keys;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tq = lane & 3;
    const int g_w = warp / A::wph, part = warp % A::wph;
    const int key0 = part * 16;  // this warp's keys within a stage
    const int nst = (cnt + GK - 1) / GK;
    const int p_max = src.p_max;
    auto load_pos = [&](int st) { return attn_stage_pos<HKV>(pos, cnt, st, iota0); };
    auto issue_stage = [&](int st, int raw) {
        attn_issue_stage<HKV, SPLIT>(ring, spos, cnt, st, raw, src, kbar);
    };
    if (SPLIT && tid == 0) {
        for (int i = 0; i < kAttStages; ++i) ptx::mbar_init(kbar + i, GK);  // one arrival per key
        ptx::fence_mbar_init();
    }

    float* m = out.m;  // heads 2tq, 2tq + 1
    float* l = out.l;
    float (*o)[4] = out.o;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.0f;
#pragma unroll
    for (int t = 0; t < 8; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[t][e] = 0.0f;

    const uint32_t head_off = (uint32_t)(g_w * 128 * 2);
    // ldmatrix lane addressing: K as A (keys x dims), V as A^T (dims x keys)
    const int ka_key = key0 + (lane & 7) + ((lane >> 3) & 1) * 8, ka_dim = (lane >> 4) * 8;
    const int va_key = key0 + (lane & 7) + (lane >> 4) * 8, va_dim = ((lane >> 3) & 1) * 8;

    __syncthreads();  // the ring is free
#pragma unroll
    for (int st = 0; st < kAttStages - 1; ++st) {
        if (st < nst) issue_stage(st, load_pos(st));
        ptx::cp_async_commit();  // (possibly empty) group per stage keeps the count uniform
    }
    // the positions of the next stage to issue are loaded one iteration ahead
    int next_pos = load_pos(kAttStages - 1);
#pragma unroll 1
    for (int st = 0; st < nst; ++st) {
        ptx::cp_async_wait_group<kAttStages - 2>();  // this thread's copies of stage st landed
        if (SPLIT && !ptx::mbar_wait_bounded(kbar + st % kAttStages, (st / kAttStages) & 1, 1u << 22))
            record_error(status, kDevTimeout);  // (the stage's K rows)
        // all copies of stage st are visible, and every warp is done with
        // stage st - 1, whose slot the next issue reuses
        __syncthreads();
        if (st + kAttStages - 1 < nst) issue_stage(st + kAttStages - 1, next_pos);
        ptx::cp_async_commit();
        next_pos = load_pos(st + kAttStages);
        const uint32_t kb = ptx::smem_u32(ring + (st % kAttStages) * A::stage_bytes);
        const uint32_t vb = kb + GK * A::krow;
        const int* stpos = spos + (st % kAttStages) * GK;

        // scores of this warp's 16 keys x 8 heads (two accumulation chains)
        float s0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, s1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int ks = 0; ks < 8; ks += 2) {
            uint32_t a0[4], a1[4];
            ptx::ldmatrix_x4(a0, kb + ka_key * A::krow + head_off + (ks * 16 + ka_dim) * 2);
            ptx::ldmatrix_x4(a1, kb + ka_key * A::krow + head_off + ((ks + 1) * 16 + ka_dim) * 2);
            ptx::mma_bf16(s0, a0, q.f[ks][0], q.f[ks][1]);
            ptx::mma_bf16(s1, a1, q.f[ks + 1][0], q.f[ks + 1][1]);
        }
        // element e: key key0 + gid + 8 (e >> 1), head 2tq + (e & 1)
        float v[4];
        bool bad = false;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int ps = stpos[key0 + gid + 8 * r];  // -1 past the list
            const bool listed = st * GK + key0 + gid + 8 * r < cnt;
            const bool ok = listed && ps >= 0 && ps <= p_max;
            bad |= listed && !ok;
#pragma unroll
            for (int h = 0; h < 2; ++h)
                v[2 * r + h] = ok ? (s0[2 * r + h] + s1[2 * r + h]) * scale_log2 : -INFINITY;
        }
        if (bad) record_error(status, kDevBounds);
        float corr[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float mt = fmaxf(v[h], v[2 + h]);
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
            const float m_new = fmaxf(m[h], mt);
            corr[h] = (m_new == -INFINITY) ? 1.0f : ptx::ex2(m[h] - m_new);
            m[h] = m_new;
            l[h] *= corr[h];
        }
        float p[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float mm = m[e & 1];
            p[e] = (mm == -INFINITY) ? 0.0f : ptx::ex2(v[e] - mm);
            l[e & 1] += p[e];
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            o[t][0] *= corr[0]; o[t][1] *= corr[1];
            o[t][2] *= corr[0]; o[t][3] *= corr[1];
        }
        // P^T fragments (keys x heads) -> B operand (k = keys, n = heads)
        const uint32_t b0 = ptx::movmatrix_trans(ptx::pack_bf16(p[0], p[1]));
        const uint32_t b1 = ptx::movmatrix_trans(ptx::pack_bf16(p[2], p[3]));
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            uint32_t va[4];
            ptx::ldmatrix_x4_trans(va, vb + va_key * A::krow + head_off + (t * 16 + va_dim) * 2);
            ptx::mma_bf16(o[t], va, b0, b1);
        }
    }
    ptx::cp_async_wait_all();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 4);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 8);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 16);
    }
    if (A::wph == 1) return;
    __syncthreads();  // every warp is done with the ring

    // ---- the other warps of the KV head hand their state to its first warp
    float* xf = reinterpret_cast<float*>(ring) + warp * 36 * 32 + lane;  // [36][32] per warp
    if (part != 0) {
        xf[0] = m[0]; xf[32] = m[1]; xf[64] = l[0]; xf[96] = l[1];
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) xf[(4 + t * 4 + e) * 32] = o[t][e];
    }
    __syncthreads();
    if (part != 0) return;
#pragma unroll 1
    for (int k = 1; k < A::wph; ++k) {
        const float* yf = xf + k * 36 * 32;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float mk = yf[h * 32], lk = yf[(2 + h) * 32];
            const float M = fmaxf(m[h], mk);
            const float a = (m[h] == -INFINITY) ? 0.0f : exp2f(m[h] - M);
            const float c = (mk == -INFINITY) ? 0.0f : exp2f(mk - M);
            m[h] = M;
            l[h] = l[h] * a + lk * c;
#pragma unroll
            for (int t = 0; t < 8; ++t)
#pragma unroll
                for (int e = h; e < 4; e += 2) o[t][e] = o[t][e] * a + yf[(4 + t * 4 + e) * 32] * c;
        }
    }
}

}  // namespace lisa
