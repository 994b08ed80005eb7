// Sparse softmax attention over given index lists (lisa_sparse_attn) for many
// query rows, bf16, head dim 128: one CTA per query row runs the gather (K rows
// by 1-D bulk copies, V rows by 16-byte cp.async) and tensor-core online
// softmax of attend_core.cuh over the row's count[b,t] positions and writes
// the normalised output (LISA, arXiv 2607.19358v1,
// Sec. 3.2 Eq. 1, the SA_M branch).  Positions outside [0, p] are masked out
// and reported as LISA_ERR_DEVICE_BOUNDS through the status word.
#include "attend_core.cuh"
#include "lisa_fast.cuh"
#include "lisa_internal.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;
struct SpParams {
    int B, T, n_past, N_max, H_q, group, M;
    float scale_log2;
    const bf16* q;
    const bf16* k;
    const bf16* v;
    const int32_t* idx;
    const int32_t* count;
    bf16* o;
    unsigned* status;
};

template <int HKV>
struct SpSmem {
    static constexpr int spos = 0;                                     // int[stages][keys]
    static constexpr int ring = (kAttStages * AttGeo<HKV>::keys * 4 + 127) / 128 * 128;
    static constexpr int kbar = ring + AttGeo<HKV>::ring_bytes;        // uint64[kAttStages]
    static constexpr int total = kbar + kAttStages * 8;
    static_assert(total <= 227 * 1024, "shared memory per CTA");
};

template <int HKV>
__global__ void __launch_bounds__(kAttThreads, 1) k_sparse_rows(const SpParams P) {
    using L = SpSmem<HKV>;
    extern __shared__ __align__(128) uint8_t sp_raw[];
    int* spos = reinterpret_cast<int*>(sp_raw + L::spos);
    const int row = blockIdx.x;
    const int b = row / P.T, t = row % P.T;
    const int p = P.n_past + t;
    const int cnt = max(0, min(P.count[row], P.M));
    const int* pos = P.idx + (int64_t)row * P.M;  // read through L1 by the gather
    const AttQ q = attn_load_q<HKV>(P.q + (int64_t)row * P.H_q * 128, P.group);
    AttOut r;
    const AttSrc kv{P.k, P.v, (int64_t)b * P.N_max, p, -1, nullptr, nullptr};
    attn_core<HKV, true>(q, sp_raw + L::ring, spos, pos, cnt, kv, P.scale_log2, P.status, r,
                         reinterpret_cast<uint64_t*>(sp_raw + L::kbar));
    // normalised output of each KV head's query heads (group rows of 128 dims,
    // contiguous in o), staged by the head's first warp in its own slot of the
    // ring and stored with 16-byte writes
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp % AttGeo<HKV>::wph != 0) return;
    const int g = warp / AttGeo<HKV>::wph, gid = lane >> 2, tq = lane & 3;
    bf16* stage = reinterpret_cast<bf16*>(sp_raw + L::ring) + warp * 36 * 32 * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int slot = 2 * tq + h;
        if (slot >= P.group) continue;
        const float inv = r.l[h] > 0.0f ? 1.0f / r.l[h] : 0.0f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            stage[slot * 128 + t * 16 + gid] = __float2bfloat16_rn(r.o[t][h] * inv);
            stage[slot * 128 + t * 16 + gid + 8] = __float2bfloat16_rn(r.o[t][h + 2] * inv);
        }
    }
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(P.o + ((int64_t)row * P.H_q + g * P.group) * 128);
    const uint4* src = reinterpret_cast<const uint4*>(stage);
    for (int c = lane; c < P.group * 16; c += 32) dst[c] = src[c];
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

}  // namespace

size_t fast_attention_ws_bytes(const Shape&, bool) { return kStatusBytes; }

bool fast_attention_supported(const Shape& s, const void* q, const void* k, const void* v,
                              bool dense) {
    if (dense) return false;
    if (s.dtype != LISA_BF16 || s.d != 128) return false;
    if (!(s.H_kv == 1 || s.H_kv == 2 || s.H_kv == 4) || s.group > 8) return false;
    return aligned16(q) && aligned16(k) && aligned16(v);
}

cudaError_t fast_attention(const Shape& s, const void* q, const void* k, const void* v,
                           const int32_t* idx, const int32_t* count, void* o, void* ws,
                           cudaStream_t st) {
    SpParams P;
    P.B = s.B; P.T = s.T; P.n_past = s.n_past; P.N_max = s.N_max; P.H_q = s.H_q;
    P.group = s.group; P.M = s.M; P.scale_log2 = s.sm_scale * 1.4426950408889634f;
    P.q = (const bf16*)q; P.k = (const bf16*)k; P.v = (const bf16*)v;
    P.idx = idx; P.count = count; P.o = (bf16*)o; P.status = (unsigned*)ws;
    static bool attrs[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attrs[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_sparse_rows<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<1>::total);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_sparse_rows<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<2>::total);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k_sparse_rows<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpSmem<4>::total);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attrs[dev] = true;
    }
    const dim3 grid(s.B * s.T);
    switch (s.H_kv) {
        case 1: k_sparse_rows<1><<<grid, kAttThreads, SpSmem<1>::total, st>>>(P); break;
        case 2: k_sparse_rows<2><<<grid, kAttThreads, SpSmem<2>::total, st>>>(P); break;
        default: k_sparse_rows<4><<<grid, kAttThreads, SpSmem<4>::total, st>>>(P); break;
    }
    return cudaGetLastError();
}

}  // namespace lisa
