// Linear-attention branch of the decode step, one slice at a time (LISA,
// arXiv 2607.19358v1, Sec. 3.1 and Sec. 3.3 Eq. 3-4): S += phi(k)^T v for one
// KV head's value columns [c0, c0 + 32), then o_lin = phi(q) S for the query
// heads of the group (divided by phi(q).z in the elu+1 mode).  Shared by the
// decode kernels; run by the kLaThreads threads that start at thread
// `first` of the block, synchronised by named barrier kLaBar.
#pragma once

#include "lisa_internal.cuh"
#include "sm100_ptx.cuh"

namespace lisa {
namespace dec {

using bf16 = __nv_bfloat16;

constexpr int kLaThreads = 128;  // threads of the linear-branch warps
constexpr int kLaBar = 2;        // their named barrier
constexpr int kLaD = 128;        // head dimension
constexpr int kLaCols = 32;      // value columns per slice

__device__ __forceinline__ void group_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ float feat(int phi, float x) {
    if (phi == LISA_PHI_IDENTITY) return x;
    return x > 0.0f ? x + 1.0f : __expf(x);
}

// One slice: sequence b, KV head g, value columns [c0, c0+32).  s_slice holds
// S[:, c0:c0+32] of that head (already loaded, or in flight as cp.async
// groups of the calling threads).  P supplies k_L, v_L, q_L, S, z, olin, H_q,
// H_kv, group and phi.
template <class PT>
__device__ void linear_slice(const PT& P, int first, int b, int g, int c0, float* s_slice, float* fk,
                             float* fq, float* vcol, float* zloc, float* den) {
    const int tid = threadIdx.x - first, lane = tid & 31, warp = tid >> 5;
    const bf16* kl = P.k_L + ((int64_t)b * P.H_kv + g) * kLaD;
    const bf16* vl = P.v_L + ((int64_t)b * P.H_kv + g) * kLaD;
    // 128-bit loads: 8 bf16 per load, one load per thread for each vector
    auto unpack8 = [](const uint4& u, float (&f)[8]) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 t = __bfloat1622float2(h2[e]);
            f[2 * e] = t.x;
            f[2 * e + 1] = t.y;
        }
    };
    for (int e = tid; e < kLaD / 8 + kLaCols / 8 + P.group * (kLaD / 8); e += kLaThreads) {
        float f[8];
        if (e < kLaD / 8) {
            unpack8(reinterpret_cast<const uint4*>(kl)[e], f);
#pragma unroll
            for (int x = 0; x < 8; ++x) fk[8 * e + x] = feat(P.phi, f[x]);
        } else if (e < kLaD / 8 + kLaCols / 8) {
            const int e2 = e - kLaD / 8;
            unpack8(reinterpret_cast<const uint4*>(vl + c0)[e2], f);
#pragma unroll
            for (int x = 0; x < 8; ++x) vcol[8 * e2 + x] = f[x];
        } else {
            const int e3 = e - kLaD / 8 - kLaCols / 8;
            const int h = e3 / (kLaD / 8), c8 = e3 % (kLaD / 8);
            unpack8(reinterpret_cast<const uint4*>(
                        P.q_L + ((int64_t)b * P.H_q + g * P.group + h) * kLaD)[c8], f);
#pragma unroll
            for (int x = 0; x < 8; ++x) fq[h * kLaD + 8 * c8 + x] = feat(P.phi, f[x]);
        }
    }
    ptx::cp_async_wait_all();  // the state slice (when it was prefetched)
    group_sync(kLaBar, kLaThreads);
    const bool norm = P.phi == LISA_PHI_ELU1_NORM;
    float* Sg = P.S + ((int64_t)b * P.H_kv + g) * kLaD * kLaD;
    if (norm) {
        const float* zg = P.z + ((int64_t)b * P.H_kv + g) * kLaD;
        for (int i = tid; i < kLaD; i += kLaThreads) zloc[i] = zg[i] + fk[i];
    }
    for (int e = tid; e < kLaD * kLaCols; e += kLaThreads) {
        const int i = e / kLaCols, c = e % kLaCols;
        const float nv = fmaf(fk[i], vcol[c], s_slice[e]);
        s_slice[e] = nv;
        Sg[(int64_t)i * kLaD + c0 + c] = nv;
    }
    group_sync(kLaBar, kLaThreads);
    if (norm) {
        // z itself is advanced by the attend kernel: the sibling slices of this
        // head still read the old z here
        for (int h = warp; h < P.group; h += kLaThreads / 32) {
            float dz = 0.0f;
            for (int i = lane; i < kLaD; i += 32) dz = fmaf(fq[h * kLaD + i], zloc[i], dz);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dz += __shfl_xor_sync(0xffffffffu, dz, o);
            if (lane == 0) den[h] = dz;
        }
        group_sync(kLaBar, kLaThreads);
    }
    for (int e = tid; e < P.group * kLaCols; e += kLaThreads) {
        const int h = e / kLaCols, c = e % kLaCols;
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four independent chains
#pragma unroll 8
        for (int i = 0; i < kLaD; i += 4)
#pragma unroll
            for (int u = 0; u < 4; ++u)
                acc[u] = fmaf(fq[h * kLaD + i + u], s_slice[(i + u) * kLaCols + c], acc[u]);
        const float sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        P.olin[((int64_t)b * P.H_q + g * P.group + h) * kLaD + c0 + c] = norm ? sum / den[h] : sum;
    }
    group_sync(kLaBar, kLaThreads);
}

}  // namespace dec
}  // namespace lisa
