// The gate of the two branches (LISA, arXiv 2607.19358v1, Sec. 3.2 Eq. 1):
// o = g * o_lin + (1 - g) * o_sparse with g = sigmoid(logit), one logit per
// (token, query head), for bf16 tensors with head dim 128.  HBM-bound: every
// thread moves 16-byte words (8 values) of the three row-major tensors.
#include "lisa_fast.cuh"
#include "lisa_internal.cuh"

namespace lisa {
namespace {

using bf16 = __nv_bfloat16;
constexpr int kGateD = 128;
constexpr int kWordsPerRow = kGateD / 8;

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __bfloat1622float2(h[e]);
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}

__global__ void __launch_bounds__(256) k_gate_bf16(int64_t words, const bf16* __restrict__ logit,
                                                   const uint4* __restrict__ o_lin,
                                                   const uint4* __restrict__ o_sp,
                                                   uint4* __restrict__ o) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float x = __bfloat162float(logit[i / kWordsPerRow]);
        const float g = 1.0f / (1.0f + __expf(-x));
        float a[8], c[8];
        unpack8(__ldcs(o_lin + i), a);
        unpack8(__ldcs(o_sp + i), c);
        uint4 r;
        __nv_bfloat162* rh = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
        for (int e = 0; e < 4; ++e)
            rh[e] = __floats2bfloat162_rn(fmaf(g, a[2 * e] - c[2 * e], c[2 * e]),
                                          fmaf(g, a[2 * e + 1] - c[2 * e + 1], c[2 * e + 1]));
        __stcs(o + i, r);
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

bool fast_gate_supported(const Shape& s, const void* o_lin, const void* o_sp, const void* o) {
    return s.dtype == LISA_BF16 && s.d == kGateD && aligned16(o_lin) && aligned16(o_sp) &&
           aligned16(o);
}

cudaError_t fast_gate(const Shape& s, const void* logit, const void* o_lin, const void* o_sp,
                      void* o, cudaStream_t st) {
    const int64_t words = (int64_t)s.B * s.T * s.H_q * kWordsPerRow;
    if (words == 0) return cudaSuccess;
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (words + 255) / 256;
    const int blocks = (int)(want < (int64_t)sms * 16 ? want : (int64_t)sms * 16);
    k_gate_bf16<<<blocks, 256, 0, st>>>(words, (const bf16*)logit, (const uint4*)o_lin,
                                        (const uint4*)o_sp, (uint4*)o);
    return cudaGetLastError();
}

}  // namespace lisa
