// Segment state transfer and correction at the end of a reasoning segment
// (LISA, arXiv 2607.19358v1, Sec. 3.3 "Segment State Update", Eq. 6-9), for
// every linear-attention state S[b, g]:
//   grad_t   = S_end - S_{t-1}                       (Eq. 6)
//   mean     = (grad_1 + ... + grad_{t-1}) / (t - 1)  (Eq. 7; zero at t = 1)
//   grad_hat = (1 - alpha) grad_t + alpha mean        (Eq. 8)
//   S_t      = S_{t-1} + grad_hat                     (Eq. 9)
// One elementwise pass over the fp32 states, 16 bytes per access: HBM-bound.
#include "lisa_fast.cuh"
#include "lisa_internal.cuh"

namespace lisa {
namespace {

__device__ __forceinline__ float transfer1(float& s, float& s0, float& g, float inv_prev,
                                           float alpha) {
    const float grad = s - s0;
    const float hat = fmaf(alpha, g * inv_prev - grad, grad);  // (1-a) grad + a mean
    const float st = s0 + hat;
    g += grad;
    s = st;
    s0 = st;
    return st;
}

__global__ void __launch_bounds__(256) k_state_transfer4(int64_t n4, float4* __restrict__ S,
                                                         float4* __restrict__ S0,
                                                         float4* __restrict__ G, float inv_prev,
                                                         float alpha) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 s = S[i], s0 = S0[i], g = G[i];
        transfer1(s.x, s0.x, g.x, inv_prev, alpha);
        transfer1(s.y, s0.y, g.y, inv_prev, alpha);
        transfer1(s.z, s0.z, g.z, inv_prev, alpha);
        transfer1(s.w, s0.w, g.w, inv_prev, alpha);
        S[i] = s;
        S0[i] = s0;
        G[i] = g;
    }
}

__global__ void __launch_bounds__(256) k_state_transfer1(int64_t n, float* __restrict__ S,
                                                         float* __restrict__ S0,
                                                         float* __restrict__ G, float inv_prev,
                                                         float alpha) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        transfer1(S[i], S0[i], G[i], inv_prev, alpha);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

cudaError_t state_transfer(const Shape& s, float* S, float* S_start, float* grad_sum, int t,
                           float alpha, cudaStream_t st) {
    const int64_t n = (int64_t)s.B * s.H_kv * s.d * s.d;
    if (n == 0) return cudaSuccess;
    const float inv_prev = t > 1 ? 1.0f / (float)(t - 1) : 0.0f;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const bool vec = (n % 4 == 0) && aligned16(S) && aligned16(S_start) && aligned16(grad_sum);
    const int64_t items = vec ? n / 4 : n;
    const int64_t want = (items + 255) / 256;
    const int blocks = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
    if (vec)
        k_state_transfer4<<<blocks, 256, 0, st>>>(items, (float4*)S, (float4*)S_start,
                                                  (float4*)grad_sum, inv_prev, alpha);
    else
        k_state_transfer1<<<blocks, 256, 0, st>>>(items, S, S_start, grad_sum, inv_prev, alpha);
    return cudaGetLastError();
}

}  // namespace lisa
