// Internal declarations shared by the liblisa translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lisa.h"

namespace lisa {

// Status word at the start of a workspace; the rest of the first 256 bytes is reserved.
constexpr size_t kStatusBytes = 256;

// Device-side error codes written to the status word (first error wins).
enum DeviceError : unsigned { kDevOk = 0, kDevTimeout = 4, kDevBounds = 5 };

__device__ __forceinline__ void record_error(unsigned* status, unsigned code) {
    if (status) atomicCAS(status, 0u, code);
}

// Resolved sizes of one call.
struct Shape {
    int B, T, n_past, N_max, H_q, H_kv, d, H_I, H_Ik, d_I, M, chunk, dtype, phi;
    int L;        // n_past + T: cached positions visible to the last token
    int group;    // H_q / H_kv
    float sm_scale;
};

Shape resolve(const lisa_dims& d);

// Element access for the two activation types.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Total order on float scores used by top-M: larger key = larger score, with
// -0 and +0 made equal.  Keys of candidates are compared as unsigned integers.
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---- generic (any shape, fp32 or bf16) path: generic.cu -------------------
cudaError_t generic_index_scores(const Shape& s, const void* q_I, const void* k_I, const float* w,
                                 int64_t w_tok_stride, float* scores, cudaStream_t st);
cudaError_t generic_topm_from_scores(const Shape& s, const float* scores, int32_t* idx,
                                     int32_t* count, cudaStream_t st);
// Sparse (idx != nullptr) or dense causal (idx == nullptr) attention.  o is act
// dtype when o_f32 == false, float32 otherwise.
cudaError_t generic_attention(const Shape& s, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* idx, const int32_t* count,
                              void* o, bool o_f32, unsigned* status, cudaStream_t st);
cudaError_t generic_linear(const Shape& s, const void* q_L, const void* k_L, const void* v_L,
                           float* S, float* z, void* o, bool o_f32, cudaStream_t st);
// o = sigmoid(x) * o_lin + (1 - sigmoid(x)) * o_sp; branch inputs in act dtype or float32.
cudaError_t generic_gate(const Shape& s, const void* logit, const void* o_lin, bool lin_f32,
                         const void* o_sp, bool sp_f32, void* o, cudaStream_t st);
cudaError_t generic_window_indices(const Shape& s, int32_t* idx, int32_t* count, cudaStream_t st);
// k_I_new / k_I_cache may be null: only k and v are appended
cudaError_t generic_append(const Shape& s, const void* k_new, const void* v_new,
                           const void* k_I_new, void* k_cache, void* v_cache, void* k_I_cache,
                           cudaStream_t st);

}  // namespace lisa
