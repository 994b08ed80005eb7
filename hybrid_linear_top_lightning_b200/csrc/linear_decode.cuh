// linear_decode.cu: one recurrent step of the linear branch on sm_100a (bf16,
// head dim 128, at most 8 query heads per KV head, 16-byte-aligned operands);
// lisa_linear_decode falls back to the generic kernel otherwise.
#pragma once

#include "lisa_internal.cuh"

namespace lisa {

bool fast_linear_decode_supported(const Shape& s, const void* q, const void* k, const void* v,
                                  const float* S);
cudaError_t fast_linear_decode(const Shape& s, const void* q, const void* k, const void* v, float* S,
                               float* z, void* o_lin, cudaStream_t st);

}  // namespace lisa
