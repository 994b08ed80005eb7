// Specialised paths not yet available: every predicate declines.
#include "lisa_fast.cuh"

namespace lisa {


size_t fast_attention_ws_bytes(const Shape&, bool) { return 0; }
bool fast_attention_supported(const Shape&, const void*, const void*, const void*, bool) { return false; }
cudaError_t fast_attention(const Shape&, const void*, const void*, const void*, const int32_t*,
                           const int32_t*, void*, void*, cudaStream_t) { return cudaErrorNotSupported; }

size_t fast_linear_prefill_ws_bytes(const Shape&) { return 0; }
bool fast_linear_prefill_supported(const Shape&, const void*, const void*, const void*) { return false; }
cudaError_t fast_linear_prefill(const Shape&, const void*, const void*, const void*, float*, float*,
                                void*, void*, cudaStream_t) { return cudaErrorNotSupported; }


}  // namespace lisa
