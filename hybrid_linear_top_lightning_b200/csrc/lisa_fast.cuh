// Specialised sm_100a paths.  Each `*_supported` predicate says whether a call
// can take the specialised kernel (shape, dtype and pointer alignment); the
// API falls back to the generic kernels otherwise.
#pragma once

#include "lisa_internal.cuh"

namespace lisa {

// Decode-step workspaces start with state that is zero between calls, at
// offsets that depend on B only, so that one workspace serves a batch at every
// context length: [status | key histograms, B x 4096 u32 | second-digit
// histograms, B x 1024 u32 | barrier lines, B x 128 bytes | scratch of the call].
inline size_t decode_hist_offset() { return kStatusBytes; }
inline size_t decode_hist2_offset(int B) { return kStatusBytes + (size_t)B * 4096 * 4; }
inline size_t decode_sync_offset(int B) { return decode_hist2_offset(B) + (size_t)B * 1024 * 4; }
inline size_t decode_scratch_offset(int B) { return decode_sync_offset(B) + (size_t)B * 128; }

// Decode step: one cooperative kernel over all SMs (decode_coop.cu) when it
// covers the call, else the four-kernel form (decode_fused.cu).
size_t fast_decode_ws_bytes(const Shape& s);
// window: the sparse branch attends over the last M positions (no indexer)
bool fast_decode_supported(const Shape& s, const lisa_decode_args& a, bool window = false);
cudaError_t fast_decode_step(const Shape& s, const lisa_decode_args& a, void* ws, cudaStream_t st,
                             bool window = false);
size_t coop_decode_ws_bytes(const Shape& s);
bool coop_decode_supported(const Shape& s, const lisa_decode_args& a, bool window);
cudaError_t coop_decode_step(const Shape& s, const lisa_decode_args& a, void* ws, cudaStream_t st,
                             bool window);

// Top-M over many query rows (prefill).
size_t fast_topm_ws_bytes(const Shape& s);
bool fast_topm_supported(const Shape& s, const void* q_I, const void* k_I, const float* w,
                         int64_t w_tok_stride);
cudaError_t fast_topm(const Shape& s, const void* q_I, const void* k_I, const float* w,
                      int64_t w_tok_stride, int32_t* idx, int32_t* count, void* ws,
                      cudaStream_t st);

// Sparse / dense attention.
size_t fast_attention_ws_bytes(const Shape& s, bool dense);
bool fast_attention_supported(const Shape& s, const void* q, const void* k, const void* v,
                              bool dense);
cudaError_t fast_attention(const Shape& s, const void* q, const void* k, const void* v,
                           const int32_t* idx, const int32_t* count, void* o, void* ws,
                           cudaStream_t st);

// Sparse attention of many query rows through a bit mask of the selections and
// tcgen05 tiles (sparse_mask_tc.cu); fast_attention takes it when the rows keep
// a sizeable share of their causal range.
bool sparse_mask_preferred(const Shape& s);
size_t sparse_mask_ws_bytes(const Shape& s);
bool sparse_mask_supported(const Shape& s, const void* q, const void* k, const void* v);
cudaError_t sparse_mask_attention(const Shape& s, const void* q, const void* k, const void* v,
                                  const int32_t* idx, const int32_t* count, void* o, void* ws,
                                  cudaStream_t st);

// Chunked linear-attention prefill.
size_t fast_linear_prefill_ws_bytes(const Shape& s);
bool fast_linear_prefill_supported(const Shape& s, const void* q, const void* k, const void* v);
cudaError_t fast_linear_prefill(const Shape& s, const void* q, const void* k, const void* v,
                                float* S, float* z, void* o, void* ws, cudaStream_t st);


// gate_fast.cu: o = g o_lin + (1 - g) o_sparse for bf16 tensors, head dim 128
bool fast_gate_supported(const Shape& s, const void* o_lin, const void* o_sp, const void* o);
cudaError_t fast_gate(const Shape& s, const void* logit, const void* o_lin, const void* o_sp,
                      void* o, cudaStream_t st);


// state_transfer.cu: segment state correction (Sec. 3.3 Eq. 6-9), any shape
cudaError_t state_transfer(const Shape& s, float* S, float* S_start, float* grad_sum, int t,
                           float alpha, cudaStream_t st);


// gate_channel.cu: per-channel gate (Sec. 3.3 Eq. 5), bf16, N % 256 == 0, D_h % 64 == 0
bool fast_gate_channel_supported(const Shape& s, int D_h, const void* h, const void* W,
                                 const void* o_lin, const void* o_sp, const void* o);
cudaError_t generic_gate_channel(const Shape& s, int D_h, const void* h, const void* W,
                                 const void* o_lin, const void* o_sp, void* o, cudaStream_t st);
cudaError_t fast_gate_channel(const Shape& s, int D_h, const void* h, const void* W,
                              const void* o_lin, const void* o_sp, void* o, void* ws,
                              cudaStream_t st);

}  // namespace lisa
