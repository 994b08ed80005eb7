// C ABI of liblisa: argument validation, workspace layout and dispatch between
// the specialised sm_100a kernels and the generic kernels.
#include <math.h>
#include <string.h>

#include "lisa_internal.cuh"
#include "linear_decode.cuh"
#include "lisa_fast.cuh"

namespace lisa {

Shape resolve(const lisa_dims& d) {
    Shape s;
    s.B = d.B; s.T = d.T; s.n_past = d.n_past; s.N_max = d.N_max;
    s.H_q = d.H_q; s.H_kv = d.H_kv; s.d = d.d;
    s.H_I = d.H_I; s.H_Ik = d.H_Ik; s.d_I = d.d_I; s.M = d.M;
    s.chunk = d.chunk; s.dtype = d.act_dtype; s.phi = d.phi;
    s.L = d.n_past + d.T;
    s.group = d.H_kv > 0 ? d.H_q / d.H_kv : 0;
    s.sm_scale = d.sm_scale > 0.0f ? d.sm_scale : 1.0f / sqrtf((float)d.d);
    return s;
}

namespace {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

lisa_status check_dims(const lisa_dims* dp) {
    if (!dp) return LISA_ERR_INVALID_ARG;
    const lisa_dims& d = *dp;
    if (d.B < 0 || d.T < 0 || d.n_past < 0 || d.N_max < 0) return LISA_ERR_INVALID_ARG;
    if (d.H_q <= 0 || d.H_kv <= 0 || d.d <= 0 || d.H_I <= 0 || d.H_Ik <= 0 || d.d_I <= 0)
        return LISA_ERR_INVALID_ARG;
    if (d.M <= 0) return LISA_ERR_INVALID_ARG;
    if (d.H_q % d.H_kv != 0) return LISA_ERR_INVALID_ARG;
    if (!(d.H_Ik == 1 || d.H_Ik == d.H_I)) return LISA_ERR_INVALID_ARG;
    if ((int64_t)d.n_past + d.T > d.N_max) return LISA_ERR_INVALID_ARG;
    if (d.act_dtype != LISA_F32 && d.act_dtype != LISA_BF16) return LISA_ERR_INVALID_ARG;
    if (d.phi != LISA_PHI_IDENTITY && d.phi != LISA_PHI_ELU1_NORM) return LISA_ERR_INVALID_ARG;
    if (!(d.sm_scale == d.sm_scale)) return LISA_ERR_INVALID_ARG;  // NaN
    if (d.d > 256 || d.d_I > 256 || d.H_q / d.H_kv > 32) return LISA_ERR_UNSUPPORTED;
    if ((int64_t)d.H_I * d.d_I > 8192) return LISA_ERR_UNSUPPORTED;
    return LISA_OK;
}

lisa_status check_w_stride(const lisa_dims& d, int64_t w_tok_stride) {
    return (w_tok_stride == 0 || w_tok_stride == d.H_I) ? LISA_OK : LISA_ERR_INVALID_ARG;
}

lisa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LISA_OK : LISA_ERR_CUDA; }

// Workspace layout of each operation (offsets from ws).
struct TopmWs { size_t scores, end; };
TopmWs topm_ws(const Shape& s) {
    TopmWs w;
    w.scores = kStatusBytes;
    w.end = w.scores + align256(sizeof(float) * (size_t)s.B * s.T * s.L);
    return w;
}

struct DecodeWs { size_t scores, idx, count, o_sp, o_lin, end; };
DecodeWs decode_ws(const Shape& s) {
    DecodeWs w;
    w.scores = decode_scratch_offset(s.B);  // after the state the fast paths keep between calls
    w.idx = w.scores + align256(sizeof(float) * (size_t)s.B * s.L);
    w.count = w.idx + align256(sizeof(int32_t) * (size_t)s.B * s.M);
    w.o_sp = w.count + align256(sizeof(int32_t) * (size_t)s.B);
    w.o_lin = w.o_sp + align256(sizeof(float) * (size_t)s.B * s.H_q * s.d);
    w.end = w.o_lin + align256(sizeof(float) * (size_t)s.B * s.H_q * s.d);
    return w;
}

size_t workspace_bytes(const Shape& s, int op);

// Whole-module prefill: the sub-operations run one after another on the
// stream and share [status | scratch]; the intermediates follow the scratch.
struct PrefillWs { size_t scratch_end, idx, count, o_sp, o_lin, end; };
PrefillWs prefill_ws(const Shape& s) {
    PrefillWs w;
    size_t scratch = workspace_bytes(s, LISA_OP_TOPM);
    const size_t lin = workspace_bytes(s, LISA_OP_LINEAR_PREFILL);
    const size_t att = workspace_bytes(s, LISA_OP_SPARSE_ATTN);
    if (lin > scratch) scratch = lin;
    if (att > scratch) scratch = att;
    const size_t esz = s.dtype == LISA_BF16 ? 2 : 4;
    w.scratch_end = align256(scratch);
    w.idx = w.scratch_end;
    w.count = w.idx + align256(sizeof(int32_t) * (size_t)s.B * s.T * s.M);
    w.o_sp = w.count + align256(sizeof(int32_t) * (size_t)s.B * s.T);
    w.o_lin = w.o_sp + align256(esz * (size_t)s.B * s.T * s.H_q * s.d);
    w.end = w.o_lin + align256(esz * (size_t)s.B * s.T * s.H_q * s.d);
    return w;
}

lisa_status check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (!ws) return LISA_ERR_WORKSPACE;
    if (((uintptr_t)ws & 255) != 0) return LISA_ERR_WORKSPACE;
    if (ws_bytes < need) return LISA_ERR_WORKSPACE;
    return LISA_OK;
}

size_t workspace_bytes(const Shape& s, int op) {
    switch (op) {
        case LISA_OP_TOPM: {
            size_t need = topm_ws(s).end;
            size_t fast = fast_topm_ws_bytes(s);
            return need > fast ? need : fast;
        }
        case LISA_OP_SPARSE_ATTN:
        case LISA_OP_DENSE_ATTN: {
            size_t fast = fast_attention_ws_bytes(s, op == LISA_OP_DENSE_ATTN);
            return kStatusBytes > fast ? kStatusBytes : fast;
        }
        case LISA_OP_LINEAR_PREFILL: {
            size_t fast = fast_linear_prefill_ws_bytes(s);
            return kStatusBytes > fast ? kStatusBytes : fast;
        }
        case LISA_OP_DECODE_STEP: {
            size_t need = decode_ws(s).end;
            size_t fast = fast_decode_ws_bytes(s);
            return need > fast ? need : fast;
        }
        case LISA_OP_PREFILL: return prefill_ws(s).end;
        case LISA_OP_GATE_CHANNEL: return kStatusBytes;
        default: return 0;
    }
}

#define LISA_TRY(expr)                          \
    do {                                        \
        lisa_status _st = (expr);               \
        if (_st != LISA_OK) return _st;         \
    } while (0)

#define LISA_CUDA(expr)                         \
    do {                                        \
        cudaError_t _e = (expr);                \
        if (_e != cudaSuccess) return LISA_ERR_CUDA; \
    } while (0)

}  // namespace
}  // namespace lisa

using namespace lisa;

extern "C" {

lisa_status lisa_workspace_size(const lisa_dims* dims, int op, size_t* bytes) {
    LISA_TRY(check_dims(dims));
    if (!bytes) return LISA_ERR_INVALID_ARG;
    if (op < LISA_OP_TOPM || op > LISA_OP_GATE_CHANNEL) return LISA_ERR_INVALID_ARG;
    *bytes = workspace_bytes(resolve(*dims), op);
    return LISA_OK;
}

lisa_status lisa_index_scores(const lisa_dims* dims, const void* q_I, const void* k_I_cache,
                              const float* w, int64_t w_tok_stride, float* scores,
                              void* stream) {
    LISA_TRY(check_dims(dims));
    LISA_TRY(check_w_stride(*dims, w_tok_stride));
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!q_I || !k_I_cache || !w || !scores) return LISA_ERR_INVALID_ARG;
    return cuda_status(generic_index_scores(s, q_I, k_I_cache, w, w_tok_stride, scores,
                                            (cudaStream_t)stream));
}

lisa_status lisa_topm(const lisa_dims* dims, const void* q_I, const void* k_I_cache,
                      const float* w, int64_t w_tok_stride, int32_t* idx, int32_t* count,
                      void* ws, size_t ws_bytes, void* stream) {
    LISA_TRY(check_dims(dims));
    LISA_TRY(check_w_stride(*dims, w_tok_stride));
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!q_I || !k_I_cache || !w || !idx || !count) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_ws(ws, ws_bytes, workspace_bytes(s, LISA_OP_TOPM)));
    cudaStream_t st = (cudaStream_t)stream;
    if (fast_topm_supported(s, q_I, k_I_cache, w, w_tok_stride))
        return cuda_status(fast_topm(s, q_I, k_I_cache, w, w_tok_stride, idx, count, ws, st));
    const TopmWs lay = topm_ws(s);
    float* scores = (float*)((char*)ws + lay.scores);
    LISA_CUDA(generic_index_scores(s, q_I, k_I_cache, w, w_tok_stride, scores, st));
    return cuda_status(generic_topm_from_scores(s, scores, idx, count, st));
}

lisa_status lisa_sparse_attn(const lisa_dims* dims, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* idx, const int32_t* count,
                             void* o_sparse, void* ws, size_t ws_bytes, void* stream) {
    LISA_TRY(check_dims(dims));
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!q || !k_cache || !v_cache || !idx || !count || !o_sparse) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_ws(ws, ws_bytes, workspace_bytes(s, LISA_OP_SPARSE_ATTN)));
    cudaStream_t st = (cudaStream_t)stream;
    unsigned* status = (unsigned*)ws;
    if (fast_attention_supported(s, q, k_cache, v_cache, false))
        return cuda_status(fast_attention(s, q, k_cache, v_cache, idx, count, o_sparse, ws, st));
    return cuda_status(generic_attention(s, q, k_cache, v_cache, idx, count, o_sparse, false,
                                         status, st));
}

lisa_status lisa_dense_attn(const lisa_dims* dims, const void* q, const void* k_cache,
                            const void* v_cache, void* o, void* ws, size_t ws_bytes,
                            void* stream) {
    LISA_TRY(check_dims(dims));
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!q || !k_cache || !v_cache || !o) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_ws(ws, ws_bytes, workspace_bytes(s, LISA_OP_DENSE_ATTN)));
    cudaStream_t st = (cudaStream_t)stream;
    if (fast_attention_supported(s, q, k_cache, v_cache, true))
        return cuda_status(fast_attention(s, q, k_cache, v_cache, nullptr, nullptr, o, ws, st));
    return cuda_status(generic_attention(s, q, k_cache, v_cache, nullptr, nullptr, o, false,
                                         (unsigned*)ws, st));
}

lisa_status lisa_linear_prefill(const lisa_dims* dims, const void* q_L, const void* k_L,
                                const void* v_L, float* S, float* z, void* o_lin, void* ws,
                                size_t ws_bytes, void* stream) {
    LISA_TRY(check_dims(dims));
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!q_L || !k_L || !v_L || !S || !o_lin) return LISA_ERR_INVALID_ARG;
    if (s.phi == LISA_PHI_ELU1_NORM && !z) return LISA_ERR_INVALID_ARG;
    if (s.chunk <= 0) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_ws(ws, ws_bytes, workspace_bytes(s, LISA_OP_LINEAR_PREFILL)));
    cudaStream_t st = (cudaStream_t)stream;
    if (fast_linear_prefill_supported(s, q_L, k_L, v_L))
        return cuda_status(fast_linear_prefill(s, q_L, k_L, v_L, S, z, o_lin, ws, st));
    return cuda_status(generic_linear(s, q_L, k_L, v_L, S, z, o_lin, false, st));
}

lisa_status lisa_linear_decode(const lisa_dims* dims, const void* q_L, const void* k_L,
                               const void* v_L, float* S, float* z, void* o_lin, void* stream) {
    LISA_TRY(check_dims(dims));
    if (dims->T != 1) return LISA_ERR_INVALID_ARG;
    const Shape s = resolve(*dims);
    if (s.B == 0) return LISA_OK;
    if (!q_L || !k_L || !v_L || !S || !o_lin) return LISA_ERR_INVALID_ARG;
    if (s.phi == LISA_PHI_ELU1_NORM && !z) return LISA_ERR_INVALID_ARG;
    if (fast_linear_decode_supported(s, q_L, k_L, v_L, S))
        return cuda_status(fast_linear_decode(s, q_L, k_L, v_L, S, z, o_lin, (cudaStream_t)stream));
    return cuda_status(generic_linear(s, q_L, k_L, v_L, S, z, o_lin, false, (cudaStream_t)stream));
}

lisa_status lisa_gate_fuse(const lisa_dims* dims, const void* gate_logit_lin, const void* o_lin,
                           const void* o_sparse, void* o, void* stream) {
    LISA_TRY(check_dims(dims));
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!gate_logit_lin || !o_lin || !o_sparse || !o) return LISA_ERR_INVALID_ARG;
    if (fast_gate_supported(s, o_lin, o_sparse, o))
        return cuda_status(fast_gate(s, gate_logit_lin, o_lin, o_sparse, o, (cudaStream_t)stream));
    return cuda_status(generic_gate(s, gate_logit_lin, o_lin, false, o_sparse, false, o,
                                    (cudaStream_t)stream));
}

lisa_status lisa_decode_step(const lisa_dims* dims, const lisa_decode_args* a, void* ws,
                             size_t ws_bytes, void* stream) {
    LISA_TRY(check_dims(dims));
    if (dims->T != 1 || !a) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_w_stride(*dims, a->w_tok_stride));
    const Shape s = resolve(*dims);
    if (s.B == 0) return LISA_OK;
    if (!a->q || !a->k_new || !a->v_new || !a->q_I || !a->k_I_new || !a->w || !a->q_L ||
        !a->k_L || !a->v_L || !a->gate_logit_lin || !a->k_cache || !a->v_cache ||
        !a->k_I_cache || !a->S || !a->o)
        return LISA_ERR_INVALID_ARG;
    if (s.phi == LISA_PHI_ELU1_NORM && !a->z) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_ws(ws, ws_bytes, workspace_bytes(s, LISA_OP_DECODE_STEP)));
    cudaStream_t st = (cudaStream_t)stream;
    if (fast_decode_supported(s, *a)) return cuda_status(fast_decode_step(s, *a, ws, st));

    const DecodeWs lay = decode_ws(s);
    char* base = (char*)ws;
    float* scores = (float*)(base + lay.scores);
    int32_t* idx = a->idx ? a->idx : (int32_t*)(base + lay.idx);
    int32_t* count = a->count ? a->count : (int32_t*)(base + lay.count);
    float* o_sp = (float*)(base + lay.o_sp);
    float* o_lin = (float*)(base + lay.o_lin);
    LISA_CUDA(generic_append(s, a->k_new, a->v_new, a->k_I_new, a->k_cache, a->v_cache,
                             a->k_I_cache, st));
    LISA_CUDA(generic_linear(s, a->q_L, a->k_L, a->v_L, a->S, a->z, o_lin, true, st));
    LISA_CUDA(generic_index_scores(s, a->q_I, a->k_I_cache, a->w, a->w_tok_stride, scores, st));
    LISA_CUDA(generic_topm_from_scores(s, scores, idx, count, st));
    LISA_CUDA(generic_attention(s, a->q, a->k_cache, a->v_cache, idx, count, o_sp, true,
                                (unsigned*)ws, st));
    return cuda_status(generic_gate(s, a->gate_logit_lin, o_lin, true, o_sp, true, a->o, st));
}

lisa_status lisa_prefill(const lisa_dims* dims, const lisa_prefill_args* a, void* ws,
                         size_t ws_bytes, void* stream) {
    LISA_TRY(check_dims(dims));
    if (!a) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_w_stride(*dims, a->w_tok_stride));
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!a->q || !a->k_cache || !a->v_cache || !a->q_I || !a->k_I_cache || !a->w || !a->q_L ||
        !a->k_L || !a->v_L || !a->gate_logit_lin || !a->S || !a->o)
        return LISA_ERR_INVALID_ARG;
    if (s.phi == LISA_PHI_ELU1_NORM && !a->z) return LISA_ERR_INVALID_ARG;
    if (s.chunk <= 0) return LISA_ERR_INVALID_ARG;
    const PrefillWs lay = prefill_ws(s);
    LISA_TRY(check_ws(ws, ws_bytes, lay.end));
    char* base = (char*)ws;
    int32_t* idx = a->idx ? a->idx : (int32_t*)(base + lay.idx);
    int32_t* count = a->count ? a->count : (int32_t*)(base + lay.count);
    void* o_sp = base + lay.o_sp;
    void* o_lin = base + lay.o_lin;
    // the sub-operations see [status | scratch] as their own workspace
    LISA_TRY(lisa_topm(dims, a->q_I, a->k_I_cache, a->w, a->w_tok_stride, idx, count, ws,
                       lay.scratch_end, stream));
    LISA_TRY(lisa_sparse_attn(dims, a->q, a->k_cache, a->v_cache, idx, count, o_sp, ws,
                              lay.scratch_end, stream));
    LISA_TRY(lisa_linear_prefill(dims, a->q_L, a->k_L, a->v_L, a->S, a->z, o_lin, ws,
                                 lay.scratch_end, stream));
    return lisa_gate_fuse(dims, a->gate_logit_lin, o_lin, o_sp, a->o, stream);
}

lisa_status lisa_window_indices(const lisa_dims* dims, int32_t* idx, int32_t* count, void* stream) {
    LISA_TRY(check_dims(dims));
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!idx || !count) return LISA_ERR_INVALID_ARG;
    return cuda_status(generic_window_indices(s, idx, count, (cudaStream_t)stream));
}

lisa_status lisa_decode_step_window(const lisa_dims* dims, const lisa_decode_args* a, void* ws,
                                    size_t ws_bytes, void* stream) {
    LISA_TRY(check_dims(dims));
    if (dims->T != 1 || !a) return LISA_ERR_INVALID_ARG;
    const Shape s = resolve(*dims);
    if (s.B == 0) return LISA_OK;
    if (!a->q || !a->k_new || !a->v_new || !a->q_L || !a->k_L || !a->v_L || !a->gate_logit_lin ||
        !a->k_cache || !a->v_cache || !a->S || !a->o)
        return LISA_ERR_INVALID_ARG;
    if (s.phi == LISA_PHI_ELU1_NORM && !a->z) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_ws(ws, ws_bytes, workspace_bytes(s, LISA_OP_DECODE_STEP)));
    cudaStream_t st = (cudaStream_t)stream;
    if (fast_decode_supported(s, *a, true)) return cuda_status(fast_decode_step(s, *a, ws, st, true));

    const DecodeWs lay = decode_ws(s);
    char* base = (char*)ws;
    int32_t* idx = a->idx ? a->idx : (int32_t*)(base + lay.idx);
    int32_t* count = a->count ? a->count : (int32_t*)(base + lay.count);
    float* o_sp = (float*)(base + lay.o_sp);
    float* o_lin = (float*)(base + lay.o_lin);
    LISA_CUDA(generic_append(s, a->k_new, a->v_new, nullptr, a->k_cache, a->v_cache, nullptr, st));
    LISA_CUDA(generic_linear(s, a->q_L, a->k_L, a->v_L, a->S, a->z, o_lin, true, st));
    LISA_CUDA(generic_window_indices(s, idx, count, st));
    LISA_CUDA(generic_attention(s, a->q, a->k_cache, a->v_cache, idx, count, o_sp, true,
                                (unsigned*)ws, st));
    return cuda_status(generic_gate(s, a->gate_logit_lin, o_lin, true, o_sp, true, a->o, st));
}

lisa_status lisa_state_transfer(const lisa_dims* dims, float* S, float* S_start, float* grad_sum,
                                int32_t t, float alpha, void* stream) {
    LISA_TRY(check_dims(dims));
    if (t < 1 || !(alpha == alpha)) return LISA_ERR_INVALID_ARG;
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.H_kv == 0) return LISA_OK;
    if (!S || !S_start || !grad_sum) return LISA_ERR_INVALID_ARG;
    return cuda_status(state_transfer(s, S, S_start, grad_sum, t, alpha, (cudaStream_t)stream));
}

lisa_status lisa_gate_channel(const lisa_dims* dims, int32_t D_h, const void* h, const void* W_g,
                              const void* o_lin, const void* o_sparse, void* o, void* ws,
                              size_t ws_bytes, void* stream) {
    LISA_TRY(check_dims(dims));
    if (D_h < 1) return LISA_ERR_INVALID_ARG;
    const Shape s = resolve(*dims);
    if ((int64_t)s.B * s.T == 0) return LISA_OK;
    if (!h || !W_g || !o_lin || !o_sparse || !o) return LISA_ERR_INVALID_ARG;
    LISA_TRY(check_ws(ws, ws_bytes, kStatusBytes));
    cudaStream_t st = (cudaStream_t)stream;
    if (fast_gate_channel_supported(s, D_h, h, W_g, o_lin, o_sparse, o))
        return cuda_status(fast_gate_channel(s, D_h, h, W_g, o_lin, o_sparse, o, ws, st));
    return cuda_status(generic_gate_channel(s, D_h, h, W_g, o_lin, o_sparse, o, st));
}

lisa_status lisa_check_status(void* ws, void* stream) {
    if (!ws) return LISA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned host = 0;
    if (cudaMemcpyAsync(&host, ws, sizeof(unsigned), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return LISA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return LISA_ERR_CUDA;
    if (host != 0) {
        const unsigned zero = 0;
        if (cudaMemcpyAsync(ws, &zero, sizeof(unsigned), cudaMemcpyHostToDevice, st) != cudaSuccess)
            return LISA_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return LISA_ERR_CUDA;
    }
    switch (host) {
        case 0: return LISA_OK;
        case kDevTimeout: return LISA_ERR_TIMEOUT;
        case kDevBounds: return LISA_ERR_DEVICE_BOUNDS;
        default: return LISA_ERR_CUDA;
    }
}

const char* lisa_status_string(lisa_status st) {
    switch (st) {
        case LISA_OK: return "ok";
        case LISA_ERR_INVALID_ARG: return "invalid argument";
        case LISA_ERR_UNSUPPORTED: return "unsupported size";
        case LISA_ERR_CUDA: return "CUDA error";
        case LISA_ERR_TIMEOUT: return "device wait timed out";
        case LISA_ERR_DEVICE_BOUNDS: return "device index out of bounds (skipped)";
        case LISA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        default: return "unknown status";
    }
}

const char* lisa_version(void) { return "liblisa 0.1.0 sm_100a"; }

}  // extern "C"
