/*
 * liblisa — forward pass of the LISA attention module on NVIDIA B200 (sm_100a).
 *
 * Source of the operations: "LISA: Linear-Indexed Sparse Attention for Efficient
 * Long-Context Reasoning" (arXiv 2607.19358v1).  The module has two branches joined
 * by a gate (Sec. 3.2, Eq. 1):
 *   o = g * o_LA + (1 - g) * o_SA_M,        g = sigmoid(gate_logit_lin)
 * o_SA_M is softmax attention over the M cached positions chosen by the Lightning
 * Indexer (Sec. 3.2, "Indexer-Guided Token Selection"); o_LA is linear attention
 * over the whole prefix (Sec. 3.1, "Linear Attention"; Sec. 3.3, Eq. 3-4).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is DEVICE memory owned by the caller.  The library
 *    allocates no device memory and keeps no state between calls: all
 *    persistent state (K/V caches, indexer-key cache, linear state S and z) is
 *    passed in.  Calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and never synchronise, except lisa_check_status.
 *  - Layouts are row-major and contiguous (innermost dimension last):
 *      q, q_L, o, o_sparse, o_lin  [B, T, H_q, d]
 *      k_cache, v_cache            [B, N_max, H_kv, d]     (position s of sequence b)
 *      k_L, v_L                    [B, T, H_kv, d]
 *      q_I                         [B, T, H_I, d_I]
 *      k_I_cache                   [B, N_max, H_Ik, d_I]
 *      w (float32)                 [B, T, H_I] if w_tok_stride == H_I,
 *                                  [B, H_I]    if w_tok_stride == 0 (same weights for every token)
 *      gate_logit_lin              [B, T, H_q]
 *      idx (int32)                 [B, T, M]   selected positions, ascending, padded with -1
 *      count (int32)               [B, T]      number of valid entries of idx = min(M, p+1)
 *      S (float32)                 [B, H_kv, d, d]  row = key feature, column = value feature
 *      z (float32)                 [B, H_kv, d]     elu+1 normaliser state (NULL for identity)
 *      scores (float32)            [B, T, n_past+T]
 *    Activation tensors (q, k, v, q_I, k_I, q_L, k_L, v_L, gate logits, outputs)
 *    have the element type dims->act_dtype (float32 or bfloat16).
 *  - Query token t of a call sits at absolute position p = n_past + t.  It
 *    selects among cached positions s in [0, p], itself included (Sec. 3.2:
 *    the indexer scores the context, the selected rows are attended); fewer
 *    than M candidates selects all of them.  Ties in the indexer score keep the
 *    lower position.  One selection per (sequence, token) is shared by all heads.
 *  - GQA: query head h reads KV head h / (H_q / H_kv) in both branches.
 *  - Return value: LISA_OK, or an error detected on the host before anything is
 *    launched (invalid argument, unsupported shape, too small a workspace, CUDA
 *    launch error).  Errors found by a kernel while it runs (an index outside
 *    [0, p], a bounded wait that gave up) are recorded in the status word at the
 *    start of the workspace and returned by lisa_check_status.  The library
 *    never aborts, traps or prints.
 *  - Workspace: entry points that take `ws` need at least lisa_workspace_size()
 *    bytes of device memory, 256-byte aligned, ZERO-FILLED when allocated.  The
 *    first 256 bytes are a header: 32-bit word 0 is the status word, words 2-3
 *    a fault-injection hook for tests (keep them zero: a non-zero word 2 makes
 *    the decode step leave out one exchange arrival on purpose), the rest is
 *    reserved.  A workspace must not be shared by calls that may run
 *    concurrently.  Every entry point other than the decode steps uses the rest
 *    as scratch that it initialises itself.  The decode steps
 *    (lisa_decode_step, lisa_decode_step_window) instead keep state between
 *    calls in their workspace (key histograms and exchange counters, all zero
 *    again when a call ends) at offsets that depend on B only: one workspace,
 *    sized for the largest context, serves a batch as its context grows.
 *    Zero-fill a workspace again before a decode step uses it when another
 *    entry point has used it since, when B has changed, or when
 *    lisa_check_status has returned LISA_ERR_TIMEOUT.
 */
#ifndef LISA_H_
#define LISA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LISA_API __attribute__((visibility("default")))
#else
#define LISA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lisa_status {
    LISA_OK = 0,
    LISA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, inconsistent dims      */
    LISA_ERR_UNSUPPORTED = 2,   /* a size beyond the compiled limits (see lisa_dims)   */
    LISA_ERR_CUDA = 3,          /* a CUDA call or kernel launch failed                 */
    LISA_ERR_TIMEOUT = 4,       /* device: a bounded wait gave up (from the status word)*/
    LISA_ERR_DEVICE_BOUNDS = 5, /* device: an index outside [0, p] was skipped          */
    LISA_ERR_WORKSPACE = 6      /* workspace missing, misaligned or too small           */
} lisa_status;

typedef enum lisa_dtype { LISA_F32 = 0, LISA_BF16 = 1 } lisa_dtype;

typedef enum lisa_phi {
    LISA_PHI_IDENTITY = 0,  /* phi(x) = x, no normaliser (Sec. 3.1, the paper's choice) */
    LISA_PHI_ELU1_NORM = 1  /* phi(x) = elu(x) + 1, o = phi(q) S / (phi(q) . z)          */
} lisa_phi;

/* Sizes of one call.  Limits: d <= 256 and d_I <= 256; H_q % H_kv == 0;
 * H_I % H_Ik == 0 with H_Ik in {1, H_I}; H_q/H_kv <= 32; n_past + T <= N_max. */
typedef struct lisa_dims {
    int32_t B;          /* batch (sequences)                                        */
    int32_t T;          /* query tokens in this call, positions n_past .. n_past+T-1 */
    int32_t n_past;     /* tokens cached before this call's first token              */
    int32_t N_max;      /* cache capacity in tokens (batch stride of the caches)     */
    int32_t H_q;        /* query heads                                              */
    int32_t H_kv;       /* key/value heads                                          */
    int32_t d;          /* head dimension                                           */
    int32_t H_I;        /* indexer query heads                                      */
    int32_t H_Ik;       /* indexer key heads: 1 (shared key) or H_I (own key per head) */
    int32_t d_I;        /* indexer dimension                                        */
    int32_t M;          /* top-M budget (>= 1)                                      */
    int32_t chunk;      /* linear-attention chunk length in prefill (rounding only)  */
    int32_t act_dtype;  /* lisa_dtype of the activation tensors                     */
    int32_t phi;        /* lisa_phi                                                 */
    float sm_scale;     /* softmax scale of the sparse branch; <= 0 means 1/sqrt(d)   */
} lisa_dims;

/* Operation codes for lisa_workspace_size. */
typedef enum lisa_op {
    LISA_OP_TOPM = 0,
    LISA_OP_SPARSE_ATTN = 1,
    LISA_OP_LINEAR_PREFILL = 2,
    LISA_OP_DECODE_STEP = 3,
    LISA_OP_DENSE_ATTN = 4,
    LISA_OP_PREFILL = 5,
    LISA_OP_GATE_CHANNEL = 6
} lisa_op;

/* Lightning Indexer scores (Sec. 3.2; the per-head score vector defined under
 * Eq. 2, summed over the indexer heads):
 *   scores[b,t,s] = sum_j w[b,t,j] * ReLU(<q_I[b,t,j,:], k_I_cache[b,s,j mod H_Ik,:]>)
 * for s <= p; entries s > p are written as -infinity.  Materialises
 * B*T*(n_past+T) floats: meant for tests and short contexts.  k_I_cache must
 * hold positions [0, n_past+T). */
LISA_API lisa_status lisa_index_scores(const lisa_dims* dims, const void* q_I, const void* k_I_cache,
                              const float* w, int64_t w_tok_stride, float* scores,
                              void* stream);

/* Indexer scores followed by top-M selection (Sec. 3.2: the M positions with the
 * highest summed score are kept), without materialising the scores for the caller.
 * Writes idx [B,T,M] (ascending positions, -1 padded) and count [B,T]. */
LISA_API lisa_status lisa_topm(const lisa_dims* dims, const void* q_I, const void* k_I_cache,
                      const float* w, int64_t w_tok_stride, int32_t* idx, int32_t* count,
                      void* ws, size_t ws_bytes, void* stream);

/* Sparse softmax attention SA_M (Sec. 3.2, Eq. 1) of each query head over the
 * count[b,t] positions in idx[b,t,:] (any order; entries past count ignored):
 *   o_sparse[h] = softmax_s(sm_scale * <q[h], K[s,g]>) . V[s,g],  g = h / (H_q/H_kv)
 * The positions of a row are a set: they must be distinct (lisa_topm and
 * lisa_window_indices write distinct positions); a repeated position may
 * count once or twice.  Positions outside [0, p] are skipped and reported as
 * LISA_ERR_DEVICE_BOUNDS through the status word.  count == 0 gives a zero
 * output.  Calls whose rows keep a sizeable share of their causal range (a
 * prefill) run as masked tensor-core tiles over the key tiles the rows select
 * from; others gather each selected row.  Workspace:
 * lisa_workspace_size(.., LISA_OP_SPARSE_ATTN) (the selection mask, about
 * B*T*(n_past+T)/8 bytes, for the first form). */
LISA_API lisa_status lisa_sparse_attn(const lisa_dims* dims, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* idx, const int32_t* count,
                             void* o_sparse, void* ws, size_t ws_bytes, void* stream);

/* Linear attention over the T tokens of a call, chunked-parallel form of the
 * recurrence of Sec. 3.1 / Sec. 3.3 Eq. 3-4 (inclusive of the current token):
 *   S <- S + phi(k_L[t])^T v_L[t];  z <- z + phi(k_L[t]);  o_lin[t,h] = phi(q_L[t,h]) S
 *   (elu+1 mode: divided by phi(q_L[t,h]) . z).
 * S (and z) hold the state before token 0 on entry and after token T-1 on
 * return.  dims->chunk sets the chunk length (it changes rounding only). */
LISA_API lisa_status lisa_linear_prefill(const lisa_dims* dims, const void* q_L, const void* k_L,
                                const void* v_L, float* S, float* z, void* o_lin,
                                void* ws, size_t ws_bytes, void* stream);

/* One recurrent step of the same linear attention (T must be 1). */
LISA_API lisa_status lisa_linear_decode(const lisa_dims* dims, const void* q_L, const void* k_L,
                               const void* v_L, float* S, float* z, void* o_lin, void* stream);

/* Gate (Sec. 3.2, Eq. 1): o = g * o_lin + (1 - g) * o_sparse, g = sigmoid(gate_logit_lin),
 * one logit per (token, query head). */
LISA_API lisa_status lisa_gate_fuse(const lisa_dims* dims, const void* gate_logit_lin, const void* o_lin,
                           const void* o_sparse, void* o, void* stream);

/* Arguments of one fused decode step (T == 1).  All device pointers. */
typedef struct lisa_decode_args {
    const void* q;               /* [B,1,H_q,d]                                       */
    const void* k_new;           /* [B,1,H_kv,d]   appended to k_cache at n_past        */
    const void* v_new;           /* [B,1,H_kv,d]   appended to v_cache at n_past        */
    const void* q_I;             /* [B,1,H_I,d_I]                                     */
    const void* k_I_new;         /* [B,1,H_Ik,d_I] appended to k_I_cache at n_past      */
    const float* w;              /* indexer weights, see w_tok_stride                  */
    int64_t w_tok_stride;        /* 0 or H_I                                          */
    const void* q_L;             /* [B,1,H_q,d]    linear-branch query                  */
    const void* k_L;             /* [B,1,H_kv,d]   linear-branch key                    */
    const void* v_L;             /* [B,1,H_kv,d]   linear-branch value                  */
    const void* gate_logit_lin;  /* [B,1,H_q]                                         */
    void* k_cache;               /* [B,N_max,H_kv,d]   in/out                          */
    void* v_cache;               /* [B,N_max,H_kv,d]   in/out                          */
    void* k_I_cache;             /* [B,N_max,H_Ik,d_I] in/out                          */
    float* S;                    /* [B,H_kv,d,d]   in/out                               */
    float* z;                    /* [B,H_kv,d]     in/out, NULL unless ELU1_NORM         */
    void* o;                     /* [B,1,H_q,d]    output                               */
    int32_t* idx;                /* [B,1,M]  optional output (NULL: not written)       */
    int32_t* count;              /* [B,1]    optional output (NULL: not written)       */
} lisa_decode_args;

/* One decode step of the whole module (Sec. 3.2, the generation step): append
 * the new token's k, v and k_I at position p = n_past; update the linear state
 * and read it out; score all p+1 cached keys with the indexer, keep the top M,
 * attend over them; gate the two branches into o.  T must be 1. */
LISA_API lisa_status lisa_decode_step(const lisa_dims* dims, const lisa_decode_args* args, void* ws,
                             size_t ws_bytes, void* stream);

/* Arguments of a whole-module prefill over the T tokens of a call.  All device
 * pointers.  The caches must already hold positions [0, n_past + T). */
typedef struct lisa_prefill_args {
    const void* q;               /* [B,T,H_q,d]                                       */
    const void* k_cache;         /* [B,N_max,H_kv,d]                                  */
    const void* v_cache;         /* [B,N_max,H_kv,d]                                  */
    const void* q_I;             /* [B,T,H_I,d_I]                                     */
    const void* k_I_cache;       /* [B,N_max,H_Ik,d_I]                                */
    const float* w;              /* indexer weights, see w_tok_stride                  */
    int64_t w_tok_stride;        /* 0 or H_I                                          */
    const void* q_L;             /* [B,T,H_q,d]                                       */
    const void* k_L;             /* [B,T,H_kv,d]                                      */
    const void* v_L;             /* [B,T,H_kv,d]                                      */
    const void* gate_logit_lin;  /* [B,T,H_q]                                         */
    float* S;                    /* [B,H_kv,d,d]  in: state before token 0, out: after  */
    float* z;                    /* [B,H_kv,d]    in/out, NULL unless ELU1_NORM         */
    void* o;                     /* [B,T,H_q,d]   output                               */
    int32_t* idx;                /* [B,T,M] optional output (NULL: kept in workspace)  */
    int32_t* count;              /* [B,T]   optional output                            */
} lisa_prefill_args;

/* The whole module over the T tokens of a call (Sec. 3.2 Eq. 1): indexer scores
 * and top-M of every token, sparse attention over the selected rows, the
 * linear branch in chunked form (advancing S and z), and the gate.  Equivalent
 * to lisa_topm, lisa_sparse_attn, lisa_linear_prefill and lisa_gate_fuse in a
 * row; intermediates live in the workspace (LISA_OP_PREFILL). */
LISA_API lisa_status lisa_prefill(const lisa_dims* dims, const lisa_prefill_args* args, void* ws,
                                  size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Beyond the main path: the Stage-1 sparse branch and the segment state update.
 * ------------------------------------------------------------------------- */

/* Sliding-window index rows (LISA Sec. 3.2, Stage 1, the branch the Indexer
 * later replaces): token t at position p = n_past + t keeps the positions
 * [max(0, p-M+1), p] in ascending order.  Same outputs and layout as
 * lisa_topm (idx [B,T,M] int32, -1 padded; count [B,T] = min(M, p+1)); feed
 * them to lisa_sparse_attn.  Uses B, T, n_past and M of dims. */
LISA_API lisa_status lisa_window_indices(const lisa_dims* dims, int32_t* idx, int32_t* count,
                                         void* stream);

/* One decode step of the module with the Stage-1 sparse branch: as
 * lisa_decode_step, but the sparse attention runs over the last min(M, n)
 * positions instead of the Indexer's top-M (LISA Sec. 3.2 Eq. 1 with o_SA_M the
 * sliding-window output).  q_I, k_I_new, k_I_cache and w are not used and may
 * be NULL; the k_I cache is not appended.  idx/count, when given, receive the
 * window.  Workspace: lisa_workspace_size(.., LISA_OP_DECODE_STEP). */
LISA_API lisa_status lisa_decode_step_window(const lisa_dims* dims, const lisa_decode_args* args,
                                             void* ws, size_t ws_bytes, void* stream);

/* Segment state transfer and correction at the end of reasoning segment t
 * (t >= 1; LISA Sec. 3.3, "Segment State Update", Eq. 6-9), for every state
 * matrix S[b, g]:
 *   grad_t   = S - S_start                           (Eq. 6, S_start = S_{t-1})
 *   mean     = grad_sum / (t - 1), zero when t = 1   (Eq. 7)
 *   grad_hat = (1 - alpha) grad_t + alpha mean       (Eq. 8)
 *   S_t      = S_start + grad_hat                    (Eq. 9)
 * In place, all fp32 [B, H_kv, d, d] device arrays: S (in: the state the
 * segment's tokens reached; out: S_t), S_start (in: S_{t-1}; out: S_t, the
 * start of the next segment), grad_sum (in: grad_1 + ... + grad_{t-1}, zeros
 * before the first segment; out: the sum through grad_t).  alpha is the
 * paper's correction coefficient (unstated there; a caller's parameter).
 * Applies to S only: the elu+1 normaliser z is left as the tokens made it.
 * Errors: LISA_ERR_INVALID_ARG for t < 1, a NaN alpha or a null pointer. */
LISA_API lisa_status lisa_state_transfer(const lisa_dims* dims, float* S, float* S_start,
                                         float* grad_sum, int32_t t, float alpha, void* stream);

/* Per-channel gate (LISA Sec. 3.3, Eq. 5) joining the branches as in Eq. 1:
 *   g[m][c] = sigmoid(sum_k W_g[c][k] h[m][k]),
 *   o[m][c] = g o_lin[m][c] + (1 - g) o_sparse[m][c]
 * for every token m of the B*T tokens and channel c of the H_q*d output
 * channels (query head major).  Device arrays of the activation type:
 * h [B,T,D_h] (the module's input hidden states), W_g [H_q*d, D_h] (row c is
 * channel c's gate weights), o_lin, o_sparse, o [B,T,H_q,d].  Nothing is
 * retained; o may alias neither input.  On bf16 with H_q*d a multiple of 256,
 * D_h a multiple of 64 and 16-byte aligned arrays the contraction runs on the
 * tensor cores (tiles of 128 tokens; fewer than 64 tokens take a kernel that
 * streams W_g once); every other size takes a plain kernel.
 * Workspace: lisa_workspace_size(.., LISA_OP_GATE_CHANNEL) (the status word).
 * Errors: LISA_ERR_INVALID_ARG for D_h < 1 or a null pointer; a device wait
 * that gives up is reported by lisa_check_status as LISA_ERR_TIMEOUT. */
LISA_API lisa_status lisa_gate_channel(const lisa_dims* dims, int32_t D_h, const void* h,
                                       const void* W_g, const void* o_lin, const void* o_sparse,
                                       void* o, void* ws, size_t ws_bytes, void* stream);

/* Dense causal softmax attention over every cached position s <= p (Sec. 3.1,
 * the standard attention LISA replaces); the O(n) reference line. */
LISA_API lisa_status lisa_dense_attn(const lisa_dims* dims, const void* q, const void* k_cache,
                            const void* v_cache, void* o, void* ws, size_t ws_bytes,
                            void* stream);

/* lisa_topm without a workspace, for callers that cannot allocate device memory
 * for the library (a host framework whose allocator is off-limits, plugin or
 * callback interfaces that pass only the call's tensors, loops where a
 * cudaMalloc and its device synchronisation are not acceptable).  The paper
 * has no counterpart: this is a packaging variant of lisa_topm.  Same inputs,
 * outputs and result as lisa_topm; the scores of the call are kept in a 4 MiB
 * device array built into the library, held on every GPU that loads it until
 * the process exits.
 *  - Calls needing more than 4 MiB of scores (B*T*(n_past+T) floats) return
 *    LISA_ERR_UNSUPPORTED without launching anything.
 *  - The array is shared by every call on a device and keeps the last call's
 *    contents; calls that may overlap on the GPU race on it, so the caller must
 *    order them (one stream, or explicit events).
 *  - The first call on each device sets up the array's device address (with
 *    that device current); make that first call before any stream capture. */
LISA_API lisa_status lisa_topm_noalloc(const lisa_dims* dims, const void* q_I, const void* k_I_cache,
                              const float* w, int64_t w_tok_stride, int32_t* idx, int32_t* count,
                              void* stream);

/* Workspace bytes needed by `op` for these dims (0 if none). */
LISA_API lisa_status lisa_workspace_size(const lisa_dims* dims, int op, size_t* bytes);

/* Synchronise `stream`, read and clear the status word of `ws`.  Returns
 * LISA_OK, LISA_ERR_TIMEOUT or LISA_ERR_DEVICE_BOUNDS (or LISA_ERR_CUDA if the
 * stream reported an error). */
LISA_API lisa_status lisa_check_status(void* ws, void* stream);

/* Static description of a status code. */
LISA_API const char* lisa_status_string(lisa_status status);

/* Library version string, e.g. "liblisa 0.1.0 sm_100a". */
LISA_API const char* lisa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LISA_H_ */
