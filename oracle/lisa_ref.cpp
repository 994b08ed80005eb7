// CPU oracle for the forward pass of the LISA attention module.
//
// TEST INFRASTRUCTURE ONLY.  The tests, the package's smoke check and the
// benchmark's CPU-baseline leg load this library; the product library never
// does, and it shares no code, header, table or helper with it.
//
// Source: "LISA: Linear-Indexed Sparse Attention for Efficient Long-Context
// Reasoning" (arXiv 2607.19358v1, HTML version).  Each function restates one
// step of the method as plainly as possible, with fp64 arithmetic throughout.
// Inputs arrive as float32 arrays whose values are exactly the (bf16- or
// fp32-rounded) inputs of the GPU path; they are widened to double on read.
//
// Readings of points the paper leaves open (all recorded in the design notes):
//  * the gate weights the linear branch (Eq. 1: o = g*o_LA + (1-g)*o_SA_M) and
//    is one sigmoid scalar per (token, query head);
//  * indexer score = sum_j w_j * ReLU(<q_I[j], k_I[j mod H_Ik]>)  (H_Ik = H_I,
//    w = 1 is the paper's per-head-key form of Sec. 3.2; H_Ik = 1 with weights
//    is the shared-key weighted form);
//  * query position p selects among keys s in [0, p] (itself included); ties
//    are broken by the lower position; fewer than M candidates selects all;
//  * one index set per (sequence, token), shared by every query head;
//  * sparse softmax uses scale sm_scale (1/sqrt(d) unless told otherwise);
//  * linear attention is inclusive (Eq. 3-4 read with the current token's
//    k^T v added before read-out); phi = identity without normaliser
//    (Sec. 3.1), or phi = elu+1 with normaliser phi(q).z as an option;
//  * GQA: query head h reads KV head g = h / (H_q / H_kv), for both branches.
//
// Parity pins: brute force on tiny inputs, closed forms (dense causal softmax
// attention when M >= p+1, S_n = K^T V, the parallel masked form of linear
// attention), limits of the gate and hand-worked fixtures; see tests/.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

struct RefDims {
    int32_t B;       // batch
    int32_t T;       // query tokens; absolute positions n_past .. n_past+T-1
    int32_t n_past;  // tokens before the first query token
    int32_t N_max;   // cache capacity in tokens (batch stride of the caches)
    int32_t H_q;     // query heads
    int32_t H_kv;    // key/value heads
    int32_t d;       // head dimension
    int32_t H_I;     // indexer query heads
    int32_t H_Ik;    // indexer key heads (1 or H_I)
    int32_t d_I;     // indexer dimension
    int32_t M;       // top-M budget
    int32_t phi;     // 0: identity, no normaliser; 1: elu+1 with normaliser
    double sm_scale; // softmax scale of the sparse branch
};

int ref_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void ref_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

// Row r of a sampled call is query token rows[r] (rows == NULL: r itself).
static inline int row_token(const int32_t* rows, int r) { return rows ? rows[r] : r; }

// Indexer head weight w[b, t, j]: per token when w_tok_stride == H_I
// ([B, T, H_I]), per sequence when w_tok_stride == 0 ([B, H_I]).
static inline double weight_at(const RefDims* D, const float* w, int64_t w_tok_stride,
                               int b, int t, int j) {
    int64_t batch_stride = w_tok_stride ? (int64_t)D->T * w_tok_stride : D->H_I;
    return (double)w[b * batch_stride + (int64_t)t * w_tok_stride + j];
}

// ---------------------------------------------------------------------------
// Lightning Indexer score (Sec. 3.2, "Indexer-Guided Token Selection", and the
// score vector S^(j) defined under Eq. 2): for query position p = n_past + t
// and every key s <= p,
//     I[p, s] = sum_j w[t, j] * ReLU( <q_I[t, j, :], k_I[s, j mod H_Ik, :]> ).
// Entries s > p are not candidates and are written as -infinity.
// scores: [B, R, L] with L = n_past + T.
// ---------------------------------------------------------------------------
void ref_index_scores(const RefDims* D, const float* q_I, const float* k_I,
                      const float* w, int64_t w_tok_stride,
                      const int32_t* rows, int32_t R, double* scores) {
    const int L = D->n_past + D->T;
    // one (sequence, row, key) entry per iteration: a decode step (one row per
    // sequence) still spreads over every host core
#pragma omp parallel for collapse(3) schedule(dynamic, 256)
    for (int b = 0; b < D->B; ++b) {
        for (int r = 0; r < R; ++r) {
            for (int s = 0; s < L; ++s) {
                const int t = row_token(rows, r);
                const int p = D->n_past + t;
                double* out = scores + ((int64_t)b * R + r) * L;
                if (s > p) { out[s] = -INFINITY; continue; }
                double total = 0.0;
                for (int j = 0; j < D->H_I; ++j) {
                    const float* qv = q_I + (((int64_t)b * D->T + t) * D->H_I + j) * D->d_I;
                    const int jk = j % D->H_Ik;
                    const float* kv = k_I + (((int64_t)b * D->N_max + s) * D->H_Ik + jk) * D->d_I;
                    double dot = 0.0;
                    for (int c = 0; c < D->d_I; ++c) dot += (double)qv[c] * (double)kv[c];
                    const double relu = dot > 0.0 ? dot : 0.0;
                    total += weight_at(D, w, w_tok_stride, b, t, j) * relu;
                }
                out[s] = total;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Top-M selection (Sec. 3.2, "Indexer-Guided Token Selection": the summed
// indexer scores pick the M highest-scoring positions).  All
// candidates s <= p are sorted by (score descending, position ascending); the
// first min(M, p+1) are kept.  Output: the kept positions in ascending order,
// padded with -1 to M entries; count = min(M, p+1).
// scores: [B, R, L]; idx: [B, R, M]; count: [B, R].
// ---------------------------------------------------------------------------
void ref_topm(const RefDims* D, const double* scores, const int32_t* rows, int32_t R,
              int32_t* idx, int32_t* count) {
    const int L = D->n_past + D->T;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < D->B; ++b) {
        for (int r = 0; r < R; ++r) {
            const int t = row_token(rows, r);
            const int p = D->n_past + t;
            const double* sc = scores + ((int64_t)b * R + r) * L;
            std::vector<std::pair<double, int>> cand;
            cand.reserve(p + 1);
            for (int s = 0; s <= p; ++s) cand.push_back({sc[s], s});
            std::sort(cand.begin(), cand.end(),
                      [](const std::pair<double, int>& a, const std::pair<double, int>& c) {
                          if (a.first != c.first) return a.first > c.first;
                          return a.second < c.second;
                      });
            const int keep = std::min(D->M, p + 1);
            std::vector<int> chosen;
            for (int i = 0; i < keep; ++i) chosen.push_back(cand[i].second);
            std::sort(chosen.begin(), chosen.end());
            int32_t* out = idx + ((int64_t)b * R + r) * D->M;
            for (int i = 0; i < D->M; ++i) out[i] = i < keep ? chosen[i] : -1;
            count[(int64_t)b * R + r] = keep;
        }
    }
}

// Softmax attention of one query head over an explicit list of key positions
// (Sec. 3.1 "Softmax Attention"): l_s = sm_scale * <q, K[s]>,
// out = sum_s exp(l_s - max l) V[s] / sum_s exp(l_s - max l).
static void attend(const RefDims* D, const float* qh, const float* k_cache,
                   const float* v_cache, int b, int g, const int32_t* pos, int npos,
                   double* out) {
    std::vector<double> logit(npos);
    double mx = -INFINITY;
    for (int i = 0; i < npos; ++i) {
        const float* kv = k_cache + (((int64_t)b * D->N_max + pos[i]) * D->H_kv + g) * D->d;
        double dot = 0.0;
        for (int c = 0; c < D->d; ++c) dot += (double)qh[c] * (double)kv[c];
        logit[i] = D->sm_scale * dot;
        mx = std::max(mx, logit[i]);
    }
    double denom = 0.0;
    for (int c = 0; c < D->d; ++c) out[c] = 0.0;
    for (int i = 0; i < npos; ++i) {
        const double e = std::exp(logit[i] - mx);
        denom += e;
        const float* vv = v_cache + (((int64_t)b * D->N_max + pos[i]) * D->H_kv + g) * D->d;
        for (int c = 0; c < D->d; ++c) out[c] += e * (double)vv[c];
    }
    for (int c = 0; c < D->d; ++c) out[c] /= denom;
}

// ---------------------------------------------------------------------------
// Sparse self-attention SA_M over the selected positions (Sec. 3.2, Eq. 1; the
// cached entries at the chosen positions feed SA_M): query
// head h attends with KV head g = h / (H_q / H_kv) over the count[b, r] valid
// entries of idx[b, r, :].  q: [B, T, H_q, d]; caches: [B, N_max, H_kv, d];
// idx: [B, R, M]; o: [B, R, H_q, d].
// ---------------------------------------------------------------------------
void ref_sparse_attn(const RefDims* D, const float* q, const float* k_cache,
                     const float* v_cache, const int32_t* rows, int32_t R,
                     const int32_t* idx, const int32_t* count, double* o) {
    const int group = D->H_q / D->H_kv;
    // one (sequence, row, query head) per iteration
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < D->B; ++b) {
        for (int r = 0; r < R; ++r) {
            for (int h = 0; h < D->H_q; ++h) {
                const int t = row_token(rows, r);
                const int32_t* pos = idx + ((int64_t)b * R + r) * D->M;
                const int npos = count[(int64_t)b * R + r];
                const float* qh = q + (((int64_t)b * D->T + t) * D->H_q + h) * D->d;
                double* out = o + (((int64_t)b * R + r) * D->H_q + h) * D->d;
                attend(D, qh, k_cache, v_cache, b, h / group, pos, npos, out);
            }
        }
    }
}

// Dense causal softmax attention over every key s <= p (Sec. 3.1): the
// standard attention LISA replaces, and the limit of SA_M when M >= p + 1.
void ref_dense_attn(const RefDims* D, const float* q, const float* k_cache,
                    const float* v_cache, const int32_t* rows, int32_t R, double* o) {
    const int group = D->H_q / D->H_kv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < D->B; ++b) {
        for (int r = 0; r < R; ++r) {
            const int t = row_token(rows, r);
            const int p = D->n_past + t;
            std::vector<int32_t> pos(p + 1);
            for (int s = 0; s <= p; ++s) pos[s] = s;
            for (int h = 0; h < D->H_q; ++h) {
                const float* qh = q + (((int64_t)b * D->T + t) * D->H_q + h) * D->d;
                double* out = o + (((int64_t)b * R + r) * D->H_q + h) * D->d;
                attend(D, qh, k_cache, v_cache, b, h / group, pos.data(), p + 1, out);
            }
        }
    }
}

// Feature map of the linear branch: identity with no normaliser (the choice
// Sec. 3.1 adopts), or elu(x) + 1.
static inline double feature(int phi, double x) {
    if (phi == 0) return x;
    return x > 0.0 ? x + 1.0 : std::exp(x);
}

// ---------------------------------------------------------------------------
// Linear attention, recurrent form (Sec. 3.1 "Linear Attention"; Sec. 3.3
// Eq. 3-4), one token at a time, for each KV head g of each sequence:
//     S <- S + phi(k_t)^T v_t          (d x d, row = key feature, col = value)
//     z <- z + phi(k_t)                (elu+1 mode only)
//     o_t[h] = phi(q_t[h]) S           (identity: no normaliser)
//     o_t[h] = phi(q_t[h]) S / (phi(q_t[h]) . z)   (elu+1 mode)
// for every query head h of the group of g.  S: [B, H_kv, d, d] and z:
// [B, H_kv, d] hold the state before token 0 on entry and after token T-1 on
// return.  q_L: [B, T, H_q, d]; k_L, v_L: [B, T, H_kv, d]; o: [B, R, H_q, d]
// (only the sampled rows are written).
// ---------------------------------------------------------------------------
void ref_linear(const RefDims* D, const float* q_L, const float* k_L, const float* v_L,
                double* S, double* z, const int32_t* rows, int32_t R, double* o) {
    const int d = D->d;
    const int group = D->H_q / D->H_kv;
    std::vector<int> row_of_token(D->T, -1);
    for (int r = 0; r < R; ++r) row_of_token[row_token(rows, r)] = r;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < D->B; ++b) {
        for (int g = 0; g < D->H_kv; ++g) {
            double* Sg = S + ((int64_t)b * D->H_kv + g) * d * d;
            double* zg = z ? z + ((int64_t)b * D->H_kv + g) * d : nullptr;
            std::vector<double> fk(d), fq(d);
            for (int t = 0; t < D->T; ++t) {
                const float* kt = k_L + (((int64_t)b * D->T + t) * D->H_kv + g) * d;
                const float* vt = v_L + (((int64_t)b * D->T + t) * D->H_kv + g) * d;
                for (int i = 0; i < d; ++i) fk[i] = feature(D->phi, kt[i]);
                for (int i = 0; i < d; ++i)
                    for (int j = 0; j < d; ++j) Sg[(int64_t)i * d + j] += fk[i] * (double)vt[j];
                if (D->phi == 1)
                    for (int i = 0; i < d; ++i) zg[i] += fk[i];
                const int r = row_of_token[t];
                if (r < 0) continue;
                for (int hh = 0; hh < group; ++hh) {
                    const int h = g * group + hh;
                    const float* qt = q_L + (((int64_t)b * D->T + t) * D->H_q + h) * d;
                    for (int i = 0; i < d; ++i) fq[i] = feature(D->phi, qt[i]);
                    double denom = 1.0;
                    if (D->phi == 1) {
                        denom = 0.0;
                        for (int i = 0; i < d; ++i) denom += fq[i] * zg[i];
                    }
                    double* out = o + (((int64_t)b * R + r) * D->H_q + h) * d;
                    for (int j = 0; j < d; ++j) {
                        double acc = 0.0;
                        for (int i = 0; i < d; ++i) acc += fq[i] * Sg[(int64_t)i * d + j];
                        out[j] = acc / denom;
                    }
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Gate (Sec. 3.2 Eq. 1): o = g * o_LA + (1 - g) * o_SA_M with
// g = sigmoid(logit), one logit per (token, query head).
// logit: [B, T, H_q]; o_lin, o_sp, o: [B, R, H_q, d].
// ---------------------------------------------------------------------------
void ref_gate(const RefDims* D, const float* logit, const int32_t* rows, int32_t R,
              const double* o_lin, const double* o_sp, double* o) {
    for (int b = 0; b < D->B; ++b) {
        for (int r = 0; r < R; ++r) {
            const int t = row_token(rows, r);
            for (int h = 0; h < D->H_q; ++h) {
                const double x = logit[((int64_t)b * D->T + t) * D->H_q + h];
                const double g = 1.0 / (1.0 + std::exp(-x));
                const int64_t base = (((int64_t)b * R + r) * D->H_q + h) * D->d;
                for (int c = 0; c < D->d; ++c)
                    o[base + c] = g * o_lin[base + c] + (1.0 - g) * o_sp[base + c];
            }
        }
    }
}

// ---------------------------------------------------------------------------
// The whole module for the query tokens of one call, in the order of the
// paper's decoding description (Sec. 3.2): indexer scores over the full
// cache, top-M, sparse attention over the selected positions, the linear
// branch, and the gate.  The caches must already hold positions
// [0, n_past + T) (the current tokens included).  Outputs are for the
// sampled rows; S and z are advanced over all T tokens.
// idx: [B, R, M], count: [B, R]; o, o_sp, o_lin: [B, R, H_q, d].
// ---------------------------------------------------------------------------
int ref_forward(const RefDims* D, const float* q, const float* k_cache, const float* v_cache,
                const float* q_I, const float* k_I, const float* w, int64_t w_tok_stride,
                const float* q_L, const float* k_L, const float* v_L, const float* gate_logit,
                double* S, double* z, const int32_t* rows, int32_t R,
                int32_t* idx, int32_t* count, double* o_sp, double* o_lin, double* o) {
    const int64_t L = (int64_t)D->n_past + D->T;
    std::vector<double> scores((size_t)D->B * R * L);
    ref_index_scores(D, q_I, k_I, w, w_tok_stride, rows, R, scores.data());
    ref_topm(D, scores.data(), rows, R, idx, count);
    ref_sparse_attn(D, q, k_cache, v_cache, rows, R, idx, count, o_sp);
    ref_linear(D, q_L, k_L, v_L, S, z, rows, R, o_lin);
    ref_gate(D, gate_logit, rows, R, o_lin, o_sp, o);
    return 0;
}

// ---------------------------------------------------------------------------
// Sliding-window selection (Sec. 3.2, Stage 1: the sparse branch attends over
// a fixed window of the last M positions before the Indexer replaces it):
// query position p keeps [max(0, p-M+1), p], in ascending order, -1 padded.
// idx: [B, R, M], count: [B, R].
// ---------------------------------------------------------------------------
void ref_window_indices(const RefDims* D, const int32_t* rows, int32_t R, int32_t* idx,
                        int32_t* count) {
    for (int b = 0; b < D->B; ++b) {
        for (int r = 0; r < R; ++r) {
            const int p = D->n_past + row_token(rows, r);
            const int first = std::max(0, p - D->M + 1);
            const int c = p - first + 1;
            int32_t* out = idx + ((int64_t)b * R + r) * D->M;
            for (int i = 0; i < D->M; ++i) out[i] = i < c ? first + i : -1;
            count[(int64_t)b * R + r] = c;
        }
    }
}

// ---------------------------------------------------------------------------
// Segment state transfer and correction at the end of reasoning segment t
// (t >= 1), Sec. 3.3 Eq. 6-9, for every state matrix S[b, g] (d x d):
//   grad_t    = S_end - S_start                  (Eq. 6; S_start = S_{t-1})
//   mean_prev = grad_sum / (t - 1), or 0 at t = 1 (Eq. 7)
//   grad_hat  = (1 - alpha) grad_t + alpha mean_prev        (Eq. 8)
//   S_t       = S_start + grad_hat                          (Eq. 9)
// In place: S (in: the state the segment's tokens reached; out: S_t),
// S_start (out: S_t, the start of the next segment), grad_sum (out: the sum
// of grad_1 .. grad_t).  All [B, H_kv, d, d].
// ---------------------------------------------------------------------------
void ref_state_transfer(const RefDims* D, double* S, double* S_start, double* grad_sum, int t,
                        double alpha) {
    const int64_t n = (int64_t)D->B * D->H_kv * D->d * D->d;
    for (int64_t i = 0; i < n; ++i) {
        const double grad_t = S[i] - S_start[i];
        const double mean_prev = t > 1 ? grad_sum[i] / (t - 1) : 0.0;
        const double grad_hat = (1.0 - alpha) * grad_t + alpha * mean_prev;
        const double S_t = S_start[i] + grad_hat;
        grad_sum[i] += grad_t;
        S[i] = S_t;
        S_start[i] = S_t;
    }
}

// ---------------------------------------------------------------------------
// Per-channel gate (Sec. 3.3 Eq. 5): g = sigmoid(W_g h), one gate per output
// channel (query head x dim), mixing the two branches as in Eq. 1:
// o = g * o_LA + (1 - g) * o_SA_M.  h: [B, T, D_h]; W_g: [H_q*d, D_h];
// o_lin, o_sp, o: [B, R, H_q, d].
// ---------------------------------------------------------------------------
void ref_gate_channel(const RefDims* D, int D_h, const float* h, const float* W_g,
                      const int32_t* rows, int32_t R, const double* o_lin, const double* o_sp,
                      double* o) {
    const int N = D->H_q * D->d;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < D->B; ++b) {
        for (int r = 0; r < R; ++r) {
            const int t = row_token(rows, r);
            const float* hv = h + ((int64_t)b * D->T + t) * D_h;
            const int64_t base = ((int64_t)b * R + r) * N;
            for (int c = 0; c < N; ++c) {
                double x = 0.0;
                for (int k = 0; k < D_h; ++k) x += (double)W_g[(int64_t)c * D_h + k] * hv[k];
                const double g = 1.0 / (1.0 + std::exp(-x));
                o[base + c] = (1.0 - g) * o_sp[base + c] + g * o_lin[base + c];
            }
        }
    }
}

}  // extern "C"
