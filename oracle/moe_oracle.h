/*
 * CPU oracle of the top-k softmax-routed (latent) mixture-of-experts layer forward.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * load this library.  It shares no code, header, table or helper with the CUDA library; the two
 * see the same inputs only through the seeded input generator.
 *
 * It is the plain definition, evaluated one token at a time: every dot product accumulates in
 * double, no blocking, no permutation of rows, no fusion.  Values are rounded to the storage
 * dtype exactly at the boundaries the pages fix (see moe_oracle.c).
 *
 * Sources (the pages this layer is taken from):
 *   [MUSE]    "Muse Spark Open: Norm-Preserving Gates Are Not a Norm Guarantee" (flozi.net)
 *   [ARCHDB]  "Muse-Spark-Open-816B-A42B" model sheet (archdb.vladsavinov.com)
 *   [SHAZEER] "816 billion parameters, and only 42 billion show up for each token"
 *             (bobbyburns.tech), explaining Shazeer et al.'s sparsely gated MoE layer
 *   [ATLAS]   "Muse Spark Open (816B-A42B)" architecture card (llm-atlas)
 *
 * Every function is pinned by a CPU test (worked examples printed on the pages, closed forms,
 * reductions to textbook cases, brute force on tiny inputs); see tests/test_oracle_pins.py.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int T, d_model, d_latent, d_ff, n_experts, top_k;
  int is_bf16;     /* 1: tensors are bf16 bit patterns and bf16 rounding is mirrored; 0: fp32;
                      2: fp32 tensors, float64 storage (no rounding; used by the pins) */
  int act;         /* 0: ReLU expert (Shazeer), 1: SwiGLU expert (Muse) */
  int pre_norm;    /* centred RMSNorm C_pre after the latent down-projection */
  int expert_norm; /* input-scaled RMSNorm I_gamma on each expert output, before weighting */
  int resid_mode;  /* 0: none, 1: Muse residual gate, 2: literal h + g*b */
  double eps, tau, resid_floor, routed_scale;
  int gate_mode;     /* 0: softmax over all n then renormalise over the kept k;
                        1: Muse sigmoid gate (scores sigmoid(l), selection by score + correction
                           bias, weights score / (sum_sel score + 1e-15)) */
  int router_f32;    /* 1: router weights are fp32 (whatever the tensors' dtype) */
  double logit_mult; /* output_multiplier applied to the router logits (sigmoid gate) */
  int input_norm;    /* decoder wrap: u = C_in(h), the residual stream's centred RMSNorm */
  int post_norm;     /* decoder wrap: the FFN's input-scaled output norm I_post on b before the
                        residual gate */
  double eps_block;  /* epsilon of the two decoder-level norms */
} orc_cfg;

typedef struct {
  const void* u;            /* [T, d_model] layer input (router and down-projection read it) */
  const void* h;            /* [T, d_model] residual stream r (may equal u) */
  const void* w_router;     /* [n, d_model] */
  const float* logit_bias;  /* [n] added to the logits, or NULL */
  const void* p_down;       /* [d_latent, d_model] */
  const void* p_up;         /* [d_model, d_latent] */
  const void* const* w_gu;  /* per expert e: [2*d_ff (gate rows, then up rows) or d_ff, E_in] */
  const void* const* w_down;/* per expert e: [E_in, d_ff] */
  const float* gamma_pre;   /* [d_latent] */
  const float* gamma_expert;/* [E_in], one gain shared by every expert */
  const float* resid_g;     /* [d_model] */
  const float* correction_bias; /* [n] sigmoid gate: added to the scores for selection only */
  const float* gamma_in;    /* [d_model] input_norm gain */
  const float* gamma_post;  /* [d_model] post_norm gain */
} orc_tensors;

/* storage rounding of the configured dtype (bf16 RNE, or fp32) */
double orc_round(const orc_cfg* c, double x);
/* bf16 bit pattern <-> double */
double orc_bf16_to_double(uint16_t b);
uint16_t orc_double_to_bf16(double x);

/* Norms on a D-vector (double in, double out, no storage rounding; eps as given). */
void orc_rms_normalize(const double* x, int D, double eps, double* out);
void orc_centered_rmsnorm(const double* x, const double* gamma, int D, double eps, double* out);
void orc_input_scaled_rmsnorm(const orc_cfg* c, const double* x, const double* gamma, int D,
                              double eps, double* out);
/* The vector I_gamma reduces: s = (1 + gamma) * x rounded to the storage dtype. */
void orc_input_scaled_vector(const orc_cfg* c, const double* x, const double* gamma, int D,
                             double* s);

/* Softmax over n logits then top-k by (logit desc, index asc); weights renormalised to sum 1
 * and multiplied by routed_scale.  Slot order is the selection order. */
void orc_softmax_topk(const double* logits, int n, int k, double routed_scale, int* idx, double* w);
/* Same selection on float logits (used to check a given logit vector's selection). */
void orc_softmax_topk_f32(const float* logits, int n, int k, double routed_scale, int* idx,
                          double* w);

/* Residual gate coefficients for one channel. */
void orc_resid_gate_coeffs(double g, double tau, double floor_, double* alpha, double* beta);

/* Muse sigmoid gate on logits l (already multiplied by output_multiplier):
 * s = sigmoid(l); the k experts with the largest s + correction_bias (ties to the lower index),
 * in that order; w_j = s_j / (sum_sel s + 1e-15) * routed_scale.  scores (may be NULL) gets s. */
void orc_sigmoid_topk(const double* logits, const float* correction_bias, int n, int k,
                      double routed_scale, int* idx, double* w, double* scores);
/* The same selection taken in fp32 on given fp32 scores: key = (float)(s + bias) (an exact
 * IEEE fp32 addition), ties to the lower index; weights from the given scores in double. */
void orc_sigmoid_topk_scores_f32(const float* scores, const float* correction_bias, int n, int k,
                                 double routed_scale, int* idx, double* w);

/* Per-token steps. */
void orc_router_token(const orc_cfg* c, const orc_tensors* x, int64_t t, double* logits, int* idx,
                      double* w);
void orc_expert_input_token(const orc_cfg* c, const orc_tensors* x, int64_t t, double* z);
void orc_expert_token(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                      const float* gamma_expert, const double* z, double* nout);
/* The same expert's output before its norm: s = dtype((1 + gamma_expert) * o) with expert_norm
 * (the vector I_gamma reduces), else o. */
void orc_expert_token_scaled(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                             const float* gamma_expert, const double* z, double* s);
void orc_combine_token(const orc_cfg* c, const double* n_slots, const double* w, double* y);
void orc_output_token(const orc_cfg* c, const orc_tensors* x, int64_t t, const double* y,
                      double* out);

/* The whole layer for a list of tokens, threads over tokens.  out: [ntok, d_model];
 * logits: [ntok, n] or NULL; idx: [ntok, k] or NULL; w: [ntok, k] or NULL;
 * y_latent: [ntok, E_in] or NULL (the combined expert output before the output step). */
void orc_layer_forward(const orc_cfg* c, const orc_tensors* x, const int64_t* tokens, int ntok,
                       double* out, double* logits, int* idx, double* w, double* y_latent,
                       int nthreads);

/* Router step (orc_router_token) for rows[i] of the tensors, i < nrows, threads over rows:
 * logits [nrows, n] (the sigmoid scores in that mode), idx [nrows, k], w [nrows, k]. */
void orc_router_batch(const orc_cfg* c, const orc_tensors* x, const int64_t* rows, int nrows,
                      double* logits, int* idx, double* w, int nthreads);

/* Expert step for a batch of (token, slot) rows routed to one expert; threads over rows. */
void orc_expert_batch(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                      const float* gamma_expert, const double* z_rows, int nrows, double* n_rows,
                      int nthreads);
/* The same, also returning each row's pre-norm vector (orc_expert_token_scaled) in s_rows
 * [nrows, E_in] when it is not NULL. */
void orc_expert_batch_parts(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                            const float* gamma_expert, const double* z_rows, int nrows,
                            double* s_rows, double* n_rows, int nthreads);

/* Shazeer et al.'s noisy top-k gate and its balancing statistics [SHAZEER "The gate", "Keeping the
 * experts busy"], for one token from its clean logits l = x W_g, noise logits m = x W_noise and
 * the standard-normal draw eps (all [n]):
 *   H_i = l_i + eps_i * softplus(m_i);  G = Softmax(KeepTopK(H, k)) (dense [n], zeros off the
 *   top k; selection by H desc, ties to the lower index; idx gets the k selected in order);
 *   P_i = Phi((l_i - kth_excluding(H, k, i)) / softplus(m_i)), kth_excluding(H, k, i) being the
 *   k-th largest of H over the experts other than i. */
void orc_noisy_gate_token(const double* l, const double* m, const double* eps, int n, int k,
                          double* H, double* G, double* P, int* idx);
/* CV(v)^2 = population variance / mean^2 of v[n]. */
double orc_cv_squared(const double* v, int n);

/* Canonical permutation of routed slots: rows grouped by expert ascending, and within an expert
 * by token ascending.  offsets[n+1], perm_token[T*k] (row -> token), inv_perm[T*k]
 * (slot t*k+j -> row).  Returns 0, or -1 if an index is out of range or repeated in a token. */
int orc_permutation(int T, int k, int n, const int32_t* idx, int32_t* offsets,
                    int32_t* perm_token, int32_t* inv_perm);

#ifdef __cplusplus
}
#endif
#endif
