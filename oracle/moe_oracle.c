/*
 * CPU oracle of the top-k softmax-routed (latent) MoE layer forward.
 *
 * TEST INFRASTRUCTURE: only tests/, the smoke check and the benchmark's CPU-baseline leg load it.
 * It shares nothing with the CUDA library.
 *
 * The layer, per token t (sources in moe_oracle.h):
 *
 *  1. Router [SHAZEER "The gate"; MUSE "Latent experts"; ARCHDB gating fields]:
 *     l = u_t . W_g^T (+ bias), p = softmax(l), keep the k largest, w_j = p_j / sum_sel p
 *     (times routed_scaling_factor = 1).  Softmax-then-renormalise over the kept entries equals
 *     the page's Softmax(KeepTopK(l, k)) in real arithmetic.
 *  2. Expert input [MUSE "Latent experts"]: z = C_pre(P_down u_t), where C_gamma(x) =
 *     (1+gamma) * R_eps(x) is the output-scaled centred RMSNorm and R_eps(x) = x / sqrt(mean(x^2)
 *     + eps) [MUSE "Two normalization orders"].  Shazeer layer: z = u_t.
 *  3. Experts [MUSE "Latent experts"; ARCHDB "SwiGLU"; SHAZEER "The math"]:
 *     SwiGLU  f_e(z) = W_d,e (SiLU(W_gate,e z) * (W_up,e z)), gate rows first in the packed matrix;
 *     ReLU    E_e(z) = W_2,e ReLU(W_1,e z), no biases.
 *  4. Per-expert norm before mixing [MUSE "Latent experts", "Two normalization orders"]:
 *     n_j = I_gamma(f_e(z)) = R_eps(round(D_gamma f)), the scaled vector rounded to the input dtype
 *     before the reduction; one gain vector shared by all experts.
 *  5. Weighted combine [SHAZEER "The math": y = sum_i G(x)_i E_i(x)]: y = sum_j w_j n_j.
 *  6. Output [MUSE "Residual gates"; ARCHDB residual field]: b = P_up y;
 *     out = alpha*h + beta*b with beta = sigmoid(g/tau), alpha = sqrt(max(sigmoid(-g/tau)(1+beta),
 *     delta)) per channel; or the literal h + g*b; or b alone (no residual).
 *
 * Arithmetic: every dot product and reduction accumulates in double.  With is_bf16, values are
 * rounded to bf16 (round to nearest even, through fp32) where a bf16 implementation stores them:
 * every GEMM output (z_raw, SwiGLU/ReLU activation, expert output o, y, b), each norm's output
 * (norms return the input dtype, [MUSE "What this means for serving and kernel work"]), the
 * I_gamma scaled vector before its reduction [MUSE "Two normalization orders"], and the layer
 * output.  With fp32 tensors the same boundaries round to fp32.  Exponentials, square roots and
 * divisions are the C library's double-precision ones.
 */
#include "moe_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ scalar conversions */

double orc_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

uint16_t orc_double_to_bf16(double x) {
  float f = (float)x;
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

double orc_round(const orc_cfg* c, double x) {
  if (c->is_bf16 == 1) return orc_bf16_to_double(orc_double_to_bf16(x));
  if (c->is_bf16 == 2) return x; /* float64 storage: no rounding (used by the pins) */
  return (double)(float)x;
}

/* element i of a tensor stored as bf16 codes or fp32 */
static double ld(const void* p, size_t i, int is_bf16) {
  if (is_bf16 == 1) return orc_bf16_to_double(((const uint16_t*)p)[i]);
  return (double)((const float*)p)[i];
}

/* sum_i W[row, i] * x[i] over one row of a row-major matrix of width n, in double */
static double dot_row(const void* W, size_t row, int n, const double* x, int is_bf16) {
  double acc = 0.0;
  size_t base = row * (size_t)n;
  if (is_bf16 == 1) {
    const uint16_t* w = (const uint16_t*)W + base;
    for (int i = 0; i < n; ++i) acc += orc_bf16_to_double(w[i]) * x[i];
  } else {
    const float* w = (const float*)W + base;
    for (int i = 0; i < n; ++i) acc += (double)w[i] * x[i];
  }
  return acc;
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* ------------------------------------------------------------------ norms */

/* R_eps(x) = x / sqrt(mean(x^2) + eps)  [MUSE "Two normalization orders"; the mean (not the sum)
 * is fixed by the page's worked example, where I_gamma((1,1)) = (2,1)/sqrt(2.5)]. */
void orc_rms_normalize(const double* x, int D, double eps, double* out) {
  double ss = 0.0;
  for (int i = 0; i < D; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / D + eps);
  for (int i = 0; i < D; ++i) out[i] = x[i] * inv;
}

/* C_gamma(x) = D_gamma R_eps(x), D_gamma = diag(1 + gamma): output-scaled centred RMSNorm. */
void orc_centered_rmsnorm(const double* x, const double* gamma, int D, double eps, double* out) {
  orc_rms_normalize(x, D, eps, out);
  for (int i = 0; i < D; ++i) out[i] *= 1.0 + gamma[i];
}

/* D_gamma x = (1 + gamma) * x, rounded to the input dtype: the vector I_gamma reduces. */
void orc_input_scaled_vector(const orc_cfg* c, const double* x, const double* gamma, int D,
                             double* s) {
  for (int i = 0; i < D; ++i) s[i] = orc_round(c, (1.0 + gamma[i]) * x[i]);
}

/* I_gamma(x) = R_eps(D_gamma x), with D_gamma x rounded to the input dtype before the reduction. */
void orc_input_scaled_rmsnorm(const orc_cfg* c, const double* x, const double* gamma, int D,
                              double eps, double* out) {
  double* s = (double*)malloc(sizeof(double) * (size_t)D);
  orc_input_scaled_vector(c, x, gamma, D, s);
  orc_rms_normalize(s, D, eps, out);
  free(s);
}

/* ------------------------------------------------------------------ gate */

/* Selection by (logit desc, index asc), then softmax over all n and renormalisation over the
 * kept k [SHAZEER "The gate"; ARCHDB "Selected expert weights are renormalized to sum to 1"]. */
void orc_softmax_topk(const double* logits, int n, int k, double routed_scale, int* idx,
                      double* w) {
  double mx = logits[0];
  for (int e = 1; e < n; ++e)
    if (logits[e] > mx) mx = logits[e];
  double z = 0.0;
  for (int e = 0; e < n; ++e) z += exp(logits[e] - mx);
  char* taken = (char*)calloc((size_t)n, 1);
  double sel = 0.0;
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < n; ++e) {
      if (taken[e]) continue;
      if (best < 0 || logits[e] > logits[best]) best = e; /* strict: ties keep the lower index */
    }
    taken[best] = 1;
    idx[j] = best;
    w[j] = exp(logits[best] - mx) / z; /* p_best */
    sel += w[j];
  }
  for (int j = 0; j < k; ++j) w[j] = w[j] / sel * routed_scale;
  free(taken);
}

void orc_softmax_topk_f32(const float* logits, int n, int k, double routed_scale, int* idx,
                          double* w) {
  double* l = (double*)malloc(sizeof(double) * (size_t)n);
  for (int e = 0; e < n; ++e) l[e] = (double)logits[e];
  orc_softmax_topk(l, n, k, routed_scale, idx, w);
  free(l);
}

/* Muse sigmoid gate [MUSE "Latent experts": fp32 logits times output_multiplier, sigmoid; a
 * correction bias affects top-k selection only; weights gather the original sigmoid scores,
 * divide by their selected sum plus 1e-15 and apply routed_scaling_factor]. */
void orc_sigmoid_topk(const double* logits, const float* correction_bias, int n, int k,
                      double routed_scale, int* idx, double* w, double* scores) {
  double* s = (double*)malloc(sizeof(double) * (size_t)n);
  char* taken = (char*)calloc((size_t)n, 1);
  for (int e = 0; e < n; ++e) s[e] = sigmoid(logits[e]);
  double sel = 0.0;
  for (int j = 0; j < k; ++j) {
    int best = -1;
    double best_key = 0.0;
    for (int e = 0; e < n; ++e) {
      if (taken[e]) continue;
      double key = s[e] + (correction_bias ? (double)correction_bias[e] : 0.0);
      if (best < 0 || key > best_key) { best = e; best_key = key; }
    }
    taken[best] = 1;
    idx[j] = best;
    w[j] = s[best];
    sel += s[best];
  }
  for (int j = 0; j < k; ++j) w[j] = w[j] / (sel + 1e-15) * routed_scale;
  if (scores) memcpy(scores, s, sizeof(double) * (size_t)n);
  free(taken);
  free(s);
}

void orc_sigmoid_topk_scores_f32(const float* scores, const float* correction_bias, int n, int k,
                                 double routed_scale, int* idx, double* w) {
  char* taken = (char*)calloc((size_t)n, 1);
  double sel = 0.0;
  for (int j = 0; j < k; ++j) {
    int best = -1;
    float best_key = 0.0f;
    for (int e = 0; e < n; ++e) {
      if (taken[e]) continue;
      float key = scores[e] + (correction_bias ? correction_bias[e] : 0.0f);
      if (best < 0 || key > best_key) { best = e; best_key = key; }
    }
    taken[best] = 1;
    idx[j] = best;
    w[j] = (double)scores[best];
    sel += (double)scores[best];
  }
  for (int j = 0; j < k; ++j) w[j] = w[j] / (sel + 1e-15) * routed_scale;
  free(taken);
}

/* beta = sigmoid(g/tau), alpha = sqrt(max(sigmoid(-g/tau) * (1 + beta), delta))
 * [MUSE "Residual gates"; ARCHDB residual field].  Not rewritten as 1 - beta^2. */
void orc_resid_gate_coeffs(double g, double tau, double floor_, double* alpha, double* beta) {
  double b = sigmoid(g / tau);
  double a2 = sigmoid(-g / tau) * (1.0 + b);
  if (a2 < floor_) a2 = floor_;
  *beta = b;
  *alpha = sqrt(a2);
}

/* ------------------------------------------------------------------ per-token steps */

static int expert_in(const orc_cfg* c) { return c->d_latent > 0 ? c->d_latent : c->d_model; }

/* The layer's branch input u_t: the given u, or with input_norm the residual stream's centred
 * RMSNorm dtype(C_in(h_t)) [MUSE "The complete layer has two separately normalized residual
 * updates": the layer normalizes the residual stream, then runs the latent MoE; ARCHDB: block
 * norms are RMSNorm with a (1 + w) gain]. */
static void load_u(const orc_cfg* c, const orc_tensors* x, int64_t t, double* ut) {
  int d = c->d_model;
  if (!c->input_norm) {
    for (int i = 0; i < d; ++i) ut[i] = ld(x->u, (size_t)t * d + i, c->is_bf16);
    return;
  }
  double* h = (double*)malloc(sizeof(double) * (size_t)d);
  double* g = (double*)malloc(sizeof(double) * (size_t)d);
  for (int i = 0; i < d; ++i) {
    h[i] = ld(x->h, (size_t)t * d + i, c->is_bf16);
    g[i] = (double)x->gamma_in[i];
  }
  orc_centered_rmsnorm(h, g, d, c->eps_block, ut);
  for (int i = 0; i < d; ++i) ut[i] = orc_round(c, ut[i]);
  free(g);
  free(h);
}

void orc_router_token(const orc_cfg* c, const orc_tensors* x, int64_t t, double* logits, int* idx,
                      double* w) {
  int d = c->d_model, n = c->n_experts;
  double* ut = (double*)malloc(sizeof(double) * (size_t)d);
  load_u(c, x, t, ut);
  /* fp32 router weights are read as fp32 whatever the other tensors' dtype */
  const int w_is_bf16 = c->router_f32 ? 0 : c->is_bf16;
  for (int e = 0; e < n; ++e) {
    logits[e] = dot_row(x->w_router, (size_t)e, d, ut, w_is_bf16);
    if (c->gate_mode == 1) logits[e] *= c->logit_mult;
    if (x->logit_bias) logits[e] += (double)x->logit_bias[e];
  }
  if (c->gate_mode == 1) {
    /* logits[] returns the sigmoid scores in this mode (what the weights are made of) */
    orc_sigmoid_topk(logits, x->correction_bias, n, c->top_k, c->routed_scale, idx, w, logits);
  } else {
    orc_softmax_topk(logits, n, c->top_k, c->routed_scale, idx, w);
  }
  free(ut);
}

void orc_expert_input_token(const orc_cfg* c, const orc_tensors* x, int64_t t, double* z) {
  int d = c->d_model, L = c->d_latent;
  if (L <= 0) {
    load_u(c, x, t, z);
    return;
  }
  double* ut = (double*)malloc(sizeof(double) * (size_t)d);
  double* zr = (double*)malloc(sizeof(double) * (size_t)L);
  load_u(c, x, t, ut);
  for (int i = 0; i < L; ++i) zr[i] = orc_round(c, dot_row(x->p_down, (size_t)i, d, ut, c->is_bf16));
  if (c->pre_norm) {
    double* g = (double*)malloc(sizeof(double) * (size_t)L);
    for (int i = 0; i < L; ++i) g[i] = (double)x->gamma_pre[i];
    orc_centered_rmsnorm(zr, g, L, c->eps, z);
    for (int i = 0; i < L; ++i) z[i] = orc_round(c, z[i]);
    free(g);
  } else {
    memcpy(z, zr, sizeof(double) * (size_t)L);
  }
  free(zr);
  free(ut);
}

/* One expert on one input row: o = dtype(W_d act), act = dtype(SiLU(W_gate z) * W_up z) or
 * dtype(ReLU(W_1 z)). */
static void expert_output(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                          const double* z, double* o) {
  int E = expert_in(c), H = c->d_ff;
  double* hid = (double*)malloc(sizeof(double) * (size_t)H);
  for (int i = 0; i < H; ++i) {
    if (c->act == 1) {
      double g = dot_row(w_gu_e, (size_t)i, E, z, c->is_bf16);       /* gate row i */
      double v = dot_row(w_gu_e, (size_t)(H + i), E, z, c->is_bf16); /* up row i */
      hid[i] = orc_round(c, (g / (1.0 + exp(-g))) * v);              /* SiLU(g) * v */
    } else {
      double a = dot_row(w_gu_e, (size_t)i, E, z, c->is_bf16);
      hid[i] = orc_round(c, a > 0.0 ? a : 0.0);                      /* ReLU */
    }
  }
  for (int j = 0; j < E; ++j) o[j] = orc_round(c, dot_row(w_down_e, (size_t)j, H, hid, c->is_bf16));
  free(hid);
}

/* One expert on one row: nout = I_gamma(o) stored in the dtype (or o without expert_norm), and,
 * if s is not NULL, the vector I_gamma reduces, s = dtype(D_gamma o) (or o). */
static void expert_token_parts(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                               const float* gamma_expert, const double* z, double* s,
                               double* nout) {
  int E = expert_in(c);
  double* o = (double*)malloc(sizeof(double) * (size_t)E);
  expert_output(c, w_gu_e, w_down_e, z, o);
  if (c->expert_norm) {
    double* g = (double*)malloc(sizeof(double) * (size_t)E);
    double* sv = (double*)malloc(sizeof(double) * (size_t)E);
    for (int j = 0; j < E; ++j) g[j] = (double)gamma_expert[j];
    orc_input_scaled_vector(c, o, g, E, sv); /* I_gamma = R_eps(dtype(D_gamma o)) */
    orc_rms_normalize(sv, E, c->eps, nout);
    for (int j = 0; j < E; ++j) nout[j] = orc_round(c, nout[j]);
    if (s) memcpy(s, sv, sizeof(double) * (size_t)E);
    free(sv);
    free(g);
  } else {
    memcpy(nout, o, sizeof(double) * (size_t)E);
    if (s) memcpy(s, o, sizeof(double) * (size_t)E);
  }
  free(o);
}

void orc_expert_token(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                      const float* gamma_expert, const double* z, double* nout) {
  expert_token_parts(c, w_gu_e, w_down_e, gamma_expert, z, NULL, nout);
}

void orc_expert_token_scaled(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                             const float* gamma_expert, const double* z, double* s) {
  double* n = (double*)malloc(sizeof(double) * (size_t)expert_in(c));
  expert_token_parts(c, w_gu_e, w_down_e, gamma_expert, z, s, n);
  free(n);
}

/* y = sum_j w_j n_j, accumulated in slot order, then stored in the dtype. */
void orc_combine_token(const orc_cfg* c, const double* n_slots, const double* w, double* y) {
  int E = expert_in(c);
  for (int i = 0; i < E; ++i) {
    double acc = 0.0;
    for (int j = 0; j < c->top_k; ++j) acc += w[j] * n_slots[(size_t)j * E + i];
    y[i] = orc_round(c, acc);
  }
}

void orc_output_token(const orc_cfg* c, const orc_tensors* x, int64_t t, const double* y,
                      double* out) {
  int d = c->d_model, L = c->d_latent;
  double* bv = (double*)malloc(sizeof(double) * (size_t)d);
  for (int i = 0; i < d; ++i)
    bv[i] = (L > 0) ? orc_round(c, dot_row(x->p_up, (size_t)i, L, y, c->is_bf16)) : y[i];
  if (c->post_norm) {
    /* the FFN's input-scaled output norm before the residual gate [MUSE "The complete layer
     * has two separately normalized residual updates"]: b <- dtype(I_post(b)) */
    double* g = (double*)malloc(sizeof(double) * (size_t)d);
    double* nb = (double*)malloc(sizeof(double) * (size_t)d);
    for (int i = 0; i < d; ++i) g[i] = (double)x->gamma_post[i];
    orc_input_scaled_rmsnorm(c, bv, g, d, c->eps_block, nb);
    for (int i = 0; i < d; ++i) bv[i] = orc_round(c, nb[i]);
    free(nb);
    free(g);
  }
  for (int i = 0; i < d; ++i) {
    double b = bv[i];
    double r;
    if (c->resid_mode == 0) {
      r = b;
    } else {
      double h = ld(x->h, (size_t)t * d + i, c->is_bf16), g = (double)x->resid_g[i];
      if (c->resid_mode == 1) {
        double alpha, beta;
        orc_resid_gate_coeffs(g, c->tau, c->resid_floor, &alpha, &beta);
        r = alpha * h + beta * b;
      } else {
        r = h + g * b;
      }
    }
    out[i] = orc_round(c, r);
  }
  free(bv);
}

/* ------------------------------------------------------------------ whole layer */

typedef struct {
  const orc_cfg* c;
  const orc_tensors* x;
  const int64_t* tokens;
  int lo, hi;
  double *out, *logits, *w, *y_latent;
  int* idx;
} layer_job;

static void layer_one(const orc_cfg* c, const orc_tensors* x, int64_t t, double* out,
                      double* logits, int* idx, double* w, double* y_latent) {
  int E = expert_in(c), k = c->top_k;
  double* z = (double*)malloc(sizeof(double) * (size_t)E);
  double* ns = (double*)malloc(sizeof(double) * (size_t)E * k);
  double* y = (double*)malloc(sizeof(double) * (size_t)E);
  orc_router_token(c, x, t, logits, idx, w);
  orc_expert_input_token(c, x, t, z);
  for (int j = 0; j < k; ++j)
    orc_expert_token(c, x->w_gu[idx[j]], x->w_down[idx[j]], x->gamma_expert, z,
                     ns + (size_t)j * E);
  orc_combine_token(c, ns, w, y);
  if (y_latent) memcpy(y_latent, y, sizeof(double) * (size_t)E);
  orc_output_token(c, x, t, y, out);
  free(y);
  free(ns);
  free(z);
}

static void* layer_worker(void* p) {
  layer_job* j = (layer_job*)p;
  const orc_cfg* c = j->c;
  int n = c->n_experts, k = c->top_k, E = expert_in(c);
  double* lg = (double*)malloc(sizeof(double) * (size_t)n);
  int* id = (int*)malloc(sizeof(int) * (size_t)k);
  double* wt = (double*)malloc(sizeof(double) * (size_t)k);
  for (int i = j->lo; i < j->hi; ++i) {
    layer_one(c, j->x, j->tokens[i], j->out + (size_t)i * c->d_model, lg, id, wt,
              j->y_latent ? j->y_latent + (size_t)i * E : NULL);
    if (j->logits) memcpy(j->logits + (size_t)i * n, lg, sizeof(double) * (size_t)n);
    if (j->idx) memcpy(j->idx + (size_t)i * k, id, sizeof(int) * (size_t)k);
    if (j->w) memcpy(j->w + (size_t)i * k, wt, sizeof(double) * (size_t)k);
  }
  free(wt);
  free(id);
  free(lg);
  return NULL;
}

void orc_layer_forward(const orc_cfg* c, const orc_tensors* x, const int64_t* tokens, int ntok,
                       double* out, double* logits, int* idx, double* w, double* y_latent,
                       int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > ntok) nthreads = ntok > 0 ? ntok : 1;
  layer_job* jobs = (layer_job*)calloc((size_t)nthreads, sizeof(layer_job));
  pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  int* ok = (int*)calloc((size_t)nthreads, sizeof(int));
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = (layer_job){c, x, tokens, (int)((long)ntok * t / nthreads),
                          (int)((long)ntok * (t + 1) / nthreads), out, logits, w, y_latent, idx};
    ok[t] = pthread_create(&tid[t], NULL, layer_worker, &jobs[t]) == 0;
    if (!ok[t]) layer_worker(&jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t)
    if (ok[t]) pthread_join(tid[t], NULL);
  free(ok);
  free(tid);
  free(jobs);
}

typedef struct {
  const orc_cfg* c;
  const orc_tensors* x;
  const int64_t* rows;
  int lo, hi;
  double *logits, *w;
  int* idx;
} router_job;

static void* router_worker(void* p) {
  router_job* j = (router_job*)p;
  int n = j->c->n_experts, k = j->c->top_k;
  for (int i = j->lo; i < j->hi; ++i)
    orc_router_token(j->c, j->x, j->rows[i], j->logits + (size_t)i * n, j->idx + (size_t)i * k,
                     j->w + (size_t)i * k);
  return NULL;
}

void orc_router_batch(const orc_cfg* c, const orc_tensors* x, const int64_t* rows, int nrows,
                      double* logits, int* idx, double* w, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nrows) nthreads = nrows > 0 ? nrows : 1;
  router_job* jobs = (router_job*)calloc((size_t)nthreads, sizeof(router_job));
  pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  int* ok = (int*)calloc((size_t)nthreads, sizeof(int));
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = (router_job){c, x, rows, (int)((long)nrows * t / nthreads),
                           (int)((long)nrows * (t + 1) / nthreads), logits, w, idx};
    ok[t] = pthread_create(&tid[t], NULL, router_worker, &jobs[t]) == 0;
    if (!ok[t]) router_worker(&jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t)
    if (ok[t]) pthread_join(tid[t], NULL);
  free(ok);
  free(tid);
  free(jobs);
}

typedef struct {
  const orc_cfg* c;
  const void *wg, *wd;
  const float* gamma;
  const double* z;
  double *srow, *nrow;
  int lo, hi;
} expert_job;

static void* expert_worker(void* p) {
  expert_job* j = (expert_job*)p;
  int E = expert_in(j->c);
  for (int r = j->lo; r < j->hi; ++r)
    expert_token_parts(j->c, j->wg, j->wd, j->gamma, j->z + (size_t)r * E,
                       j->srow ? j->srow + (size_t)r * E : NULL, j->nrow + (size_t)r * E);
  return NULL;
}

void orc_expert_batch(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                      const float* gamma_expert, const double* z_rows, int nrows, double* n_rows,
                      int nthreads) {
  orc_expert_batch_parts(c, w_gu_e, w_down_e, gamma_expert, z_rows, nrows, NULL, n_rows, nthreads);
}

void orc_expert_batch_parts(const orc_cfg* c, const void* w_gu_e, const void* w_down_e,
                            const float* gamma_expert, const double* z_rows, int nrows,
                            double* s_rows, double* n_rows, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nrows) nthreads = nrows > 0 ? nrows : 1;
  expert_job* jobs = (expert_job*)calloc((size_t)nthreads, sizeof(expert_job));
  pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
  int* ok = (int*)calloc((size_t)nthreads, sizeof(int));
  for (int t = 0; t < nthreads; ++t) {
    jobs[t] = (expert_job){c, w_gu_e, w_down_e, gamma_expert, z_rows, s_rows, n_rows,
                           (int)((long)nrows * t / nthreads), (int)((long)nrows * (t + 1) / nthreads)};
    ok[t] = pthread_create(&tid[t], NULL, expert_worker, &jobs[t]) == 0;
    if (!ok[t]) expert_worker(&jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t)
    if (ok[t]) pthread_join(tid[t], NULL);
  free(ok);
  free(tid);
  free(jobs);
}

/* ------------------------------------------------------------------ noisy gate statistics */

static double softplus(double z) { return z > 30.0 ? z : log1p(exp(z)); }
static double std_normal_cdf(double z) { return 0.5 * erfc(-z / sqrt(2.0)); }

void orc_noisy_gate_token(const double* l, const double* m, const double* eps, int n, int k,
                          double* H, double* G, double* P, int* idx) {
  char* taken = (char*)calloc((size_t)n, 1);
  for (int i = 0; i < n; ++i) {
    H[i] = l[i] + eps[i] * softplus(m[i]);
    G[i] = 0.0;
  }
  /* KeepTopK: the k largest H (ties to the lower index), then a softmax over them */
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < n; ++e)
      if (!taken[e] && (best < 0 || H[e] > H[best])) best = e;
    taken[best] = 1;
    idx[j] = best;
  }
  double mx = H[idx[0]], z = 0.0;
  for (int j = 0; j < k; ++j) z += exp(H[idx[j]] - mx);
  for (int j = 0; j < k; ++j) G[idx[j]] = exp(H[idx[j]] - mx) / z;
  /* kth_excluding(H, k, i): the k-th largest H among the experts other than i */
  for (int i = 0; i < n; ++i) {
    int rank = 0; /* how many of the others have been taken so far in descending order */
    double kth = 0.0;
    char* used = (char*)calloc((size_t)n, 1);
    used[i] = 1;
    while (rank < k) {
      int best = -1;
      for (int e = 0; e < n; ++e)
        if (!used[e] && (best < 0 || H[e] > H[best])) best = e;
      used[best] = 1;
      kth = H[best];
      ++rank;
    }
    free(used);
    P[i] = std_normal_cdf((l[i] - kth) / softplus(m[i]));
  }
  free(taken);
}

double orc_cv_squared(const double* v, int n) {
  double mean = 0.0, var = 0.0;
  for (int i = 0; i < n; ++i) mean += v[i];
  mean /= n;
  for (int i = 0; i < n; ++i) var += (v[i] - mean) * (v[i] - mean);
  var /= n;
  return var / (mean * mean);
}

/* ------------------------------------------------------------------ permutation */

/* Dispatch "tokens to selected experts" [MUSE "Latent experts"] in the canonical order: count
 * rows per expert, exclusive prefix sum, then hand out rows scanning slots in (token, slot)
 * order, so rows of one expert are in token order. */
int orc_permutation(int T, int k, int n, const int32_t* idx, int32_t* offsets,
                    int32_t* perm_token, int32_t* inv_perm) {
  int32_t* cnt = (int32_t*)calloc((size_t)n, sizeof(int32_t));
  int rc = 0;
  for (int t = 0; t < T && rc == 0; ++t)
    for (int j = 0; j < k; ++j) {
      int e = idx[(size_t)t * k + j];
      if (e < 0 || e >= n) { rc = -1; break; }
      for (int jj = 0; jj < j; ++jj)
        if (idx[(size_t)t * k + jj] == e) rc = -1;
      cnt[e]++;
    }
  if (rc == 0) {
    offsets[0] = 0;
    for (int e = 0; e < n; ++e) offsets[e + 1] = offsets[e] + cnt[e];
    memset(cnt, 0, sizeof(int32_t) * (size_t)n);
    for (int t = 0; t < T; ++t)
      for (int j = 0; j < k; ++j) {
        int e = idx[(size_t)t * k + j];
        int row = offsets[e] + cnt[e]++;
        perm_token[row] = t;
        inv_perm[(size_t)t * k + j] = row;
      }
  }
  free(cnt);
  return rc;
}
