/*
 * moe.h - C ABI of the B200 (sm_100a) forward pass of a top-k softmax-routed (latent)
 * mixture-of-experts layer:  y = sum_i G(x)_i E_i(x)  with the Muse latent-expert structure.
 *
 * The operations and where they are defined:
 *   [SHAZEER] "816 billion parameters, and only 42 billion show up for each token"
 *             (bobbyburns.tech), sections "The math" (y = sum_i G(x)_i E_i(x), ReLU experts,
 *             experts with G_i = 0 are not evaluated) and "The gate" (Softmax(KeepTopK)).
 *   [MUSE]    "Muse Spark Open: Norm-Preserving Gates Are Not a Norm Guarantee" (flozi.net),
 *             sections "Two normalization orders implement different functions" (R_eps, C_gamma,
 *             I_gamma), "Latent experts: normalization happens before the weighted sum" (latent
 *             8192->4096 projection, C_pre, dispatch, SwiGLU experts, per-expert I_gamma before the
 *             weighted sum), "Residual gates: derive the advertised intuition carefully" (learned
 *             residual gate) and "What this means for serving and kernel work" (precision
 *             contract, legal fusions).
 *   [ARCHDB]  "Muse-Spark-Open-816B-A42B" model sheet: renormalised top-k weights,
 *             routed_scaling_factor, latent width 4096, residual gate formula, no FFN biases.
 *
 * Conventions shared by every call:
 *   - Every call returns a moe_status_t.  Argument, size, alignment and workspace errors are
 *     detected on the host before anything is launched, and nothing is launched then.
 *   - Pointers are DEVICE pointers owned by the caller.  The library allocates no device memory;
 *     calls that need scratch take a caller-provided workspace (size from moe_workspace_size).
 *   - Calls are asynchronous on the given CUDA stream (cudaStream_t passed as void*; NULL is the
 *     legacy default stream).  Buffers must stay valid until the stream reaches the call.
 *   - Tensors are dense row-major.  bf16 values are passed as their 16-bit patterns.  Every
 *     pointer must be 16-byte aligned (MOE_ERR_ALIGNMENT otherwise).
 *   - Inputs are never written.  Outputs must not alias inputs, except that the residual r of
 *     moe_layer_forward may be the same buffer as u.
 *   - Device-side consistency checks (an out-of-range expert index, a bounded wait that ran out)
 *     latch an error code in a per-device status word instead of trapping; the computation is
 *     skipped for the offending element.  moe_get_device_status synchronises the stream, reads
 *     and clears it.
 *   - Supported shapes: bf16 with d_model, d_latent, d_ff multiples of 64, 1 <= n_experts <= 256,
 *     1 <= top_k <= min(8, n_experts); fp32 (CUDA-core path, for small layers) with no latent
 *     projection.  Anything else returns MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* NULL where a buffer is required, inconsistent sizes */
  MOE_ERR_UNSUPPORTED = 2,   /* shape or mode outside the supported set */
  MOE_ERR_ALIGNMENT = 3,     /* a pointer not 16-byte aligned */
  MOE_ERR_WORKSPACE = 4,     /* workspace missing or smaller than moe_workspace_size */
  MOE_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed (launch, tensor map) */
  MOE_ERR_TIMEOUT = 6,       /* device: a bounded wait inside a kernel ran out */
  MOE_ERR_DEVICE_CHECK = 7   /* device: an index failed its range check */
} moe_status_t;

enum { MOE_F32 = 0, MOE_BF16 = 1 };
enum { MOE_ACT_RELU = 0, MOE_ACT_SWIGLU = 1 };
enum { MOE_RESID_NONE = 0, MOE_RESID_MUSE_GATE = 1, MOE_RESID_LITERAL = 2 };
enum { MOE_GATE_SOFTMAX = 0, MOE_GATE_SIGMOID = 1 };

typedef struct {
  int32_t T;            /* tokens */
  int32_t d_model;      /* width of u, r and the layer output */
  int32_t d_latent;     /* latent width L of the expert path; 0 = no latent projections */
  int32_t d_ff;         /* expert hidden width: ReLU hidden h, or SwiGLU intermediate I */
  int32_t n_experts;    /* n */
  int32_t top_k;        /* k */
  int32_t dtype;        /* MOE_F32 | MOE_BF16 (activations and weights; accumulation is fp32) */
  int32_t expert_act;   /* MOE_ACT_RELU (E(x) = W2 ReLU(W1 x)) | MOE_ACT_SWIGLU */
  int32_t pre_norm;     /* 1: z = C_pre(P_down u) (centred RMSNorm, gain 1+gamma_pre) */
  int32_t expert_norm;  /* 1: each expert output goes through I_gamma before weighting */
  int32_t resid_mode;   /* MOE_RESID_NONE | MOE_RESID_MUSE_GATE | MOE_RESID_LITERAL */
  float eps;            /* RMSNorm epsilon (both norms) */
  float tau;            /* residual gate temperature */
  float resid_floor;    /* residual gate floor delta on alpha^2 */
  float routed_scale;   /* routed_scaling_factor applied to the renormalised weights */
  int32_t gate_mode;    /* MOE_GATE_SOFTMAX (softmax, keep top k, renormalise) |
                           MOE_GATE_SIGMOID (Muse: sigmoid scores, selection by score + correction
                           bias, weights = score / (sum of selected scores + 1e-15)) */
  int32_t router_f32;   /* 1: the router weights are fp32, passed as their exact bf16 split
                           [n, 3*d_model] (hi, mid, lo; see moe_router_split_weights) */
  float logit_mult;     /* output_multiplier on the router logits (sigmoid gate) */
  int32_t input_norm;   /* decoder wrap (bf16): the branch input is u = dtype(C_in(r)), the
                           residual stream's centred RMSNorm (gain 1+gamma_in, eps_block) */
  int32_t post_norm;    /* decoder wrap (bf16, latent): the up-projection b goes through the
                           FFN's input-scaled output norm I_post (gain 1+gamma_post, eps_block)
                           before the residual gate */
  float eps_block;      /* epsilon of the two decoder-level norms */
} moe_config_t;

typedef struct {
  const void* w_router;     /* [n, d_model]                          dtype */
  const void* p_down;       /* [d_latent, d_model]  (latent only)     dtype */
  const void* p_up;         /* [d_model, d_latent]  (latent only)     dtype */
  const void* w_gu;         /* [n, 2*d_ff, E_in] SwiGLU: rows [0, d_ff) gate, [d_ff, 2*d_ff) up;
                               [n, d_ff, E_in] ReLU.  E_in = d_latent, or d_model without latent */
  const void* w_down;       /* [n, E_in, d_ff]                        dtype */
  const float* gamma_pre;   /* [d_latent] (pre_norm only) */
  const float* gamma_expert;/* [E_in] one gain shared by all experts (expert_norm only) */
  const float* resid_g;     /* [d_model] residual gate parameter g (resid_mode != NONE) */
  const float* logit_bias;  /* [n] added to every token's router logits, or NULL */
  const float* correction_bias; /* [n] sigmoid gate: added to the scores for selection only */
  const float* gamma_in;    /* [d_model] input_norm gain */
  const float* gamma_post;  /* [d_model] post_norm gain */
} moe_weights_t;

/* Human-readable name of a status code (static storage). */
MOE_API const char* moe_status_string(moe_status_t s);

/* Bytes of workspace moe_layer_forward needs for this configuration (also an upper bound for
 * moe_permute and moe_expert_ffn).  Only host arithmetic. */
MOE_API moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes);

/* Router [SHAZEER "The gate"; ARCHDB gating fields; MUSE "Latent experts" for the sigmoid gate]:
 *   l = u W_router^T, fp32 accumulation of exact products (bf16 weights, or the exact
 *   hi/mid/lo split of fp32 weights when cfg->router_f32).
 *   Softmax gate: l += logit_bias; the k largest l are selected (ties to the lower expert
 *   index) in descending order; w_j = exp(l_j - l_1) / sum_sel exp(.) * routed_scale, which
 *   equals softmax-then-renormalise over the kept experts.  logits_out returns l.
 *   Sigmoid gate: s = sigmoid(logit_mult * l + logit_bias); the k largest keys
 *   s + correction_bias (one fp32 addition; ties to the lower index) are selected in descending
 *   key order; w_j = s_j / (sum_sel s + 1e-15) * routed_scale.  logits_out returns s.
 * u: [T, d_model]; topk_idx: [T, k] int32; topk_w: [T, k] fp32; logits_out: [T, n] fp32 or
 * NULL; logit_bias, correction_bias: [n] fp32 or NULL. */
MOE_API moe_status_t moe_route(const moe_config_t* cfg, const void* u, const void* w_router,
                       const float* logit_bias, const float* correction_bias, float* logits_out,
                       int32_t* topk_idx, float* topk_w, void* stream);

/* Prepares fp32 router weights w [n, d] for the tensor-core router: w_split [n, 3*d] bf16 holds
 * per row the bf16 parts hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid) (each
 * subtraction exact in fp32), so hi + mid + lo = w exactly for every normal fp32 w with a normal
 * lo part (zero remainders stay exact).  Run once per weight load.  Device pointers, d a
 * multiple of 64. */
MOE_API moe_status_t moe_router_split_weights(const float* w, int32_t n, int32_t d, void* w_split,
                                              void* stream);

/* Dispatch [MUSE "Latent experts"; SHAZEER "The math"]: groups the T*k routed slots by expert
 * in the canonical order (experts ascending; within an expert, tokens ascending), so that every
 * index output is unique and bit-exact:
 *   expert_offsets [n+1] (exclusive prefix sum of per-expert counts), perm_token [T*k]
 *   (row -> token), inv_perm [T*k] (slot t*k+j -> row).
 * If x is not NULL it also gathers rows: x_perm[inv_perm[t*k+j]] = f(x[t]) where x is [T, E_in]
 * and f is C_pre with gain 1+gamma_pre when gamma_pre is not NULL (cfg->pre_norm), else the
 * identity.  workspace: at least moe_workspace_size bytes.  An index outside [0, n) latches
 * MOE_ERR_DEVICE_CHECK and that slot is dropped. */
MOE_API moe_status_t moe_permute(const moe_config_t* cfg, const int32_t* topk_idx,
                         int32_t* expert_offsets, int32_t* perm_token, int32_t* inv_perm,
                         const void* x, const float* gamma_pre, void* x_perm, void* workspace,
                         size_t workspace_bytes, void* stream);

/* The row half of moe_permute, for a caller that already holds the permutation (for example
 * after reading the expert offsets back while another kernel runs): x_perm[inv_perm[t*k+j]] =
 * f(x[t]) with f = C_pre (gain 1+gamma_pre) when gamma_pre is not NULL (bf16 with a latent
 * width), else the identity [MUSE "Latent experts"].  x: [T, E_in]; x_perm: [T*k, E_in];
 * inv_perm: [T*k] as moe_permute returns it (a negative entry skips that slot).  Errors as for
 * moe_permute. */
MOE_API moe_status_t moe_dispatch_rows(const moe_config_t* cfg, const int32_t* inv_perm,
                                       const void* x, const float* gamma_pre, void* x_perm,
                                       void* stream);

/* moe_permute without a workspace argument, for callers that cannot allocate device memory: a
 * plugin or embedding host that hands the library only its input and output buffers (no
 * allocator handle, no scratch pool), or code that may not call cudaMalloc on its path because
 * that call can synchronise the device.  The pages describe no such variant: it exists for this
 * library's callers only.
 *
 * Same arguments, outputs and errors as moe_permute, minus workspace/workspace_bytes.  Its
 * scratch (the per-chunk expert histograms, ceil(T/128) * n_experts int32 values) lives in one
 * device array inside the library of MOE_PERMUTE_STATIC_MAX_COUNTS int32 (256 KB), which every
 * GPU that loads the library keeps until the process exits; it covers T <= 32768 tokens with 256
 * experts (ceil(T/128) * n_experts <= 65536).  Larger sizes return MOE_ERR_WORKSPACE before any
 * launch.  The call allocates nothing.  The first call on each device looks up the array's
 * device address (cudaGetSymbolAddress, with that device current); make that first call before
 * any stream capture on the device.  All calls share the one array and leave their histograms in
 * it: calls that can overlap on the GPU (on different streams, or from several host threads
 * without ordering) race and produce wrong offsets; order them on one stream. */
#define MOE_PERMUTE_STATIC_MAX_COUNTS 65536
MOE_API moe_status_t moe_permute_static(const moe_config_t* cfg, const int32_t* topk_idx,
                                        int32_t* expert_offsets, int32_t* perm_token,
                                        int32_t* inv_perm, const void* x, const float* gamma_pre,
                                        void* x_perm, void* stream);

/* Experts on their routed rows only [MUSE "Latent experts"; SHAZEER "The math"]: for each expert
 * e, rows [expert_offsets[e], expert_offsets[e+1]) of x_perm [T*k, E_in]:
 *   SwiGLU: a = SiLU(x W_gate^T) * (x W_up^T) stored in dtype;  ReLU: a = ReLU(x W1^T);
 *   o = a W_down^T stored in dtype;  with expert_norm: out = dtype((1+gamma_expert) * o), the
 *   scaled vector that I_gamma reduces ([MUSE "Two normalization orders"]), else out = o.
 * out_perm: [T*k, E_in].  workspace holds the activation a.
 * row_sumsq (optional, bf16 with expert_norm only, else ignored): [T*k, P] fp32 with P from
 * moe_row_sumsq_parts; part p of row r is the sum of squares of out's bf16 values over one fixed
 * block of its columns (the blocks partition the row), so that I_gamma's reduction
 * mean(s^2) = (sum_p row_sumsq[r, p]) / E_in needs no second pass over the row (moe_combine). */
MOE_API moe_status_t moe_expert_ffn(const moe_config_t* cfg, const void* x_perm,
                            const int32_t* expert_offsets, const void* w_gu, const void* w_down,
                            const float* gamma_expert, void* out_perm, float* row_sumsq,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Number of partial sums of squares per row (P) that moe_expert_ffn writes to row_sumsq for this
 * configuration (host arithmetic only). */
MOE_API moe_status_t moe_row_sumsq_parts(const moe_config_t* cfg, int32_t* parts);

/* Normalise and combine [MUSE "Latent experts" (normalise each expert output, then weight and
 * accumulate); SHAZEER "The math"]: for each token t,
 *   y_t = dtype( sum_j topk_w[t,j] * n_j ),  n_j = dtype(s_j / sqrt(mean(s_j^2) + eps)) with
 *   s_j = out_perm[inv_perm[t*k+j]] when expert_norm, else n_j = s_j;  fp32 accumulation in slot
 *   order.  y: [T, E_in].
 * row_sumsq (optional, bf16 with expert_norm): the partial sums of squares moe_expert_ffn wrote
 * for out_perm; mean(s_j^2) is then their sum (in part order) / E_in instead of a reduction over
 * the row here.  NULL: the reduction is done here. */
MOE_API moe_status_t moe_combine(const moe_config_t* cfg, const void* out_perm,
                                 const float* row_sumsq, const int32_t* inv_perm,
                                 const float* topk_w, void* y, void* stream);

/* Latent down-projection [MUSE "Latent experts"]: z_raw = dtype(u P_down^T), [T, d_latent].
 * Up to 64 rows the reduction is split over the CTAs of a thread-block cluster, which add their
 * fp32 partial sums in a fixed order (deterministic; the same bits as moe_layer_forward). */
MOE_API moe_status_t moe_latent_down(const moe_config_t* cfg, const void* u, const void* p_down,
                             void* z_raw, void* stream);

/* Latent up-projection and residual update [MUSE "Residual gates"; ARCHDB residual field]:
 *   b = dtype(y P_up^T); out = dtype(alpha*r + beta*b) with beta = sigmoid(g/tau),
 *   alpha = sqrt(max(sigmoid(-g/tau)*(1+beta), resid_floor)) per channel (MUSE_GATE), or
 *   dtype(r + g*b) (LITERAL), or b (NONE).  y: [T, d_latent]; r, out: [T, d_model].  Up to 64
 * rows the reduction is split as in moe_latent_down. */
MOE_API moe_status_t moe_latent_up(const moe_config_t* cfg, const void* y, const void* p_up,
                           const void* r, const float* resid_g, void* out, void* stream);

/* Residual update of the decoder layer's FFN sub-block [MUSE "The complete layer has two
 * separately normalized residual updates", "Residual gates"]: for each row,
 *   n = b, or with gamma_post (cfg->post_norm) the input-scaled output norm
 *   n = dtype(s / sqrt(mean(s^2) + eps_block)), s = dtype((1 + gamma_post) * b);
 *   out = dtype(alpha*r + beta*n) (MUSE_GATE), dtype(r + g*n) (LITERAL) or n (NONE).
 * b, r, out: [T, d_model] bf16; gamma_post, resid_g: [d_model] fp32.  bf16 only. */
MOE_API moe_status_t moe_residual_update(const moe_config_t* cfg, const void* b, const void* r,
                                         const float* gamma_post, const float* resid_g, void* out,
                                         void* stream);

/* Shazeer et al.'s noisy top-k gate and its balancing statistics [SHAZEER "The gate", "Keeping the
 * experts busy"] for a batch of T tokens u [T, d_model]:
 *   l = u W_router^T, m = u W_noise^T (fp32 accumulation; W_noise [n, d_model] in the router's
 *   format), H = l + eps * softplus(m) with the standard-normal draws noise_eps [T, n] (fp32,
 *   supplied by the caller);
 *   G = Softmax(KeepTopK(H, k)): topk_idx [T, k] (ties to the lower index, descending) and
 *   topk_w [T, k];
 *   P_i = Phi((l_i - kth_excluding(H, k, i)) / softplus(m_i)) (optional copy load_prob_out
 *   [T, n]); importance[n] = sum_t G, load[n] = sum_t P (fp32, deterministic order), cv2[0] =
 *   CV(importance)^2 and cv2[1] = CV(load)^2 with the population variance.
 * noisy_logits_out [T, n] (H) and load_prob_out may be NULL.  Needs top_k < n_experts and T > 0;
 * workspace of moe_noisy_gate_workspace_size bytes.  cfg->gate_mode is ignored (the two logit
 * passes are plain logits); logit_bias does not apply. */
MOE_API moe_status_t moe_noisy_gate_workspace_size(const moe_config_t* cfg, size_t* bytes);
MOE_API moe_status_t moe_noisy_gate(const moe_config_t* cfg, const void* u, const void* w_router,
                                    const void* w_noise, const float* noise_eps,
                                    float* noisy_logits_out, int32_t* topk_idx, float* topk_w,
                                    float* load_prob_out, float* importance, float* load,
                                    float* cv2, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* The whole layer: [input norm] -> route -> latent down (+C_pre) -> dispatch -> experts
 * (+I_gamma prep) -> normalise and combine -> latent up -> [output norm] -> residual update.
 * u: [T, d_model] is the branch input (router and down-projection read it; with input_norm it
 * is computed from r and this argument may be NULL), r: [T, d_model] the residual stream (may
 * equal u; ignored when resid_mode is NONE and input_norm is off), out: [T, d_model].
 * logits_out [T, n], topk_idx_out [T, k] and topk_w_out [T, k] are optional copies of the
 * routing.  The workspace holds every intermediate.  With T <= 64 (bf16, latent) the two latent
 * projections split their reduction over k ranges and add the fp32 partials in a fixed order (the
 * same bits as moe_latent_down / moe_latent_up, which split the same way), so their results are
 * deterministic but may differ in the last bit from a forward of more than 64 tokens. */
MOE_API moe_status_t moe_layer_forward(const moe_config_t* cfg, const moe_weights_t* w, const void* u,
                               const void* r, void* out, float* logits_out,
                               int32_t* topk_idx_out, float* topk_w_out, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Intermediate values of one whole-layer forward, copied out for verification (the intermediates
 * the precision contract fixes [MUSE "Latent experts: normalization happens before the weighted
 * sum", "What this means for serving and kernel work"]).  Every pointer is a caller-owned device
 * buffer, or NULL to skip that value; E_in = d_latent, or d_model without latent projections.
 *   z        [T, E_in]    each token's expert input as dispatched: dtype(C_pre(z_raw)) with
 *                         pre_norm, z_raw = dtype(u P_down^T) without, or u (no latent).
 *   s        [T*k, E_in]  each dispatched row's expert output before its norm: dtype((1+gamma) o)
 *                         with expert_norm, else o; in dispatch order (token t's slot j is row
 *                         inv_perm[t*k+j]).
 *   y        [T, E_in]    the weighted combine y = dtype(sum_j w_j n_j).
 *   inv_perm [T*k]        the dispatch row of every slot (int32). */
typedef struct {
  void* z;
  void* s;
  void* y;
  int32_t* inv_perm;
} moe_layer_taps_t;

/* moe_layer_forward that also copies the intermediates named in *taps (taps may be NULL, which is
 * moe_layer_forward itself).  The forward's kernels and their results are those of
 * moe_layer_forward; each requested value adds one device-to-device copy (z: one gather kernel)
 * on the stream after the stage that produces it.  Tap buffers must be 16-byte aligned and must not
 * overlap any other argument. */
MOE_API moe_status_t moe_layer_forward_taps(const moe_config_t* cfg, const moe_weights_t* w,
                                            const void* u, const void* r, void* out,
                                            float* logits_out, int32_t* topk_idx_out,
                                            float* topk_w_out, const moe_layer_taps_t* taps,
                                            void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device staging moe_layer_forward_host needs for this configuration: two input and two
 * output buffers of T x d_model elements, each rounded up to 256 bytes. */
MOE_API moe_status_t moe_host_staging_size(const moe_config_t* cfg, size_t* bytes);

/* The whole layer (as moe_layer_forward, with the residual r = u) over n_batches batches held in
 * HOST memory: batch i's input u_host[i] [T, d_model] is copied to the device, the layer runs on
 * it and its output is copied back to out_host[i] [T, d_model].  u_host and out_host are host
 * arrays of n_batches host pointers; the buffers should be page-locked (cudaHostAlloc /
 * cudaHostRegister), or the copies are not asynchronous.
 *   - The copies run on two copy streams owned by the library, in double-buffered device staging
 *     (moe_host_staging_size bytes, caller-owned, 16-byte aligned).  Batch i+1's input copy and
 *     batch i-1's output copy therefore overlap batch i's kernels, which run on `stream` in order.
 *   - The copy streams start after the work already queued on `stream`; when `stream` reaches
 *     the end of the call's work, every output copy has completed.  Synchronise `stream` before
 *     reading out_host.
 *   - Batches share the workspace.  Logits and routing copies are not returned.
 *   - Errors: MOE_ERR_INVALID_ARG for n_batches < 0 or a NULL array or entry, MOE_ERR_WORKSPACE for
 *     missing or short staging or workspace, MOE_ERR_ALIGNMENT for unaligned staging; any error
 *     moe_layer_forward returns for the first batch stops the call before it queues anything.
 *   - Not thread-safe per device: one host pipeline per device at a time. */
MOE_API moe_status_t moe_layer_forward_host(const moe_config_t* cfg, const moe_weights_t* w,
                                            int32_t n_batches, const void* const* u_host,
                                            void* const* out_host, void* staging,
                                            size_t staging_bytes, void* workspace,
                                            size_t workspace_bytes, void* stream);

/* Row gather [SHAZEER "Connecting the dots": the experts' batches pooled across devices], the
 * data movement of an expert-parallel exchange (regrouping rows received from several ranks by
 * expert, and back): dst[i, :] = src[rows[i], :] for i < n_rows, each row
 * row_bytes long (a multiple of 16).  rows[i] < 0 writes a zero row; rows[i] >= src_rows latches
 * MOE_ERR_DEVICE_CHECK and writes a zero row.  src, rows and dst are device pointers, 16-byte
 * aligned; dst must not overlap src.  Errors: MOE_ERR_INVALID_ARG (NULL with n_rows > 0,
 * negative sizes), MOE_ERR_UNSUPPORTED (row_bytes not a positive multiple of 16),
 * MOE_ERR_ALIGNMENT. */
MOE_API moe_status_t moe_gather_rows(const void* src, int64_t src_rows, const int32_t* rows,
                                     int64_t n_rows, int64_t row_bytes, void* dst, void* stream);

/* Synchronises the stream, returns and clears the device status word of the current device
 * (MOE_OK if no kernel latched an error since the last call). */
MOE_API moe_status_t moe_get_device_status(void* stream);

/* Stage timing of moe_layer_forward, for measurement (not part of the layer's definition).
 * moe_profile_begin(max_calls) creates CUDA events for up to max_calls forward calls on the
 * current device; each following moe_layer_forward call records MOE_PROFILE_STAGES + 1 events on
 * its stream around its stages, in this order:
 *   0 route, 1 latent down-projection, 2 dispatch (permute + row scatter), 3 expert gate/up (or
 *   ReLU) GEMM, 4 expert down GEMM, 5 normalise + combine, 6 latent up-projection + residual.
 * Stages a configuration does not have take zero time.  moe_profile_end synchronises on the
 * last recorded event, writes the summed milliseconds of each stage over the recorded calls to
 * stage_ms[MOE_PROFILE_STAGES] and the number of recorded calls to *calls, destroys the events
 * and stops recording.  Calls beyond max_calls are not recorded.  Not thread-safe: one profiling
 * session per process at a time. */
#define MOE_PROFILE_STAGES 7
MOE_API moe_status_t moe_profile_begin(int32_t max_calls);
MOE_API moe_status_t moe_profile_end(float* stage_ms, int32_t* calls);

/* Number of CUDA kernels this library has launched in this process (host-side counter, for
 * measurement: the difference across a region is the kernels that region launched). */
MOE_API unsigned long long moe_launch_count(void);

/* Self-test of the device-side failure detection (not part of the layer): one thread waits, with
 * the bounded wait the GEMM pipeline uses and a budget of budget_clocks SM clocks (1 .. about 2e9),
 * on an mbarrier that nothing arrives at.  The wait runs out, latches MOE_ERR_TIMEOUT in the
 * device status word (read it with moe_get_device_status) and writes 1 to *gave_up (device
 * int32); the kernel then returns normally and the context stays usable. */
MOE_API moe_status_t moe_selftest_wait_timeout(long long budget_clocks, int32_t* gave_up,
                                               void* stream);

#ifdef __cplusplus
}
#endif
#endif
