/* Oracle for one GPT-2-style training step -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU definition of what the step computes, used by the
 * tests, the smoke check and the benchmark's CPU-baseline leg to judge the CUDA library.
 * It shares no code, header, table or helper with the CUDA library; nothing in the
 * product path may link or call it.
 *
 * Every entry point exists twice: *_f32 computes in float (the timed baseline) and *_f64
 * computes in double (finite differences and the strict parity reference). Grad-norm sums
 * are taken in double in both.
 *
 * Flat parameter order (row-major [out, in] weights):
 *   wte [Vp,C], wpe [max_T,C],
 *   per layer: ln1.g [C], w_qkv [3C,C], w_attnproj [C,C], ln2.g [C], w_fc [mC,C], w_mlpproj [C,mC],
 *   lnf.g [C].
 */
#ifndef GPT_ORACLE_H
#define GPT_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int vocab;          /* V: ids 0..V-1 take part in the softmax                     */
  int vocab_padded;   /* Vp >= V: rows of wte (padding rows are outside the softmax) */
  int n_layer, n_head, n_embd, max_T, mlp_mult;
  const int *window_left; /* n_layer entries; <0 full causal; w>=0: keys j in [i-w, i] */
  double ln_eps;      /* 1e-5 */
} oracle_cfg;

size_t oracle_num_params(const oracle_cfg *c);
/* Writes up to cap (offset, numel) pairs in layout order; returns the tensor count. */
int oracle_layout(const oracle_cfg *c, int64_t *offsets, int64_t *numels, int cap);

/* Forward only: returns the mean loss; per_token_loss [B*T] may be NULL. */
double oracle_forward_f64(const oracle_cfg *c, const double *params, const int *tokens,
                          const int *targets, int B, int T, double *per_token_loss);
float oracle_forward_f32(const oracle_cfg *c, const float *params, const int *tokens,
                         const int *targets, int B, int T, float *per_token_loss);

/* Forward + backward: grads (same layout as params) are overwritten with dloss/dparams. */
double oracle_forward_backward_f64(const oracle_cfg *c, const double *params, const int *tokens,
                                   const int *targets, int B, int T, double *grads,
                                   double *per_token_loss);
float oracle_forward_backward_f32(const oracle_cfg *c, const float *params, const int *tokens,
                                  const int *targets, int B, int T, float *grads,
                                  float *per_token_loss);

/* sqrt(sum g^2), summed in double. */
double oracle_grad_norm_f64(size_t n, const double *g);
double oracle_grad_norm_f32(size_t n, const float *g);

/* One AdamW step on n elements with t = step (>= 1); gradient used is coef * g. */
void oracle_adamw_f64(size_t n, double *p, const double *g, double *m, double *v, double lr,
                      double wd, double beta1, double beta2, double eps, long step, double coef);
void oracle_adamw_f32(size_t n, float *p, const float *g, float *m, float *v, float lr, float wd,
                      float beta1, float beta2, float eps, long step, float coef);

/* Whole step: forward, backward (raw grads out), clip coefficient, AdamW. Returns the loss;
 * *grad_norm receives the unclipped global norm. */
double oracle_train_step_f64(const oracle_cfg *c, double *params, double *grads, double *m,
                             double *v, const int *tokens, const int *targets, int B, int T,
                             double lr, double wd, double clip, double beta1, double beta2,
                             double eps, long step, double *grad_norm);
float oracle_train_step_f32(const oracle_cfg *c, float *params, float *grads, float *m, float *v,
                            const int *tokens, const int *targets, int B, int T, float lr,
                            float wd, float clip, float beta1, float beta2, float eps, long step,
                            double *grad_norm);

/* One optimizer step over n_micro micro-batches of B x T tokens (gradient accumulation; llm.c
 * summary, "Ejecución"): loss = mean over all n_micro*B*T positions = mean of the micro-batch
 * losses; grads = mean of the micro-batch gradients (raw); then the clip and AdamW of
 * oracle_train_step. Micro-batch i holds tokens [i*B*T, (i+1)*B*T). */
double oracle_train_step_accum_f64(const oracle_cfg *c, double *params, double *grads, double *m,
                                   double *v, const int *tokens, const int *targets, int n_micro,
                                   int B, int T, double lr, double wd, double clip, double beta1,
                                   double beta2, double eps, long step, double *grad_norm);
float oracle_train_step_accum_f32(const oracle_cfg *c, float *params, float *grads, float *m,
                                  float *v, const int *tokens, const int *targets, int n_micro,
                                  int B, int T, float lr, float wd, float clip, float beta1,
                                  float beta2, float eps, long step, double *grad_norm);

/* Single pieces, exposed for the oracle's own pins (double only). */
void oracle_layernorm_fwd_f64(const double *x, const double *g, int rows, int C, double eps,
                              double *y, double *mean, double *rstd);
void oracle_layernorm_bwd_f64(const double *x, const double *g, const double *mean,
                              const double *rstd, const double *dy, int rows, int C, double *dx,
                              double *dg);
/* qkv [B,T,3C] (q | k | v, head h at columns h*hd..), o [B,T,C]. */
void oracle_attention_fwd_f64(const double *qkv, int B, int T, int C, int H, int window,
                              double *o);
void oracle_attention_bwd_f64(const double *qkv, const double *dout, int B, int T, int C, int H,
                              int window, double *dqkv);
double oracle_gelu_f64(double x);
double oracle_gelu_grad_f64(double x);
/* Cross-entropy over the first V of Vp logits per row: returns the mean loss; dlogits
 * [rows, Vp] (may be NULL) receives d(mean loss)/dlogits. */
double oracle_cross_entropy_f64(const double *logits, const int *targets, int rows, int V,
                                int Vp, double *dlogits);

/* ---- hybrid Muon + AdamW update (muon_oracle.cpp; nanochat architecture page,
 * "Optimierungsstrategien Muon und AdamW") ---- */
/* Polar Express in place on X (rows x cols, row-major): Frobenius normalisation (x 1.01 + 1e-6)
 * then ns iterations with the coefficient triples coeffs[3*i .. 3*i+2] = (a, b, c); exact, or
 * with bf16 != 0 every matrix the iteration stores rounded to bf16 once formed. */
void oracle_polar_express_f64(double *X, int rows, int cols, const double *coeffs, int ns,
                              int bf16);
/* One optimizer step on n parameters: Muon on the n_mat matrices (offset, rows, cols) with
 * the momentum in m and the factored second moment at v[offset ..], AdamW (step t = step) on
 * every other element; both on coef * g, coef = min(1, clip / (||g|| + 1e-6)). bf16 != 0: the
 * update cast to bf16 and the iteration at bf16 (oracle_polar_express_f64). Returns ||g||. */
double oracle_muon_adamw_f64(size_t n, double *p, const double *g, double *m, double *v,
                             int n_mat, const int64_t *mat_off, const int *mat_rows,
                             const int *mat_cols, double lr, double wd, double beta1,
                             double beta2, double eps, double matrix_lr, double muon_wd,
                             double mu, double beta2_muon, double s_eps, const double *coeffs,
                             int ns, double clip, long step, int bf16);

#ifdef __cplusplus
}
#endif
#endif
