/* gpt_step.h -- C ABI of the B200 (sm_100a) GPT-2-style training-step library.
 *
 * One call runs one whole training step of a nanoGPT/GPT-2 decoder on one GPU: token +
 * position embedding, n_layer pre-LayerNorm blocks (causal attention with an optional left
 * window per layer, GELU(tanh) MLP), final LayerNorm, tied lm_head with mean softmax
 * cross-entropy, the full backward pass, a global grad-norm clip and a fused AdamW update.
 * gpt_train_step_accum runs one such update over several micro-batches (gradient
 * accumulation).
 *
 * What the operations follow (pages cited by title and section):
 *   - model and config fields: nanoGPT README (intro: reproduces GPT-2 124M, loads OpenAI's
 *     GPT-2 weights) and the Panthalia "Create a Plugin" page (GPTConfig: block_size,
 *     vocab_size, n_layer, n_head, n_embd, dropout, bias=False);
 *   - per-layer sliding window and the FLOPs count: nanochat architecture page,
 *     "Modellarchitektur und FLOPs-Berechnung";
 *   - loss: NiNo README, "Usage" (F.cross_entropy over the logits, mean reduction);
 *   - clipping: llm.c summary ("Reimplementando el modelo GPT-2 ... con llm.c"),
 *     "Proceso de entrenamiento";
 *   - AdamW order and hyper-parameters held in device memory so a captured step replays
 *     with a new lr: nanochat architecture page, "Optimierungsstrategien Muon und AdamW",
 *     "AdamW Fused Step";
 *   - the flat parameter vector: Panthalia page, "Components of the Example Plugin" (the
 *     model adapter maps the model to and from a flattened tensor);
 *   - gradient accumulation: llm.c summary, "Ejecución" (a total batch of -d tokens reached
 *     with several micro-batches per optimizer step).
 *
 * Threading: a handle is not thread-safe; use one handle per host thread.
 * Errors: every int-returning call returns GPT_OK (0) or a negative GPT_ERR_* code; no C++
 * exception crosses this boundary. gpt_strerror() names a code.
 */
#ifndef GPT_STEP_H
#define GPT_STEP_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPT_OK                  0
#define GPT_ERR_INVALID_ARG    -1  /* NULL handle/pointer, bad enum, bad hyper-parameter      */
#define GPT_ERR_SHAPE          -2  /* config not supported, B > max_B, T > max_T, B*T = 0     */
#define GPT_ERR_ALIGN          -3  /* a device pointer is not 16-byte aligned                 */
#define GPT_ERR_OOM            -4  /* cudaMalloc of the workspace failed                      */
#define GPT_ERR_CUDA           -5  /* a CUDA runtime/driver call failed (see gpt_last_cuda_error) */
#define GPT_ERR_NONFINITE      -6  /* loss or grad norm is NaN/Inf: the update was skipped    */
#define GPT_ERR_DEVICE_TIMEOUT -7  /* a bounded device-side wait expired                      */
#define GPT_ERR_BAD_TOKEN      -8  /* a token id outside [0, vocab) or target outside [0, vocab) */

#define GPT_MAX_TOKENS (1 << 20) /* largest max_B * max_T (tokens of one micro-batch)         */

#define GPT_FP32 0  /* validation mode: fp32 activations and fp32 GEMMs (CUDA cores)          */
#define GPT_BF16 1  /* bf16 operands on tcgen05 tensor cores, fp32 accumulation/master state  */

typedef struct {
  int vocab;             /* V: ids 0..V-1 take part in the softmax                            */
  int vocab_padded;      /* Vp >= V: rows of wte; rows >= V are outside the softmax            */
  int n_layer, n_head, n_embd;
  int max_T;             /* rows of wpe and the largest T a call may use                       */
  int max_B;             /* largest B a call may use (sizes the workspace)                     */
  int mlp_mult;          /* MLP hidden = mlp_mult * n_embd (4 for GPT-2)                      */
  const int *window_left;/* n_layer entries (copied), or NULL for all -1. -1 = full causal;
                            w >= 0 = query i attends keys j with i-w <= j <= i                 */
  float ln_eps;          /* LayerNorm epsilon (1e-5)                                            */
  float beta1, beta2;    /* AdamW betas (0.9, 0.95)                                             */
  float adam_eps;        /* AdamW epsilon (1e-8)                                                */
  int precision;         /* GPT_FP32 or GPT_BF16                                                */
  int lmhead_chunk_rows; /* rows per lm_head backward chunk (0 = library default); the largest
                            B*T*V-shaped buffer the step keeps is chunk_rows * Vp bf16          */
  int recompute_gelu;    /* 1: activation recompute (llm.c summary, "Ejecución", -r): each layer
                            keeps only its MLP pre-activation; the backward recomputes GELU and
                            its derivative from it (saves n_layer-1 activations of B*T*4C) */
} gpt_config;

typedef struct {
  char name[32];         /* e.g. "wte", "h3.w_fc", "lnf.g"                                     */
  long long offset;      /* element offset into the flat fp32 vector                           */
  int ndim;              /* 1 or 2                                                              */
  long long shape[2];    /* row-major [out, in] for weights                                     */
} gpt_tensor_desc;

typedef struct gpt_handle gpt_handle;

/* Validates cfg, computes the parameter layout, allocates the workspace (activations for
 * max_B*max_T tokens, the bf16 weight shadow, device scalars) on the current CUDA device.
 * Returns NULL and sets *status (if non-NULL) on failure. Supported shapes: n_embd % n_head
 * == 0, head_dim in {32, 64, 128} (bf16: n_embd % 64 == 0, head_dim == 64),
 * max_B * max_T <= GPT_MAX_TOKENS, vocab_padded <= 131072. */
gpt_handle *gpt_create(const gpt_config *cfg, int *status);
void gpt_destroy(gpt_handle *h);

/* Number of fp32 elements in the flat params/grads/adam_m/adam_v vectors. */
size_t gpt_num_params(const gpt_handle *h);

/* Writes up to cap descriptors in flat order: wte [Vp,C], wpe [max_T,C], per layer
 * (ln1.g [C], w_qkv [3C,C], w_attnproj [C,C], ln2.g [C], w_fc [mC,C], w_mlpproj [C,mC]),
 * lnf.g [C]. Returns the number of tensors (6*n_layer + 3), or a negative code. */
int gpt_param_layout(const gpt_handle *h, gpt_tensor_desc *out, int cap);

/* All device work of later calls is ordered on this cudaStream_t (NULL = legacy default).
 * Inside a training call, the backward's weight-gradient GEMMs and LayerNorm dgamma sums
 * run on a second stream that the handle owns. That stream forks from this one and joins
 * back into it, through events, before the call's last kernels. So work the caller enqueues
 * on this stream after the call sees every result, and a graph captured on this stream
 * holds both branches. */
int gpt_set_stream(gpt_handle *h, void *cuda_stream);

/* Forward pass only. params: device fp32 [num_params], read only. tokens, targets: int32
 * [B,T] row-major, device memory or host memory (host buffers are copied in; pinned host
 * memory keeps the copy asynchronous). loss: host float, the mean cross-entropy.
 * per_token_loss: NULL or device fp32 [B,T]. Blocks until the loss is on the host. */
int gpt_forward_loss(gpt_handle *h, const float *params, const int *tokens, const int *targets,
                     int B, int T, float *loss, float *per_token_loss);

/* One training step with t = (current step) + 1:
 *   forward -> loss; backward -> grads (RAW, unclipped, overwritten; every element written);
 *   norm = ||grads||_2; coef = min(1, clip / (norm + 1e-6));
 *   AdamW on coef*grads: p *= 1 - lr*wd; m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
 *   p -= (lr / (1-b1^t)) * m / (sqrt(v / (1-b2^t)) + eps).
 * params, adam_m, adam_v: device fp32 [num_params], updated in place (caller-owned; adam_m
 * and adam_v start zeroed). grads: device fp32 [num_params], written. tokens/targets as in
 * gpt_forward_loss. loss: host float. Weight decay applies to every element.
 * On GPT_ERR_NONFINITE, GPT_ERR_BAD_TOKEN and GPT_ERR_DEVICE_TIMEOUT the update is skipped:
 * params, adam_m, adam_v (and the handle's bf16 weight copy) are unchanged and the step
 * counter does not advance; grads then hold whatever the failed backward wrote. */
int gpt_train_step(gpt_handle *h, float *params, float *grads, float *adam_m, float *adam_v,
                   const int *tokens, const int *targets, int B, int T, float lr, float wd,
                   float clip, float *loss);

/* Gradient accumulation (llm.c summary, "Ejecución": a total batch of -d tokens reached with
 * several micro-batches per optimizer step): one optimizer step over n_micro >= 1 micro-batches
 * of B x T tokens. tokens/targets hold n_micro*B*T ids (device or host), micro-batch i at
 * offset i*B*T. The loss is the mean over all n_micro*B*T positions (with equal micro-batches,
 * the mean of the micro-batch losses); grads (RAW, written) are its gradient, the mean of the
 * micro-batch gradients, accumulated in fp32 in the grads buffer; then one clip and one AdamW
 * update exactly as in gpt_train_step, which is this call with n_micro = 1. Peak memory is that
 * of one micro-batch. Errors and GPT_ERR_NONFINITE (any micro-batch's loss or the norm) as in
 * gpt_train_step. */
int gpt_train_step_accum(gpt_handle *h, float *params, float *grads, float *adam_m,
                         float *adam_v, const int *tokens, const int *targets, int n_micro,
                         int B, int T, float lr, float wd, float clip, float *loss);

/* ---- data parallelism with sharded optimizer state --------------------------------------
 * The pieces of one data-parallel step (the nanoGPT README's DDP reproduction, "reproducing
 * GPT-2", and the llm.c summary, "Ejecución": ZeRO-1, the optimizer state split across
 * ranks). Each rank runs gpt_forward_backward on its own batch; the caller reduce-scatters
 * the gradients (the rank keeps the sum over ranks of its own ranges), all-reduces one
 * gpt_sumsq per rank into the global sum of squares, runs gpt_adamw_ranges on its ranges and
 * all-gathers the parameters. The collectives belong to the caller (NCCL, for instance). */

/* Forward and backward over n_micro micro-batches (layout as gpt_train_step_accum), no
 * clip, no update, step counter unchanged: grads (written) = grad_scale * d(mean loss over
 * the n_micro*B*T positions)/d(params). With grad_scale = 1/world_size the SUM of the ranks'
 * grads is the gradient of the global mean loss. loss: host, this call's mean loss.
 * GPT_ERR_NONFINITE when a loss is not finite (grads are written all the same). */
int gpt_forward_backward(gpt_handle *h, const float *params, float *grads, const int *tokens,
                         const int *targets, int n_micro, int B, int T, float grad_scale,
                         float *loss);

/* *sumsq_dev (a device double, 8-byte aligned) = sum over x[0..n) of x^2: device fp32 x,
 * 16-byte aligned; float sums per thread, double across them, in a fixed order. Enqueued on
 * the handle's stream; does not synchronise. */
int gpt_sumsq(gpt_handle *h, const float *x, size_t n, double *sumsq_dev);

/* AdamW (the arithmetic of gpt_train_step) on nranges <= 64 parameter ranges: range k is
 * params[offsets[k] .. offsets[k]+counts[k]) (offsets, counts: host arrays, multiples of 4);
 * its gradients and moments are stored compactly: grads, adam_m, adam_v hold the ranges one
 * after the other (range k at sum_{j<k} counts[j]). The clip coefficient is
 * min(1, clip / (sqrt(*sumsq_dev) + 1e-6)) with *sumsq_dev the global sum of squares in device
 * memory; nothing is updated when it is not finite. step: t >= 1 of the bias corrections
 * (the handle's counter is not used or changed). The bf16 weight copy is marked stale. */
int gpt_adamw_ranges(gpt_handle *h, float *params, const float *grads, float *adam_m,
                     float *adam_v, const long long *offsets, const long long *counts,
                     int nranges, float lr, float wd, float clip, const double *sumsq_dev,
                     long step);

/* ---- hybrid Muon + AdamW optimizer --------------------------------------------------------
 * nanochat architecture page, "Optimierungsstrategien Muon und AdamW": Muon for the 2-D block
 * matrices (w_qkv, w_attnproj, w_fc, w_mlpproj of every layer), AdamW for wte (embedding and
 * tied lm_head), wpe and the LayerNorm gains. Per matrix W (rows x cols) on the clipped
 * gradient g = coef * grad, coef = min(1, clip / (||grad|| + 1e-6)):
 *   momentum (Nesterov, lerp form): buf = lerp(buf, g, 1 - momentum); u = lerp(g, buf, momentum)
 *   Polar Express: X = bf16(u) / (||X||_F * 1.01 + 1e-6); per coefficient triple (a, b, c):
 *     rows > cols: A = X^T X, B = b A + c A^2, X = a X + X B; else A = X X^T, X = a X + B X
 *     (bf16 operands, fp32 accumulation, tensor cores; all layers' matrices of one shape batched)
 *   factored second moment: v = mean of X^2 per row (rows > cols) or per column;
 *     s = lerp(s, v, 1 - beta2); X' = X / sqrt(max(s, eps)), rescaled to ||X||_F
 *   cautious update: W -= matrix_lr * X' + matrix_lr * weight_decay * W * [X' * W >= 0]
 * Everything else: the AdamW of gpt_train_step with lr, wd and t = (step counter) + 1.
 * State in the caller's flat adam_m / adam_v: for a matrix, adam_m holds its momentum buffer
 * and adam_v, from the matrix's offset, its second moment (rows or cols floats); both start
 * zeroed. grads: the raw gradient (e.g. from gpt_forward_backward). bf16 mode only
 * (GPT_ERR_SHAPE otherwise). On success the step counter advances; on GPT_ERR_NONFINITE
 * (non-finite norm) nothing is updated. The first call allocates the handle's Muon scratch. */
typedef struct {
  float matrix_lr;      /* Muon learning rate (the page's matrix_lr, 0.02)                   */
  float weight_decay;   /* Muon cautious weight decay (the page: 0.0)                        */
  float momentum;       /* 0.95                                                              */
  float beta2;          /* EMA factor of the factored second moment, 0.95                    */
  float eps;            /* floor of the second moment, 1e-10                                 */
  int ns_steps;         /* Polar Express iterations (the page: 5), <= 16                     */
  const float *coeffs;  /* host, ns_steps triples (a, b, c)                                  */
} gpt_muon_config;
int gpt_muon_update(gpt_handle *h, float *params, const float *grads, float *adam_m,
                    float *adam_v, const gpt_muon_config *mc, float lr, float wd, float clip);

/* Step counter (number of completed AdamW updates); gpt_set_step is for resuming. */
int gpt_get_step(const gpt_handle *h, long *step);
int gpt_set_step(gpt_handle *h, long step);

/* Unclipped global grad norm of the last gpt_train_step (NaN before the first). */
float gpt_last_grad_norm(const gpt_handle *h);

/* In bf16 mode the step keeps a bf16 copy of the weights that AdamW refreshes. Call this
 * after changing params outside gpt_train_step (e.g. loading a checkpoint into the same
 * buffer); a different params pointer is detected automatically. */
int gpt_params_changed(gpt_handle *h);

/* Options (gpt_set_option): capture each (B,T) step shape into a CUDA graph (default 1);
 * record CUDA events around every GEMM launch for kernel timing (default 0). */
#define GPT_OPT_USE_GRAPHS 1
#define GPT_OPT_TIME_KERNELS 2
int gpt_set_option(gpt_handle *h, int option, long value);

/* Kernel timings accumulated by GPT_OPT_TIME_KERNELS since the last reset: CUDA events on the
 * step's stream around each launch of the class `kind` (CUDA graphs are off while timing).
 * *launches, *total_ms, and *work = the launches' ALGORITHMIC work:
 *   GPT_KSTAT_GEMM            every tensor-core GEMM launch's time; work = FLOPs (2*M*N*K) of the
 *                             method's own contractions (block GEMMs, lm_head forward, dX, dwte),
 *                             the cross-entropy backward's logits recompute excluded
 *   GPT_KSTAT_GEMM_RECOMPUTE  that logits recompute alone (executed FLOPs)
 *   GPT_KSTAT_ATTN_FWD / _BWD FLOPs: 4*hd (forward) and 8*hd (backward) per admitted score
 *                             (the backward's recompute of the scores not counted)
 *   GPT_KSTAT_LN_FWD          bytes: bf16 x read, y written, mean/rstd written (4C+8 per row)
 *   GPT_KSTAT_LN_BWD          bytes: x, dy, residual gradient read, residual gradient written
 *                             (8C+8 per row in bf16; the first has no residual input)
 *   GPT_KSTAT_EMBED_FWD/_BWD  bytes: wte and wpe rows read, x written (6C per token);
 *                             dx read once and dwpe written (the per-id fp32 rows not counted)
 *   GPT_KSTAT_CE              bytes of the cross-entropy combine (statistics read)
 *   GPT_KSTAT_GRAD_NORM       bytes: 4 per parameter
 *   GPT_KSTAT_ADAMW           bytes: 30 per parameter in bf16 mode (p, g, m, v read; p, m, v
 *                             and the bf16 copy written), 28 in fp32 mode
 * Reading any kind with reset != 0 clears all of them. */
#define GPT_KSTAT_GEMM 0
#define GPT_KSTAT_GEMM_RECOMPUTE 1
#define GPT_KSTAT_ATTN_FWD 2
#define GPT_KSTAT_ATTN_BWD 3
#define GPT_KSTAT_LN_FWD 4
#define GPT_KSTAT_LN_BWD 5
#define GPT_KSTAT_EMBED_FWD 6
#define GPT_KSTAT_EMBED_BWD 7
#define GPT_KSTAT_CE 8
#define GPT_KSTAT_GRAD_NORM 9
#define GPT_KSTAT_ADAMW 10
#define GPT_KSTAT_MUON 11          /* gpt_muon_update's Muon part per matrix group: FLOPs of
                                      the Polar Express GEMMs */
#define GPT_KSTAT_COUNT 12
int gpt_kernel_stats(gpt_handle *h, int kind, long long *launches, double *total_ms,
                     double *work, int reset);

/* Number of kernels the last gpt_train_step / gpt_forward_loss enqueued. */
int gpt_last_launch_count(const gpt_handle *h);

const char *gpt_strerror(int status);
/* Text of the last CUDA error seen by this handle ("" if none). */
const char *gpt_last_cuda_error(const gpt_handle *h);

#ifdef __cplusplus
}
#endif
#endif /* GPT_STEP_H */
