// Launchers of the step's kernels. T is the activation type: float (validation mode) or
// bf16. Every launcher enqueues on `st` and returns the launch status.
#pragma once
#include "common.cuh"

// K1: x[m] = wte[tok[m]] + wpe[m % T]; flags ids outside [0, V) (tokens and targets).
template <typename T>
cudaError_t launch_embed_fwd(const int *tok, const int *tgt, const T *wte, const T *wpe, T *x,
                             int M, int Tlen, int C, int V, DevScalars *sc, cudaStream_t st);

// K13: dwpe[t] = sum_b dx[b,t] (rows t >= T zeroed; added to dwpe when accumulate); dwte[id]
// += sum over positions with that id, in position order (deterministic; a stable radix sort of
// the ids over several CTAs, then windowed segment sums). dwte already holds the lm_head part.
struct EmbedBwdWs {
  void *base;  // embed_bwd_ws_bytes(maxM, C) bytes, 256-byte aligned
};
size_t embed_bwd_ws_bytes(int maxM, int C);
int embed_bwd_launches(int Vp);
template <typename T>
cudaError_t launch_embed_bwd(const int *tok, const T *dx, float *dwte, float *dwpe, int M,
                             int Tlen, int maxT, int C, int Vp, EmbedBwdWs ws, cudaStream_t st,
                             bool accumulate = false);

// K2: y = (x - mean) * rstd * g, one warp per row.
template <typename T>
cudaError_t launch_layernorm_fwd(const T *x, const T *g, T *y, float *mean, float *rstd, int M,
                                 int C, float eps, cudaStream_t st);

// K12: dres += LN_backward(dy) (dres = LN_backward(dy) when !dres_in: the incoming residual
// gradient is zero and dres is not read); dgamma partial sums per block -> dg (fp32) after
// reduce (added to dg when accumulate).
template <typename T>
cudaError_t launch_layernorm_bwd(const T *x, const T *g, const float *mean, const float *rstd,
                                 const T *dy, T *dres, float *dg_partial, float *dg, int M,
                                 int C, cudaStream_t st, bool accumulate = false,
                                 bool dres_in = true, bool colsum = true);
// dgamma from the per-block partials of launch_layernorm_bwd(..., colsum = false), in block order
cudaError_t launch_ln_colsum(const float *dg_partial, int M, int C, float *dg, bool accumulate,
                             cudaStream_t st);
int layernorm_bwd_blocks(int M);

// Cross-entropy: per-row lse and loss from the per-tile stats; mean loss into sc->loss.
cudaError_t launch_ce_combine(const float *stats, const float *tgt_logit, float *lse,
                              float *per_token, int M, int ntiles, DevScalars *sc,
                              cudaStream_t st);

// K14: sum of squares of g[0..n) (two-stage, fixed order) -> sc->norm, sc->coef.
cudaError_t launch_grad_norm(const float *g, size_t n, double *partials, DevScalars *sc,
                             cudaStream_t st);
int grad_norm_blocks();

// K15: AdamW with g <- coef*g; skipped when sc->nonfinite or any sc->err bit is set. shadow (bf16, may be NULL)
// receives the rounded new params.
cudaError_t launch_adamw(float *p, const float *g, float *m, float *v, bf16 *shadow, size_t n,
                         const DevScalars *sc, cudaStream_t st);

// Sharded optimizer pieces (data parallelism): sum of squares into a device double, and
// AdamW over parameter ranges with compactly stored gradients and moments.
constexpr int ADAM_MAX_RANGES = 64;
struct AdamRanges {
  int n;
  long long offset[ADAM_MAX_RANGES];  // first parameter of range k (multiple of 4)
  long long count[ADAM_MAX_RANGES];   // elements of range k (multiple of 4)
  long long base[ADAM_MAX_RANGES];    // compact offset of range k in g, m, v
  float lr, wd, clip, beta1, beta2, eps, bias1, bias2;
};
cudaError_t launch_sumsq(const float *x, size_t n, double *partials, unsigned *counter,
                         double *out, cudaStream_t st);
cudaError_t launch_adamw_ranges(float *p, const float *g, float *m, float *v,
                                const AdamRanges &rg, const double *sumsq, cudaStream_t st);

// fp32 -> bf16 copy of the weights.
cudaError_t launch_to_bf16(const float *p, bf16 *out, size_t n, cudaStream_t st);

// Attention (head h of q/k/v at columns h*hd of each third of qkv [M, 3C]).
template <typename T>
cudaError_t launch_attention_fwd(const T *qkv, T *o, float *lse, int B, int Tlen, int C, int H,
                                 int window, cudaStream_t st);
template <typename T>
cudaError_t launch_attention_bwd(const T *qkv, const T *o, const T *dout, const float *lse,
                                 float *Dbuf, T *dqkv, int B, int Tlen, int C, int H, int window,
                                 cudaStream_t st);

// Attention on the tensor cores (head_dim 64, bf16): forward, and backward. Backward with
// dst == NULL: a dQ pass that also writes D = rowsum(dO o O), then the dK/dV pass. With dst
// (B*H*T*T bf16 scratch): D, then the dK/dV pass also writing dS^T to dst, then dQ = dS K
// from dst on the tensor cores (no second pass over the scores); d_ready: Dbuf already holds
// D (the GEMM that produced dO wrote it), only with dst. err: device error word.
bool attention_tc_supported(int C, int H);
cudaError_t launch_attention_fwd_tc(const bf16 *qkv, bf16 *o, float *lse, int B, int T, int C,
                                    int H, int window, unsigned *err, cudaStream_t st);
cudaError_t launch_attention_bwd_tc(const bf16 *qkv, const bf16 *o, const bf16 *dout,
                                    const float *lse, float *Dbuf, bf16 *dqkv, int B, int T,
                                    int C, int H, int window, unsigned *err, cudaStream_t st,
                                    bf16 *dst = nullptr, bool d_ready = false);

// The same backward with its D scratch in a file-scope device array (no allocation); rejects
// B*H*T > attention_bwd_noalloc_max_rows() with cudaErrorInvalidValue.
size_t attention_bwd_noalloc_max_rows();
cudaError_t launch_attention_bwd_tc_noalloc(const bf16 *qkv, const bf16 *o, const bf16 *dout,
                                            const float *lse, bf16 *dqkv, int B, int T, int C,
                                            int H, int window, unsigned *err, cudaStream_t st);

// GEMM on CUDA cores (fp32 validation mode and shapes the tensor-core path does not take).
template <typename T>
cudaError_t launch_gemm_simt(const GemmDesc &d, cudaStream_t st);
// Ordered reduction of split-K partials through the (elementwise) epilogue.
template <typename T>
cudaError_t launch_splitk_reduce(const GemmDesc &d, cudaStream_t st);
