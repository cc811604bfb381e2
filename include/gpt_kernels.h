/* gpt_kernels.h -- single-kernel entry points of the step library, for tests and per-kernel
 * measurement. They run exactly the kernels gpt_train_step uses, on caller-owned device
 * buffers, on the given cudaStream_t (NULL = legacy default stream), and do not
 * synchronise. Status codes are those of gpt_step.h.
 *
 * Operation (the dense contractions of the GPT-2 block and tied lm_head; nanoGPT README,
 * intro; llm.c summary, "Estructura del código", where these were library GEMMs):
 *   acc[m][n] = sum_k A[m][k] * B[n][k]   (bf16 operands, fp32 accumulation)
 *   A[m][k] = A[m*lda + k] if a_kmajor else A[k*lda + m]     (bf16, device)
 *   B[n][k] = B[n*ldb + k] if b_kmajor else B[k*ldb + n]     (bf16, device)
 * then epilogue `epi`:
 *   GPTK_EPI_STORE      out[m*ldo+n]  = bf16(acc)
 *   GPTK_EPI_STORE_GELU out[m*ldo+n]  = bf16(gelu_tanh'(acc)); out2[m*ldo2+n] = bf16(gelu_tanh(acc))
 *   GPTK_EPI_RESID      out[m*ldo+n]  = bf16(aux[m*ld_aux+n] + acc)
 *   GPTK_EPI_DGELU      out[m*ldo+n]  = bf16(acc * aux[m*ld_aux+n])  (aux: the derivative the
 *                       forward stored with GPTK_EPI_STORE_GELU)
 *   GPTK_EPI_F32_STORE  outf[m*ldf+n] = acc
 *   GPTK_EPI_F32_ACCUM  outf[m*ldf+n] += acc
 * K >= 1. split_k > 1 splits K into split_k ranges whose fp32 partials are summed in a fixed order
 * (only for the two F32 epilogues; needs scratch of split_k*M*N floats, caller-owned).
 * split_k = 0 on the tensor-core path lets the launcher choose the CTA group and a split of at
 * most 16 that fits in scratch_floats (no split without scratch); on the SIMT path 0 means 1.
 * path: GPTK_PATH_TCGEN05 (tensor cores; needs lda, ldb, ldo... multiples of 8 elements and
 * 16-byte aligned pointers, else GPT_ERR_ALIGN) or GPTK_PATH_SIMT (CUDA cores, any layout).
 * dev_err: device unsigned word that receives GPT_DEVERR bits (bounded-wait timeout = 2).
 */
#ifndef GPT_KERNELS_H
#define GPT_KERNELS_H
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPTK_EPI_STORE 0
#define GPTK_EPI_STORE_GELU 1
#define GPTK_EPI_RESID 2
#define GPTK_EPI_DGELU 3
#define GPTK_EPI_F32_STORE 4
#define GPTK_EPI_F32_ACCUM 5
#define GPTK_PATH_TCGEN05 0
#define GPTK_PATH_SIMT 1

int gptk_gemm_bf16(int M, int N, int K, const void *A, long lda, int a_kmajor, const void *B,
                   long ldb, int b_kmajor, int epi, void *out, long ldo, void *out2, long ldo2,
                   const void *aux, long ld_aux, float *outf, long ldf, int split_k,
                   float *scratch, size_t scratch_floats, unsigned *dev_err, int path,
                   void *stream);

/* The tensor-core launch plan gptk_gemm_bf16 (split_k = 0) and gpt_train_step use for an M x
 * N x K GEMM with epilogue `epi`, given scratch_floats of split-K scratch, on a GPU with `sms`
 * SMs: *cta_group = 1 (128-row tiles) or 2 (256-row tiles on CTA pairs), *split_k = number of
 * K ranges (1 = no split). Host-only arithmetic (an estimate of the wave-quantised main loop
 * plus the split-K reduce traffic); no GPU is touched. GPT_ERR_INVALID_ARG on bad sizes. */
int gptk_gemm_plan(int M, int N, int K, int epi, size_t scratch_floats, int sms, int *cta_group,
                   int *split_k);

/* Causal attention with an optional left window (window < 0: full causal; w >= 0: query i
 * attends keys i-w..i), per head h of qkv [B*T, 3C] (q | k | v, head h at columns h*hd of
 * each third), nanochat architecture page, "Modellarchitektur und FLOPs-Berechnung".
 * forward:  o [B*T, C] bf16, lse [B, H, T] fp32 (natural-log log-sum-exp of the scaled scores).
 * backward: dqkv [B*T, 3C] bf16 from dout [B*T, C] and the forward's o and lse; Dbuf [B, H, T]
 *           fp32 scratch (receives rowsum(dout * o)).
 * GPTK_PATH_TCGEN05 needs head_dim 64; GPTK_PATH_SIMT takes head_dim 32, 64 or 128. */
int gptk_attention_fwd_bf16(const void *qkv, void *o, float *lse, int B, int T, int C, int H,
                            int window, unsigned *dev_err, int path, void *stream);
int gptk_attention_bwd_bf16(const void *qkv, const void *o, const void *dout, const float *lse,
                            float *Dbuf, void *dqkv, int B, int T, int C, int H, int window,
                            unsigned *dev_err, int path, void *stream);

/* The tensor-core backward in the form gpt_train_step runs it: D, then the dK/dV pass, which
 * also writes dS^T (the softmax Jacobian applied to dP, bf16) to ds_scratch, then dQ = dS K
 * as tensor-core products over the stored dS^T (the scores are not recomputed for dQ).
 * ds_scratch: device bf16 [B*H][T][T] (keys x queries per head; only the tiles inside the
 * causal/window band are written and read), 16-byte aligned. T must be a multiple of 8 (the
 * row stride of ds_scratch is a whole number of 16-byte units), head_dim 64, else
 * GPT_ERR_SHAPE. Other arguments and results as gptk_attention_bwd_bf16. */
int gptk_attention_bwd_bf16_ds(const void *qkv, const void *o, const void *dout, const float *lse,
                               float *Dbuf, void *ds_scratch, void *dqkv, int B, int T, int C,
                               int H, int window, unsigned *dev_err, void *stream);

/* LayerNorm as the step runs it (bf16 activations, fp32 statistics; gain only, no bias).
 * forward: y = (x - mean) * rstd * g per row of x [M, C]; mean, rstd fp32 [M] written;
 *   rstd = 1 / sqrt(biased variance + eps). C % 8 == 0, C <= 2048; 16-byte aligned pointers.
 * backward: with xh = (x - mean) * rstd and dyh = dy * g,
 *   dres[m] (+)= rstd * (dyh - mean_c(dyh) - xh * mean_c(dyh * xh))   (+= when dres_in)
 *   dg (+)= sum_m dy * xh                                             (+= when accumulate)
 *   summed in a fixed order (per-block partials in scratch, then a column sum);
 *   scratch: gptk_layernorm_bwd_scratch_floats(M, C) floats. */
int gptk_layernorm_fwd_bf16(const void *x, const void *g, void *y, float *mean, float *rstd, int M,
                            int C, float eps, void *stream);
size_t gptk_layernorm_bwd_scratch_floats(int M, int C);
int gptk_layernorm_bwd_bf16(const void *x, const void *g, const float *mean, const float *rstd,
                            const void *dy, void *dres, int dres_in, float *dg, int accumulate,
                            float *scratch, size_t scratch_floats, int M, int C, void *stream);

/* Failure-detection self test: launches one CTA that waits on an mbarrier nothing arrives
 * on, with the bounded wait every kernel of the step uses for its barriers; after timeout_us
 * (1 .. 2,000,000) it gives up, ORs GPT_DEVERR_TIMEOUT (2) into *dev_err and returns, leaving
 * the CUDA context usable. Does not synchronise. */
int gptk_selftest_bounded_wait(unsigned timeout_us, unsigned *dev_err, void *stream);

/* Attention backward that allocates nothing (no counterpart in the pages: it exists for
 * callers that cannot call cudaMalloc, such as code running inside an allocator hook or a
 * memory pool that must not re-enter the allocator). Same arguments and results as
 * gptk_attention_bwd_bf16 on the tensor-core path, minus the Dbuf scratch: the per-row
 * scratch D = rowsum(dout * o) lives in a static device array of 2^20 floats (4 MiB) that
 * every GPU loading this library holds until the process exits.
 * Limits: head_dim 64; B * H * T <= 1048576, else GPT_ERR_SHAPE (nothing is launched).
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress);
 * make that first call before any stream capture. The address is kept for later calls; a
 * cudaDeviceReset invalidates it (do not use this entry point after one). Host threads may
 * make their first calls at the same time. All calls on one device share the array:
 * calls that overlap on the GPU (unordered streams) race on it. Nothing in it needs clearing
 * between calls: every row of D is written before it is read. Calls no allocating routine. */
int gptk_attention_bwd_bf16_noalloc(const void *qkv, const void *o, const void *dout,
                                    const float *lse, void *dqkv, int B, int T, int C, int H,
                                    int window, unsigned *dev_err, void *stream);

#ifdef __cplusplus
}
#endif
#endif
