// Single-kernel entry points (include/gpt_kernels.h): the step's own kernels on caller
// buffers, for tests and per-kernel timing.
#include "../../include/gpt_kernels.h"
#include "../../include/gpt_step.h"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace {
TcGemm *tc_instance() {
  static TcGemm *t = nullptr;
  if (!t) tc_gemm_create(&t);
  return t;
}
}  // namespace

extern "C" int gptk_gemm_bf16(int M, int N, int K, const void *A, long lda, int a_kmajor,
                              const void *B, long ldb, int b_kmajor, int epi, void *out, long ldo,
                              void *out2, long ldo2, const void *aux, long ld_aux, float *outf,
                              long ldf, int split_k, float *scratch, size_t scratch_floats,
                              unsigned *dev_err, int path, void *stream) {
  if (M < 0 || N < 0 || K < 1 || !A || !B || !dev_err) return GPT_ERR_INVALID_ARG;
  if (epi < GPTK_EPI_STORE || epi > GPTK_EPI_F32_ACCUM) return GPT_ERR_INVALID_ARG;
  const bool f32 = epi == GPTK_EPI_F32_STORE || epi == GPTK_EPI_F32_ACCUM;
  if (f32 ? !outf : !out) return GPT_ERR_INVALID_ARG;
  if ((epi == GPTK_EPI_STORE_GELU && !out2) ||
      ((epi == GPTK_EPI_RESID || epi == GPTK_EPI_DGELU) && !aux))
    return GPT_ERR_INVALID_ARG;
  if (split_k < 0 || (split_k == 0 && path != GPTK_PATH_TCGEN05)) split_k = 1;
  if (split_k > 1 && (!f32 || !scratch || scratch_floats < (size_t)split_k * M * N))
    return GPT_ERR_INVALID_ARG;
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.M = M; d.N = N; d.K = K;
  d.A = A; d.lda = lda; d.a_kmajor = a_kmajor ? 1 : 0;
  d.B = B; d.ldb = ldb; d.b_kmajor = b_kmajor ? 1 : 0;
  d.epi.kind = epi;  // GPTK_EPI_* equal EPI_* for these six kinds
  d.epi.out = out; d.epi.ldo = ldo; d.epi.out2 = out2; d.epi.ldo2 = ldo2;
  d.epi.aux = aux; d.epi.ld_aux = ld_aux; d.epi.outf = outf; d.epi.ldf = ldf;
  d.split_k = split_k;
  d.partial = scratch;
  d.err = dev_err;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (M == 0 || N == 0) return GPT_OK;
  if (path == GPTK_PATH_TCGEN05) {
    if (!tc_gemm_supported(d)) return GPT_ERR_ALIGN;
    int n = 0;
    tc_gemm_set_splitk_capacity(tc_instance(), scratch ? scratch_floats : 0);
    e = tc_gemm_launch(tc_instance(), d, st, &n);
  } else if (path == GPTK_PATH_SIMT) {
    e = launch_gemm_simt<bf16>(d, st);
  } else {
    return GPT_ERR_INVALID_ARG;
  }
  return e == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

extern "C" int gptk_gemm_plan(int M, int N, int K, int epi, size_t scratch_floats, int sms,
                              int *cta_group, int *split_k) {
  if (M < 1 || N < 1 || K < 1 || sms < 2 || !cta_group || !split_k) return GPT_ERR_INVALID_ARG;
  if (epi < GPTK_EPI_STORE || epi > GPTK_EPI_F32_ACCUM) return GPT_ERR_INVALID_ARG;
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.M = M; d.N = N; d.K = K;
  d.epi.kind = epi;
  d.split_k = 0;
  tc_gemm_plan(d, scratch_floats, sms, cta_group, split_k);
  return GPT_OK;
}

extern "C" int gptk_attention_fwd_bf16(const void *qkv, void *o, float *lse, int B, int T, int C,
                                       int H, int window, unsigned *dev_err, int path,
                                       void *stream) {
  if (!qkv || !o || !lse || !dev_err || B <= 0 || T <= 0 || H <= 0 || C % H) return GPT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (path == GPTK_PATH_TCGEN05) {
    if (!attention_tc_supported(C, H)) return GPT_ERR_SHAPE;
    e = launch_attention_fwd_tc((const bf16 *)qkv, (bf16 *)o, lse, B, T, C, H, window, dev_err, st);
  } else if (path == GPTK_PATH_SIMT) {
    e = launch_attention_fwd<bf16>((const bf16 *)qkv, (bf16 *)o, lse, B, T, C, H, window, st);
  } else {
    return GPT_ERR_INVALID_ARG;
  }
  return e == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

extern "C" int gptk_attention_bwd_bf16(const void *qkv, const void *o, const void *dout,
                                       const float *lse, float *Dbuf, void *dqkv, int B, int T,
                                       int C, int H, int window, unsigned *dev_err, int path,
                                       void *stream) {
  if (!qkv || !o || !dout || !lse || !Dbuf || !dqkv || !dev_err || B <= 0 || T <= 0 || H <= 0 ||
      C % H)
    return GPT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (path == GPTK_PATH_TCGEN05) {
    if (!attention_tc_supported(C, H)) return GPT_ERR_SHAPE;
    e = launch_attention_bwd_tc((const bf16 *)qkv, (const bf16 *)o, (const bf16 *)dout, lse, Dbuf,
                                (bf16 *)dqkv, B, T, C, H, window, dev_err, st);
  } else if (path == GPTK_PATH_SIMT) {
    e = launch_attention_bwd<bf16>((const bf16 *)qkv, (const bf16 *)o, (const bf16 *)dout, lse,
                                   Dbuf, (bf16 *)dqkv, B, T, C, H, window, st);
  } else {
    return GPT_ERR_INVALID_ARG;
  }
  return e == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

extern "C" int gptk_attention_bwd_bf16_ds(const void *qkv, const void *o, const void *dout,
                                          const float *lse, float *Dbuf, void *ds_scratch,
                                          void *dqkv, int B, int T, int C, int H, int window,
                                          unsigned *dev_err, void *stream) {
  if (!qkv || !o || !dout || !lse || !Dbuf || !ds_scratch || !dqkv || !dev_err || B <= 0 ||
      T <= 0 || H <= 0 || C % H)
    return GPT_ERR_INVALID_ARG;
  if (!attention_tc_supported(C, H) || (T & 7)) return GPT_ERR_SHAPE;
  if (((uintptr_t)ds_scratch & 15u) != 0) return GPT_ERR_ALIGN;
  cudaError_t e = launch_attention_bwd_tc((const bf16 *)qkv, (const bf16 *)o, (const bf16 *)dout,
                                          lse, Dbuf, (bf16 *)dqkv, B, T, C, H, window, dev_err,
                                          (cudaStream_t)stream, (bf16 *)ds_scratch);
  return e == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

extern "C" int gptk_layernorm_fwd_bf16(const void *x, const void *g, void *y, float *mean,
                                       float *rstd, int M, int C, float eps, void *stream) {
  if (!x || !g || !y || !mean || !rstd || M < 0 || C <= 0 || !(eps > 0.f)) return GPT_ERR_INVALID_ARG;
  if ((C % 8) || C > 2048) return GPT_ERR_SHAPE;
  if ((((uintptr_t)x | (uintptr_t)g | (uintptr_t)y) & 15u) != 0) return GPT_ERR_ALIGN;
  if (M == 0) return GPT_OK;
  const cudaError_t e = launch_layernorm_fwd<bf16>((const bf16 *)x, (const bf16 *)g, (bf16 *)y,
                                                   mean, rstd, M, C, eps, (cudaStream_t)stream);
  return e == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

extern "C" size_t gptk_layernorm_bwd_scratch_floats(int M, int C) {
  return M <= 0 || C <= 0 ? 0 : (size_t)layernorm_bwd_blocks(M) * C;
}

extern "C" int gptk_layernorm_bwd_bf16(const void *x, const void *g, const float *mean,
                                       const float *rstd, const void *dy, void *dres, int dres_in,
                                       float *dg, int accumulate, float *scratch,
                                       size_t scratch_floats, int M, int C, void *stream) {
  if (!x || !g || !mean || !rstd || !dy || !dres || !dg || !scratch || M <= 0 || C <= 0)
    return GPT_ERR_INVALID_ARG;
  if ((C % 8) || C > 2048) return GPT_ERR_SHAPE;
  if (scratch_floats < gptk_layernorm_bwd_scratch_floats(M, C)) return GPT_ERR_INVALID_ARG;
  if ((((uintptr_t)x | (uintptr_t)g | (uintptr_t)dy | (uintptr_t)dres) & 15u) != 0)
    return GPT_ERR_ALIGN;
  const cudaError_t e = launch_layernorm_bwd<bf16>(
      (const bf16 *)x, (const bf16 *)g, mean, rstd, (const bf16 *)dy, (bf16 *)dres, scratch, dg, M,
      C, (cudaStream_t)stream, accumulate != 0, dres_in != 0);
  return e == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

// Attention backward without any allocation: see include/gpt_kernels.h.
extern "C" int gptk_attention_bwd_bf16_noalloc(const void *qkv, const void *o, const void *dout,
                                               const float *lse, void *dqkv, int B, int T, int C,
                                               int H, int window, unsigned *dev_err,
                                               void *stream) {
  if (!qkv || !o || !dout || !lse || !dqkv || !dev_err || B <= 0 || T <= 0 || H <= 0 || C % H)
    return GPT_ERR_INVALID_ARG;
  if (!attention_tc_supported(C, H)) return GPT_ERR_SHAPE;
  if ((size_t)B * H * T > attention_bwd_noalloc_max_rows()) return GPT_ERR_SHAPE;
  cudaError_t e = launch_attention_bwd_tc_noalloc((const bf16 *)qkv, (const bf16 *)o,
                                                  (const bf16 *)dout, lse, (bf16 *)dqkv, B, T, C,
                                                  H, window, dev_err, (cudaStream_t)stream);
  return e == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

namespace {
// Waits, with the library's bounded wait, on an mbarrier that nothing ever arrives on. The
// wait gives up after timeout_ns, sets the timeout bit in the device error word and the
// kernel returns: the context stays usable.
__global__ void wait_selftest_kernel(unsigned long long timeout_ns, unsigned *err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    tc::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  const uint64_t t0 = tc::globaltimer();
  while (!tc::mbar_try_wait(&bar, 0)) {
    if (tc::globaltimer() - t0 > timeout_ns) {
      atomicOr(err, GPT_DEVERR_TIMEOUT);
      return;
    }
  }
}
}  // namespace

extern "C" int gptk_selftest_bounded_wait(unsigned timeout_us, unsigned *dev_err, void *stream) {
  if (!dev_err || timeout_us == 0 || timeout_us > 2000000u) return GPT_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(1000ull * timeout_us, dev_err);
  return cudaGetLastError() == cudaSuccess ? GPT_OK : GPT_ERR_CUDA;
}

