// Shared device-side definitions of the step library (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

typedef __nv_bfloat16 bf16;

// ---- device error word bits -------------------------------------------------------------
#define GPT_DEVERR_BAD_TOKEN 1u
#define GPT_DEVERR_TIMEOUT 2u
#define GPT_DEVERR_BAD_TARGET 4u

// Hyper-parameters and results that live in device memory. The host writes the first part
// before each step (one small copy), so a captured CUDA graph replays with a new lr.
struct DevScalars {
  // written by the host before each step
  float lr, wd, clip, beta1, beta2, eps;
  float bias1, bias2;  // 1 - beta^t, computed on the host in double
  float inv_M;         // 1 / (positions in the optimizer step: n_micro * B * T)
  int step;
  int pad0[6];
  // written by the device
  double sumsq;        // sum of squared raw grads
  float norm, coef;    // global grad norm, clip coefficient
  float loss;          // mean loss of the last micro-batch
  float loss_sum;      // sum of the micro-batch mean losses of this optimizer step
  int nonfinite;       // a loss or the norm not finite: the update is skipped
  unsigned err;        // GPT_DEVERR_* bits
  unsigned counter;    // arrival counter of the grad-norm last-block reduction
  unsigned counter2;   // arrival counter of gpt_sumsq's last-block reduction
  int pad1[6];
};

// ---- type helpers -----------------------------------------------------------------------
__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float x) { return __float2bfloat16_rn(x); }

// GELU, tanh form (Hendrycks & Gimpel). tanhf from the CUDA math library.
__device__ __forceinline__ float gelu_f(float x) {
  const float k = 0.7978845608028654f;
  float u = k * (x + 0.044715f * x * x * x);
  return 0.5f * x * (1.f + tanhf(u));
}
__device__ __forceinline__ float gelu_grad_f(float x) {
  const float k = 0.7978845608028654f;
  float x2 = x * x;
  float u = k * (x + 0.044715f * x2 * x);
  float t = tanhf(u);
  return 0.5f * (1.f + t) + 0.5f * x * (1.f - t * t) * k * (1.f + 3.f * 0.044715f * x2);
}

// GELU for bf16 mode: the same tanh form with the PTX tanh.approx.f32 instruction (max
// relative error about 2^-11, below bf16 resolution).
__device__ __forceinline__ float tanh_fast(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// With u = k (x + c x^3), t = tanh(u) and h = (1 + t) / 2:  gelu(x) = x h  and, since
// 1 - t^2 = 4 h (1 - h),  gelu'(x) = h + 2 x u' h (1 - h) = h (1 + w (1 - h)), w = 2 x u',
// u' = k (1 + 3 c x^2): the same functions in fewer operations.
__device__ __forceinline__ float gelu_fast(float x) {
  const float k = 0.7978845608028654f, kc = 0.7978845608028654f * 0.044715f;
  const float x2 = x * x;
  const float h = fmaf(0.5f, tanh_fast(fmaf(kc, x2, k) * x), 0.5f);
  return x * h;
}
__device__ __forceinline__ float gelu_grad_fast(float x) {
  const float k = 0.7978845608028654f, kc = 0.7978845608028654f * 0.044715f;
  const float x2 = x * x;
  const float h = fmaf(0.5f, tanh_fast(fmaf(kc, x2, k) * x), 0.5f);
  const float w = fmaf(6.f * kc, x2, 2.f * k) * x;
  return fmaf(h, fmaf(-w, h, w), h);
}
// gelu(x) and gelu'(x) together (one tanh): the forward stores gelu'(pre) for the backward.
__device__ __forceinline__ float gelu_and_grad_fast(float x, float &g) {
  const float k = 0.7978845608028654f, kc = 0.7978845608028654f * 0.044715f;
  const float x2 = x * x;
  const float h = fmaf(0.5f, tanh_fast(fmaf(kc, x2, k) * x), 0.5f);
  const float w = fmaf(6.f * kc, x2, 2.f * k) * x;
  g = fmaf(h, fmaf(-w, h, w), h);
  return x * h;
}
template <typename T> __device__ __forceinline__ float gelu_t(float x) { return gelu_fast(x); }
template <> __device__ __forceinline__ float gelu_t<float>(float x) { return gelu_f(x); }
template <typename T> __device__ __forceinline__ float gelu_grad_t(float x) { return gelu_grad_fast(x); }
template <> __device__ __forceinline__ float gelu_grad_t<float>(float x) { return gelu_grad_f(x); }

// exp: exact-rounding library expf in fp32 validation mode, the fast intrinsic in bf16 mode.
template <typename T> __device__ __forceinline__ float exp_t(float x) { return __expf(x); }
template <> __device__ __forceinline__ float exp_t<float>(float x) { return expf(x); }

// ---- GEMM epilogues ---------------------------------------------------------------------
// Every GEMM computes acc[m][n] = sum_k A[m][k] * B[n][k] in fp32 and hands each
// accumulator to one of these epilogues.
enum EpiKind {
  EPI_STORE = 0,      // out[m][n] = acc                                  (activation type)
  EPI_STORE_GELU,     // out[m][n] = gelu'(acc) ; out2[m][n] = gelu(acc)  (activation type)
  EPI_RESID,          // out[m][n] = aux[m][n] + acc  (aux may equal out)  (activation type)
  EPI_DGELU,          // out[m][n] = acc * aux[m][n], aux = gelu'(pre)    (activation type)
  EPI_F32_STORE,      // outf[m][n] = acc                                  (fp32)
  EPI_F32_ACCUM,      // outf[m][n] += acc                                 (fp32)
  EPI_CE_STATS,       // per (row, column tile): max and sum(exp(acc - max)) over cols < V;
                      // the target's logit to tgt_logit[row]
  EPI_CE_DS,          // out[m][n] = (exp(acc - lse[row]) - [n == target]) * inv_M, 0 for n >= V
  // GELU recompute (the backward recomputes the activation instead of the forward keeping it)
  EPI_STORE_PRE_GELU, // out[m][n] = acc (pre-activation) ; out2[m][n] = gelu(acc)
  EPI_DGELU_RECOMP,   // out[m][n] = acc * gelu'(aux[m][n]) ; out2[m][n] = gelu(aux[m][n]),
                      // aux = the pre-activation the forward kept
  EPI_AXPBY,          // out[m][n] = alpha * acc + beta * aux[m][n]        (activation type)
  // attention backward: dO and, per row and 64-column head, D = rowsum(dO * O)
  EPI_STORE_DOT,      // out[m][n] = acc ; outf[(b * N/64 + n/64) * dot_T + t] = sum over the
                      // head's 64 columns of bf16(acc) * aux[m][n], for row m = b * dot_T + t
};

struct Epi {
  int kind;
  void *out; long ldo;
  void *out2; long ldo2;
  const void *aux; long ld_aux;
  float *outf; long ldf;
  // cross-entropy epilogues (row index = row_offset + local row)
  const int *targets;
  const float *lse;
  float *stats;       // [rows][ntiles][2] (max, sumexp)
  float *tgt_logit;   // [rows]
  int ntiles, tile_n; // column tiles of width tile_n
  int V;
  int row_offset;
  const DevScalars *sc;  // inv_M
  float alpha, beta;     // EPI_AXPBY
  long aux_bstride;      // batched GEMMs: elements between the aux matrices of two batches
  int dot_T;             // EPI_STORE_DOT: rows per sequence
};

struct GemmDesc {
  int M, N, K;
  const void *A; long lda; int a_kmajor;  // A[m][k] = A[m*lda+k] (K-major) or A[k*lda+m]
  const void *B; long ldb; int b_kmajor;  // B[n][k] = B[n*ldb+k] (K-major) or B[k*ldb+n]
  Epi epi;
  int split_k;       // > 1: fp32 partials [split][M][N] then an ordered reduction
  float *partial;
  unsigned *err;     // device error word (bounded-wait timeouts); NULL = &epi.sc->err
  // batched GEMM (tensor-core path; no K split): `batch` independent products, operand and
  // output matrices `*_bstride` elements apart (0 or 1: one product)
  int batch;
  long a_bstride, b_bstride, out_bstride;
};

template <typename T>
__device__ __forceinline__ void epi_elem(const Epi &e, int m, int n, float acc) {
  switch (e.kind) {
    case EPI_STORE:
      ((T *)e.out)[(long)m * e.ldo + n] = from_f<T>(acc);
      break;
    case EPI_STORE_GELU:
      ((T *)e.out)[(long)m * e.ldo + n] = from_f<T>(gelu_grad_t<T>(acc));
      ((T *)e.out2)[(long)m * e.ldo2 + n] = from_f<T>(gelu_t<T>(acc));
      break;
    case EPI_RESID: {
      float r = to_f(((const T *)e.aux)[(long)m * e.ld_aux + n]);
      ((T *)e.out)[(long)m * e.ldo + n] = from_f<T>(r + acc);
      break;
    }
    case EPI_DGELU: {
      float gd = to_f(((const T *)e.aux)[(long)m * e.ld_aux + n]);
      ((T *)e.out)[(long)m * e.ldo + n] = from_f<T>(acc * gd);
      break;
    }
    case EPI_STORE_PRE_GELU: {  // gelu of the stored (rounded) value: recompute is exact
      const T pre = from_f<T>(acc);
      ((T *)e.out)[(long)m * e.ldo + n] = pre;
      ((T *)e.out2)[(long)m * e.ldo2 + n] = from_f<T>(gelu_t<T>(to_f(pre)));
      break;
    }
    case EPI_DGELU_RECOMP: {
      const float pre = to_f(((const T *)e.aux)[(long)m * e.ld_aux + n]);
      ((T *)e.out)[(long)m * e.ldo + n] = from_f<T>(acc * gelu_grad_t<T>(pre));
      ((T *)e.out2)[(long)m * e.ldo2 + n] = from_f<T>(gelu_t<T>(pre));
      break;
    }
    case EPI_AXPBY: {
      const float a = to_f(((const T *)e.aux)[(long)m * e.ld_aux + n]);
      ((T *)e.out)[(long)m * e.ldo + n] = from_f<T>(e.alpha * acc + e.beta * a);
      break;
    }
    case EPI_F32_STORE:
      e.outf[(long)m * e.ldf + n] = acc;
      break;
    case EPI_F32_ACCUM:
      e.outf[(long)m * e.ldf + n] += acc;
      break;
    case EPI_CE_DS: {
      int row = e.row_offset + m;
      float v = 0.f;
      if (n < e.V) {
        v = exp_t<T>(acc - e.lse[row]);
        if (n == e.targets[row]) v -= 1.f;
        v *= e.sc->inv_M;
      }
      ((T *)e.out)[(long)m * e.ldo + n] = from_f<T>(v);
      break;
    }
    default:
      break;
  }
}

#define CUDA_TRY(x)                                   \
  do {                                                \
    cudaError_t err__ = (x);                          \
    if (err__ != cudaSuccess) return err__;           \
  } while (0)
