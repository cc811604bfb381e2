// Causal attention with an optional left window, on CUDA cores (fp32 validation mode and any
// head_dim). One warp per query (forward, dQ) or per key (dK, dV); online softmax; no atomics,
// so results are deterministic.
//
// Semantics (nanochat architecture page, "Modellarchitektur und FLOPs-Berechnung": a left
// window per layer; reading: window w >= 0 admits keys j with i - w <= j <= i):
//   s_ij = q_i . k_j / sqrt(hd) ; p = softmax over admitted j ; o_i = sum_j p_ij v_j ;
//   lse_i = log sum_j exp(s_ij) is kept for the backward pass.
#include "kernels.cuh"

namespace {

constexpr int AW = 4;  // warps per block

__device__ __forceinline__ float wsum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float wmax(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <typename T, int HD>
__global__ void __launch_bounds__(AW * 32)
attn_fwd_simt(const T *__restrict__ qkv, T *__restrict__ o, float *__restrict__ lse, int Tlen,
              int C, int H, int window, float scale) {
  constexpr int R = HD / 32;
  __shared__ float qs[AW][HD];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int i = blockIdx.x * AW + w;
  const int h = blockIdx.y, b = blockIdx.z;
  if (i >= Tlen) return;
  const long rs = 3L * C;
  const T *base = qkv + (long)b * Tlen * rs;
  for (int d = lane; d < HD; d += 32) qs[w][d] = to_f(base[(long)i * rs + h * HD + d]) * scale;
  __syncwarp();
  float mrun = -INFINITY, lrun = 0.f, acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  const int jlo = window >= 0 ? max(0, i - window) : 0;
  for (int j0 = jlo; j0 <= i; j0 += 32) {
    const int j = j0 + lane;
    float s = -INFINITY;
    if (j <= i) {
      const T *k = base + (long)j * rs + C + h * HD;
      float d = 0.f;
#pragma unroll 8
      for (int e = 0; e < HD; ++e) d += qs[w][e] * to_f(k[e]);
      s = d;
    }
    const float mnew = fmaxf(mrun, wmax(s));
    const float p = (j <= i) ? expf(s - mnew) : 0.f;
    const float corr = expf(mrun - mnew);
    lrun = lrun * corr + wsum(p);
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] *= corr;
    const int nj = min(32, i - j0 + 1);
    for (int jj = 0; jj < nj; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const T *v = base + (long)(j0 + jj) * rs + 2 * C + h * HD;
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] += pj * to_f(v[lane + 32 * r]);
    }
    mrun = mnew;
  }
  const float inv = 1.f / lrun;
#pragma unroll
  for (int r = 0; r < R; ++r)
    o[((long)b * Tlen + i) * C + h * HD + lane + 32 * r] = from_f<T>(acc[r] * inv);
  if (lane == 0) lse[((long)b * H + h) * Tlen + i] = mrun + logf(lrun);
}

// dQ pass (warp per query); also writes D_i = dO_i . O_i for the dK/dV pass.
template <typename T, int HD>
__global__ void __launch_bounds__(AW * 32)
attn_bwd_dq_simt(const T *__restrict__ qkv, const T *__restrict__ o, const T *__restrict__ dout,
                 const float *__restrict__ lse, float *__restrict__ Dbuf, T *__restrict__ dqkv,
                 int Tlen, int C, int H, int window, float scale) {
  constexpr int R = HD / 32;
  __shared__ float qs[AW][HD], dos[AW][HD];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int i = blockIdx.x * AW + w;
  const int h = blockIdx.y, b = blockIdx.z;
  if (i >= Tlen) return;
  const long rs = 3L * C;
  const T *base = qkv + (long)b * Tlen * rs;
  const long orow = ((long)b * Tlen + i) * C + h * HD;
  float dpart = 0.f;
  for (int d = lane; d < HD; d += 32) {
    qs[w][d] = to_f(base[(long)i * rs + h * HD + d]) * scale;
    float g = to_f(dout[orow + d]);
    dos[w][d] = g;
    dpart += g * to_f(o[orow + d]);
  }
  const float Di = wsum(dpart);
  __syncwarp();
  const long li = ((long)b * H + h) * Tlen + i;
  if (lane == 0) Dbuf[li] = Di;
  const float L = lse[li];
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  const int jlo = window >= 0 ? max(0, i - window) : 0;
  for (int j0 = jlo; j0 <= i; j0 += 32) {
    const int j = j0 + lane;
    float ds = 0.f;
    if (j <= i) {
      const T *k = base + (long)j * rs + C + h * HD;
      const T *v = base + (long)j * rs + 2 * C + h * HD;
      float s = 0.f, dp = 0.f;
#pragma unroll 8
      for (int e = 0; e < HD; ++e) {
        s += qs[w][e] * to_f(k[e]);
        dp += dos[w][e] * to_f(v[e]);
      }
      const float p = expf(s - L);
      ds = p * (dp - Di);
    }
    const int nj = min(32, i - j0 + 1);
    for (int jj = 0; jj < nj; ++jj) {
      const float d = __shfl_sync(0xffffffffu, ds, jj);
      const T *k = base + (long)(j0 + jj) * rs + C + h * HD;
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] += d * to_f(k[lane + 32 * r]);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
    dqkv[((long)b * Tlen + i) * rs + h * HD + lane + 32 * r] = from_f<T>(acc[r] * scale);
}

// dK / dV pass (warp per key): query i sees key j iff j <= i <= j + w.
template <typename T, int HD>
__global__ void __launch_bounds__(AW * 32)
attn_bwd_dkv_simt(const T *__restrict__ qkv, const T *__restrict__ dout,
                  const float *__restrict__ lse, const float *__restrict__ Dbuf,
                  T *__restrict__ dqkv, int Tlen, int C, int H, int window, float scale) {
  constexpr int R = HD / 32;
  __shared__ float ks[AW][HD], vs[AW][HD];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int j = blockIdx.x * AW + w;
  const int h = blockIdx.y, b = blockIdx.z;
  if (j >= Tlen) return;
  const long rs = 3L * C;
  const T *base = qkv + (long)b * Tlen * rs;
  for (int d = lane; d < HD; d += 32) {
    ks[w][d] = to_f(base[(long)j * rs + C + h * HD + d]) * scale;
    vs[w][d] = to_f(base[(long)j * rs + 2 * C + h * HD + d]);
  }
  __syncwarp();
  float dk[R], dv[R];
#pragma unroll
  for (int r = 0; r < R; ++r) dk[r] = dv[r] = 0.f;
  const int ihi = window >= 0 ? min(Tlen - 1, j + window) : Tlen - 1;
  const long lb = ((long)b * H + h) * Tlen;
  for (int i0 = j; i0 <= ihi; i0 += 32) {
    const int i = i0 + lane;
    float p = 0.f, ds = 0.f;
    if (i <= ihi) {
      const T *q = base + (long)i * rs + h * HD;
      const T *g = dout + ((long)b * Tlen + i) * C + h * HD;
      float s = 0.f, dp = 0.f;
#pragma unroll 8
      for (int e = 0; e < HD; ++e) {
        s += ks[w][e] * to_f(q[e]);
        dp += vs[w][e] * to_f(g[e]);
      }
      p = expf(s - lse[lb + i]);
      ds = p * (dp - Dbuf[lb + i]);
    }
    const int ni = min(32, ihi - i0 + 1);
    for (int ii = 0; ii < ni; ++ii) {
      const float pp = __shfl_sync(0xffffffffu, p, ii);
      const float dd = __shfl_sync(0xffffffffu, ds, ii);
      const T *q = base + (long)(i0 + ii) * rs + h * HD;
      const T *g = dout + ((long)b * Tlen + i0 + ii) * C + h * HD;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        dv[r] += pp * to_f(g[lane + 32 * r]);
        dk[r] += dd * to_f(q[lane + 32 * r]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    dqkv[((long)b * Tlen + j) * rs + C + h * HD + lane + 32 * r] = from_f<T>(dk[r] * scale);
    dqkv[((long)b * Tlen + j) * rs + 2 * C + h * HD + lane + 32 * r] = from_f<T>(dv[r]);
  }
}

}  // namespace

template <typename T>
cudaError_t launch_attention_fwd(const T *qkv, T *o, float *lse, int B, int Tlen, int C, int H,
                                 int window, cudaStream_t st) {
  const int hd = C / H;
  const float scale = 1.0f / sqrtf((float)hd);
  dim3 grid((Tlen + AW - 1) / AW, H, B);
  switch (hd) {
    case 32: attn_fwd_simt<T, 32><<<grid, AW * 32, 0, st>>>(qkv, o, lse, Tlen, C, H, window, scale); break;
    case 64: attn_fwd_simt<T, 64><<<grid, AW * 32, 0, st>>>(qkv, o, lse, Tlen, C, H, window, scale); break;
    case 128: attn_fwd_simt<T, 128><<<grid, AW * 32, 0, st>>>(qkv, o, lse, Tlen, C, H, window, scale); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_attention_bwd(const T *qkv, const T *o, const T *dout, const float *lse,
                                 float *Dbuf, T *dqkv, int B, int Tlen, int C, int H, int window,
                                 cudaStream_t st) {
  const int hd = C / H;
  const float scale = 1.0f / sqrtf((float)hd);
  dim3 grid((Tlen + AW - 1) / AW, H, B);
#define ATTN_BWD(HDV)                                                                        \
  attn_bwd_dq_simt<T, HDV><<<grid, AW * 32, 0, st>>>(qkv, o, dout, lse, Dbuf, dqkv, Tlen, C, H, \
                                                     window, scale);                           \
  CUDA_TRY(cudaGetLastError());                                                                \
  attn_bwd_dkv_simt<T, HDV><<<grid, AW * 32, 0, st>>>(qkv, dout, lse, Dbuf, dqkv, Tlen, C, H,   \
                                                      window, scale);
  switch (hd) {
    case 32: ATTN_BWD(32) break;
    case 64: ATTN_BWD(64) break;
    case 128: ATTN_BWD(128) break;
    default: return cudaErrorInvalidValue;
  }
#undef ATTN_BWD
  return cudaGetLastError();
}

template cudaError_t launch_attention_fwd<float>(const float *, float *, float *, int, int, int,
                                                 int, int, cudaStream_t);
template cudaError_t launch_attention_fwd<bf16>(const bf16 *, bf16 *, float *, int, int, int,
                                                int, int, cudaStream_t);
template cudaError_t launch_attention_bwd<float>(const float *, const float *, const float *,
                                                 const float *, float *, float *, int, int, int,
                                                 int, int, cudaStream_t);
template cudaError_t launch_attention_bwd<bf16>(const bf16 *, const bf16 *, const bf16 *,
                                                const float *, float *, bf16 *, int, int, int,
                                                int, int, cudaStream_t);
