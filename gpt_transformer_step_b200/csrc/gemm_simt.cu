// GEMM on CUDA cores: acc[m][n] = sum_k A[m][k] B[n][k] in fp32, any operand majorness, any
// shape, optional split-K with an ordered reduction. Used in fp32 validation mode.
#include "kernels.cuh"

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmDesc d) {
  __shared__ float As[BK][BM + 4], Bs[BK][BN + 4];
  __shared__ float tile[BM][BN + 1];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int S = d.split_k > 1 ? d.split_k : 1;
  const int kchunk = ((d.K + S - 1) / S + BK - 1) / BK * BK;
  const int kb = blockIdx.z * kchunk, ke = min(d.K, kb + kchunk);
  const T *A = (const T *)d.A;
  const T *Bm = (const T *)d.B;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = kb; k0 < ke; k0 += BK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int e = tid + 256 * r;
      int mm, kk;
      if (d.a_kmajor) { kk = e % BK; mm = e / BK; } else { mm = e % BM; kk = e / BM; }
      const int gm = m0 + mm, gk = k0 + kk;
      float v = 0.f;
      if (gm < d.M && gk < ke)
        v = to_f(d.a_kmajor ? A[(long)gm * d.lda + gk] : A[(long)gk * d.lda + gm]);
      As[kk][mm] = v;
      int nn;
      if (d.b_kmajor) { kk = e % BK; nn = e / BK; } else { nn = e % BN; kk = e / BN; }
      const int gn = n0 + nn, gk2 = k0 + kk;
      float u = 0.f;
      if (gn < d.N && gk2 < ke)
        u = to_f(d.b_kmajor ? Bm[(long)gn * d.ldb + gk2] : Bm[(long)gk2 * d.ldb + gn]);
      Bs[kk][nn] = u;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * b[j];
    }
    __syncthreads();
  }
  if (S > 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
        if (m < d.M && n < d.N) d.partial[((long)blockIdx.z * d.M + m) * d.N + n] = acc[i][j];
      }
    return;
  }
  if (d.epi.kind == EPI_CE_STATS) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) tile[ty + 16 * i][tx + 16 * j] = acc[i][j];
    __syncthreads();
    if (tid < BM && m0 + tid < d.M) {
      const Epi &e = d.epi;
      const int row = e.row_offset + m0 + tid;
      const int tgt = e.targets[row];
      const int nvalid = min(BN, min(e.V, d.N) - n0);
      float mx = -INFINITY;
      for (int c = 0; c < nvalid; ++c) mx = fmaxf(mx, tile[tid][c]);
      float s = 0.f;
      for (int c = 0; c < nvalid; ++c) s += expf(tile[tid][c] - mx);
      float *st = e.stats + ((long)row * e.ntiles + blockIdx.x) * 2;
      st[0] = mx;
      st[1] = s;
      if (tgt >= n0 && tgt < n0 + nvalid) e.tgt_logit[row] = tile[tid][tgt - n0];
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < d.M && n < d.N) epi_elem<T>(d.epi, m, n, acc[i][j]);
    }
}

template <typename T>
__global__ void splitk_reduce_kernel(GemmDesc d) {
  const long total = (long)d.M * d.N;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total;
       i += (long)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int z = 0; z < d.split_k; ++z) s += d.partial[(long)z * total + i];
    epi_elem<T>(d.epi, (int)(i / d.N), (int)(i % d.N), s);
  }
}

// N % 4 == 0: grid-stride over groups of four columns, 16-byte partial loads; the splits are
// added in split order, as above. vec_out: the fp32 store / accumulate and the plain
// activation store write their four values with one vector access (the host checks the
// alignment), the other epilogues go element by element.
template <typename T>
__global__ void __launch_bounds__(256) splitk_reduce4_kernel(GemmDesc d, int vec_out) {
  const int n4 = d.N >> 2;
  const long total4 = (long)d.M * n4;
  const float4 *part = reinterpret_cast<const float4 *>(d.partial);
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total4;
       i += (long)gridDim.x * blockDim.x) {
    const int m = (int)(i / n4), n = 4 * (int)(i - (long)m * n4);
    const float4 *p = part + i;
    float4 s = p[0];
#pragma unroll 4
    for (int z = 1; z < d.split_k; ++z) {
      const float4 v = p[z * total4];
      s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
    }
    const Epi &e = d.epi;
    if (vec_out && e.kind == EPI_F32_STORE) {
      *reinterpret_cast<float4 *>(e.outf + (long)m * e.ldf + n) = s;
    } else if (vec_out && e.kind == EPI_F32_ACCUM) {
      float4 *o = reinterpret_cast<float4 *>(e.outf + (long)m * e.ldf + n);
      float4 t = *o;
      t.x += s.x; t.y += s.y; t.z += s.z; t.w += s.w;
      *o = t;
    } else if (vec_out && e.kind == EPI_STORE) {
      T *o = (T *)e.out + (long)m * e.ldo + n;
      if (sizeof(T) == 2) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t *>(&lo);
        u.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(o) = u;
      } else {
        *reinterpret_cast<float4 *>(o) = s;
      }
    } else {
      epi_elem<T>(e, m, n, s.x);
      epi_elem<T>(e, m, n + 1, s.y);
      epi_elem<T>(e, m, n + 2, s.z);
      epi_elem<T>(e, m, n + 3, s.w);
    }
  }
}

}  // namespace

template <typename T>
cudaError_t launch_gemm_simt(const GemmDesc &d, cudaStream_t st) {
  if (d.M <= 0 || d.N <= 0) return cudaSuccess;
  if (d.epi.kind == EPI_STORE_DOT) return cudaErrorInvalidValue;  // tensor-core path only
  const int S = d.split_k > 1 ? d.split_k : 1;
  dim3 grid((d.N + BN - 1) / BN, (d.M + BM - 1) / BM, S);
  gemm_simt_kernel<T><<<grid, 256, 0, st>>>(d);
  CUDA_TRY(cudaGetLastError());
  if (S > 1) return launch_splitk_reduce<T>(d, st);
  return cudaSuccess;
}

template <typename T>
cudaError_t launch_splitk_reduce(const GemmDesc &d, cudaStream_t st) {
  if ((d.N & 3) == 0 && ((uintptr_t)d.partial & 15) == 0) {
    const Epi &e = d.epi;
    int vec = 0;
    if (e.kind == EPI_F32_STORE || e.kind == EPI_F32_ACCUM)
      vec = (e.ldf & 3) == 0 && ((uintptr_t)e.outf & 15) == 0;
    else if (e.kind == EPI_STORE)
      vec = (e.ldo & 3) == 0 && ((uintptr_t)e.out & (4 * sizeof(T) - 1)) == 0;
    const long total4 = (long)d.M * (d.N >> 2);
    long blocks = (total4 + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    splitk_reduce4_kernel<T><<<(int)blocks, 256, 0, st>>>(d, vec);
    return cudaGetLastError();
  }
  long total = (long)d.M * d.N;
  long blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  splitk_reduce_kernel<T><<<(int)blocks, 256, 0, st>>>(d);
  return cudaGetLastError();
}

template cudaError_t launch_gemm_simt<float>(const GemmDesc &, cudaStream_t);
template cudaError_t launch_gemm_simt<bf16>(const GemmDesc &, cudaStream_t);
template cudaError_t launch_splitk_reduce<float>(const GemmDesc &, cudaStream_t);
template cudaError_t launch_splitk_reduce<bf16>(const GemmDesc &, cudaStream_t);
