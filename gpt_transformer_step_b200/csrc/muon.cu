// Hybrid Muon + AdamW optimizer update (nanochat architecture page, section
// "Optimierungsstrategien Muon und AdamW"): the 2-D matrices of the blocks are updated by
// Muon, everything else by AdamW.
//
// Muon per matrix W (rows x cols), on the clipped gradient g:
//   1. momentum, Nesterov form in lerp notation: buf = lerp(buf, g, 1-mu); u = lerp(g, buf, mu)
//   2. Polar Express ("Polar Express Details"): X = bf16(u) / (||X||_F * 1.01 + 1e-6), then per
//      coefficient triple (a, b, c): tall (rows > cols) A = X^T X, B = b A + c A^2, X = a X + X B;
//      otherwise A = X X^T, X = a X + B X  (bf16 operands, fp32 accumulation in TMEM)
//   3. factored second moment ("Zustandsverwaltung"): v = mean of X^2 per row (tall) or per
//      column (wide), s = lerp(s, v, 1-beta2), X' = X / sqrt(max(s, eps)), rescaled to ||X||_F
//   4. cautious update ("Cautious Update Mechanismus"): mask = (X' * W >= 0);
//      W -= lr * X' + lr * wd * W * mask
// All matrices of one shape (one per layer) are processed together: every kernel here runs a
// grid row per matrix, and the Polar Express GEMMs are batched tcgen05 GEMMs.
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "muon.cuh"

namespace {

constexpr int MU_THREADS = 256;

__device__ __forceinline__ float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// Last-block-done reduction helper: block partial sums (double) of matrix l in fixed order.
__device__ bool last_block(unsigned *counter, unsigned nblocks) {
  __shared__ bool last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(counter, 1u) == nblocks - 1;
  }
  __syncthreads();
  return last;
}

__device__ double block_sum(double v) {
  __shared__ double sh[MU_THREADS / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < MU_THREADS / 32; ++w) t += sh[w];
  return t;  // valid in thread 0
}

// Stage 1 + the normalisation's sum of squares: buf and X for matrix l = blockIdx.y; the last
// block of the matrix writes scale[l] = 1 / (||bf16(u)||_F * 1.01 + 1e-6).
__global__ void __launch_bounds__(MU_THREADS)
muon_momentum_kernel(const float *__restrict__ g, float *__restrict__ buf, bf16 *__restrict__ X,
                     MuonGroup grp, float mu, const DevScalars *__restrict__ sc,
                     double *__restrict__ partials, unsigned *__restrict__ counters,
                     float *__restrict__ scale) {
  const int l = blockIdx.y;
  const size_t n = (size_t)grp.rows * grp.cols, base = grp.off0 + (size_t)l * grp.stride;
  const float coef = sc->coef;
  const bool skip = sc->nonfinite || sc->err;
  const float4 *g4 = reinterpret_cast<const float4 *>(g + base);
  float4 *b4 = reinterpret_cast<float4 *>(buf + base);
  uint2 *x4 = reinterpret_cast<uint2 *>(X + (size_t)l * n);
  float ss = 0.f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 4;
       i += (size_t)gridDim.x * blockDim.x) {
    const float4 gv = g4[i];
    float4 bv = b4[i];
    const float gg[4] = {coef * gv.x, coef * gv.y, coef * gv.z, coef * gv.w};
    float bb[4] = {bv.x, bv.y, bv.z, bv.w}, u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      bb[k] = bb[k] + (1.f - mu) * (gg[k] - bb[k]);
      u[k] = bf16_round(gg[k] + mu * (bb[k] - gg[k]));
      ss += u[k] * u[k];
    }
    if (!skip) b4[i] = make_float4(bb[0], bb[1], bb[2], bb[3]);
    __nv_bfloat162 lo = __floats2bfloat162_rn(u[0], u[1]), hi = __floats2bfloat162_rn(u[2], u[3]);
    x4[i] = make_uint2(*reinterpret_cast<unsigned *>(&lo), *reinterpret_cast<unsigned *>(&hi));
  }
  const double t = block_sum((double)ss);
  if (threadIdx.x == 0) partials[(size_t)l * gridDim.x + blockIdx.x] = t;
  if (last_block(&counters[l], gridDim.x) && threadIdx.x == 0) {
    __threadfence();
    double s = 0.0;
    for (unsigned b = 0; b < gridDim.x; ++b) s += ((volatile double *)partials)[(size_t)l * gridDim.x + b];
    scale[l] = (float)(1.0 / (sqrt(s) * 1.01 + 1e-6));
    counters[l] = 0u;
  }
}

// X[l] *= scale[l] (bf16).
__global__ void __launch_bounds__(MU_THREADS)
muon_scale_kernel(bf16 *__restrict__ X, size_t n, const float *__restrict__ scale) {
  const int l = blockIdx.y;
  const float s = scale[l];
  uint2 *x4 = reinterpret_cast<uint2 *>(X + (size_t)l * n);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 4;
       i += (size_t)gridDim.x * blockDim.x) {
    uint2 w = x4[i];
    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&w.x);
    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&w.y);
    float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    lo = __floats2bfloat162_rn(a.x * s, a.y * s);
    hi = __floats2bfloat162_rn(b.x * s, b.y * s);
    x4[i] = make_uint2(*reinterpret_cast<unsigned *>(&lo), *reinterpret_cast<unsigned *>(&hi));
  }
}

// Stage 3, per line (row of a tall matrix, column of a wide one): q = sum of X^2 over the line,
// s = lerp(s, q / len, 1 - beta2) (s in adam_v at the matrix's offset), rs = 1/sqrt(max(s, eps)),
// qh = q * rs^2. Tall: a warp per row; wide: a block per 256 columns.
__global__ void __launch_bounds__(MU_THREADS)
muon_lines_kernel(const bf16 *__restrict__ X, float *__restrict__ sv, MuonGroup grp, float beta2,
                  float eps, const DevScalars *__restrict__ sc, float *__restrict__ q,
                  float *__restrict__ qh, float *__restrict__ rs) {
  const int l = blockIdx.y;
  const int r = grp.rows, c = grp.cols;
  const bool tall = r > c;
  const int nl = tall ? r : c, len = tall ? c : r;
  const bf16 *x = X + (size_t)l * r * c;
  float *s = sv + grp.off0 + (size_t)l * grp.stride;
  const bool skip = sc->nonfinite || sc->err;
  float *ql = q + (size_t)l * nl, *qhl = qh + (size_t)l * nl, *rsl = rs + (size_t)l * nl;
  auto finish = [&](int line, float sum) {
    const float sold = s[line];
    const float snew = sold + (1.f - beta2) * (sum / (float)len - sold);
    if (!skip) s[line] = snew;
    const float rr = rsqrtf(fmaxf(snew, eps));
    ql[line] = sum;
    qhl[line] = sum * rr * rr;
    rsl[line] = rr;
  };
  if (tall) {
    const int lane = threadIdx.x & 31;
    for (int row = blockIdx.x * (MU_THREADS / 32) + (threadIdx.x >> 5); row < r;
         row += gridDim.x * (MU_THREADS / 32)) {
      float sum = 0.f;
      for (int j = lane * 8; j < c; j += 256) {
        const uint4 w = *reinterpret_cast<const uint4 *>(x + (size_t)row * c + j);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(h[k]);
          sum += f.x * f.x + f.y * f.y;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) finish(row, sum);
    }
  } else {
    // a block per 256 columns: 32 column groups of 8 (16-byte loads) x 8 row groups, each
    // thread summing every 8th row of its 8 columns; the 8 row-group sums are added in order
    __shared__ float part[8][256];
    const int cg = threadIdx.x & 31, rg = threadIdx.x >> 5;
    for (int c0 = blockIdx.x * 256; c0 < c; c0 += gridDim.x * 256) {
      const int col = c0 + cg * 8;
      float acc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] = 0.f;
      if (col < c) {
        for (int i = rg; i < r; i += 8) {
          const uint4 w = *reinterpret_cast<const uint4 *>(x + (size_t)i * c + col);
          const __nv_bfloat162 *hh = reinterpret_cast<const __nv_bfloat162 *>(&w);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(hh[k]);
            acc[2 * k] += f.x * f.x;
            acc[2 * k + 1] += f.y * f.y;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) part[rg][cg * 8 + k] = acc[k];
      __syncthreads();
      const int cc = c0 + threadIdx.x;
      if (cc < c) {
        float sum = 0.f;
#pragma unroll
        for (int g = 0; g < 8; ++g) sum += part[g][threadIdx.x];
        finish(cc, sum);
      }
      __syncthreads();
    }
  }
}

// gamma[l] = sqrt(sum q / sum qh) over the lines of matrix l (one block per matrix, fixed order).
__global__ void __launch_bounds__(MU_THREADS)
muon_gamma_kernel(const float *__restrict__ q, const float *__restrict__ qh, int nl,
                  float *__restrict__ gamma) {
  const int l = blockIdx.x;
  double a = 0.0, b = 0.0;
  for (int i = threadIdx.x; i < nl; i += blockDim.x) {
    a += q[(size_t)l * nl + i];
    b += qh[(size_t)l * nl + i];
  }
  const double ta = block_sum(a);
  const double tb = block_sum(b);
  if (threadIdx.x == 0) gamma[l] = tb > 0.0 ? (float)sqrt(ta / tb) : 0.f;
}

// Stage 4: W -= lr * u + lr * wd * W * [u * W >= 0], u = gamma * X * rs(line).
__global__ void __launch_bounds__(MU_THREADS)
muon_update_kernel(float *__restrict__ p, const bf16 *__restrict__ X, MuonGroup grp,
                   const float *__restrict__ rs, const float *__restrict__ gamma, float lr,
                   float wd, const DevScalars *__restrict__ sc) {
  if (sc->nonfinite || sc->err) return;
  const int l = blockIdx.y;
  const int r = grp.rows, c = grp.cols;
  const bool tall = r > c;
  const int nl = tall ? r : c;
  const size_t n = (size_t)r * c, base = grp.off0 + (size_t)l * grp.stride;
  const bf16 *x = X + (size_t)l * n;
  const float *rsl = rs + (size_t)l * nl;
  const float gm = gamma[l];
  float4 *p4 = reinterpret_cast<float4 *>(p + base);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 4;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t e = 4 * i;
    const int row = (int)(e / c), col = (int)(e % c);  // c % 4 == 0: one row per vector
    const uint2 w = *reinterpret_cast<const uint2 *>(x + e);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w.y));
    const float xv[4] = {a.x, a.y, b.x, b.y};
    float4 pv = p4[i];
    float pp[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float u = gm * xv[k] * rsl[tall ? row : col + k];
      const float mask = (u * pp[k] >= 0.f) ? 1.f : 0.f;
      pp[k] = pp[k] - (lr * u + lr * wd * pp[k] * mask);
    }
    p4[i] = make_float4(pp[0], pp[1], pp[2], pp[3]);
  }
}

// AdamW on ranges of the flat vectors (gradients and moments in the same layout as params),
// the order of adamw_kernel; coef and the skip flags from the device scalars.
__global__ void __launch_bounds__(MU_THREADS)
muon_adamw_ranges_kernel(float *__restrict__ p, const float *__restrict__ g, float *__restrict__ m,
                         float *__restrict__ v, MuonAdamRanges rg, const DevScalars *__restrict__ sc) {
  if (sc->nonfinite || sc->err) return;
  const int k = blockIdx.y;
  const float coef = sc->coef;
  const size_t off = rg.offset[k], cnt = rg.count[k];
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < cnt;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t j = off + i;
    float pp = p[j], mm = m[j], vv = v[j];
    const float gi = coef * g[j];
    pp = pp * (1.f - rg.lr * rg.wd);
    mm = mm + (1.f - rg.beta1) * (gi - mm);
    vv = rg.beta2 * vv + (1.f - rg.beta2) * gi * gi;
    const float denom = sqrtf(vv / rg.bias2) + rg.eps;
    pp = pp - (rg.lr / rg.bias1) * mm / denom;
    p[j] = pp; m[j] = mm; v[j] = vv;
  }
}

int blocks_for(size_t n4, int cap) {
  size_t b = (n4 + MU_THREADS - 1) / MU_THREADS;
  if (b < 1) b = 1;
  if (b > (size_t)cap) b = cap;
  return (int)b;
}

GemmDesc bdesc(int M, int N, int K, const bf16 *A, long lda, int ak, long abs, const bf16 *B,
               long ldb, int bk, long bbs, int batch) {
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.M = M; d.N = N; d.K = K;
  d.A = A; d.lda = lda; d.a_kmajor = ak; d.a_bstride = abs;
  d.B = B; d.ldb = ldb; d.b_kmajor = bk; d.b_bstride = bbs;
  d.batch = batch;
  d.split_k = 1;
  return d;
}

}  // namespace

size_t muon_scratch_bytes(const MuonGroup *groups, int ngroups) {
  size_t x = 0, a = 0, lines = 0, cnt = 0;
  for (int i = 0; i < ngroups; ++i) {
    const MuonGroup &g = groups[i];
    const size_t d = g.rows < g.cols ? g.rows : g.cols, nl = g.rows > g.cols ? g.rows : g.cols;
    x = x > (size_t)g.count * g.rows * g.cols ? x : (size_t)g.count * g.rows * g.cols;
    a = a > (size_t)g.count * d * d ? a : (size_t)g.count * d * d;
    lines = lines > (size_t)g.count * nl ? lines : (size_t)g.count * nl;
    cnt = cnt > (size_t)g.count ? cnt : (size_t)g.count;
  }
  const size_t al = 256;
  auto up = [&](size_t b) { return (b + al - 1) / al * al; };
  return 2 * up(x * 2) + 2 * up(a * 2) + 3 * up(lines * 4) + up(cnt * MUON_MAX_BLOCKS * 8) +
         up(cnt * 4) + 2 * up(cnt * 4) + al;
}

MuonScratch muon_scratch_carve(void *base, const MuonGroup *groups, int ngroups) {
  size_t x = 0, a = 0, lines = 0, cnt = 0;
  for (int i = 0; i < ngroups; ++i) {
    const MuonGroup &g = groups[i];
    const size_t d = g.rows < g.cols ? g.rows : g.cols, nl = g.rows > g.cols ? g.rows : g.cols;
    x = x > (size_t)g.count * g.rows * g.cols ? x : (size_t)g.count * g.rows * g.cols;
    a = a > (size_t)g.count * d * d ? a : (size_t)g.count * d * d;
    lines = lines > (size_t)g.count * nl ? lines : (size_t)g.count * nl;
    cnt = cnt > (size_t)g.count ? cnt : (size_t)g.count;
  }
  const size_t al = 256;
  auto up = [&](size_t b) { return (b + al - 1) / al * al; };
  char *p = (char *)(((uintptr_t)base + al - 1) / al * al);
  MuonScratch s;
  s.X[0] = (bf16 *)p; p += up(x * 2);
  s.X[1] = (bf16 *)p; p += up(x * 2);
  s.A = (bf16 *)p; p += up(a * 2);
  s.Bm = (bf16 *)p; p += up(a * 2);
  s.q = (float *)p; p += up(lines * 4);
  s.qh = (float *)p; p += up(lines * 4);
  s.rs = (float *)p; p += up(lines * 4);
  s.partials = (double *)p; p += up(cnt * MUON_MAX_BLOCKS * 8);
  s.counters = (unsigned *)p; p += up(cnt * 4);
  s.scale = (float *)p; p += up(cnt * 4);
  s.gamma = (float *)p;
  return s;
}

cudaError_t muon_adamw_ranges(float *p, const float *g, float *m, float *v,
                              const MuonAdamRanges &rg, const DevScalars *sc, cudaStream_t st) {
  if (rg.n <= 0) return cudaSuccess;
  long most = 1;
  for (int k = 0; k < rg.n; ++k) most = rg.count[k] > most ? rg.count[k] : most;
  int bx = blocks_for((size_t)most, 148 * 8);
  muon_adamw_ranges_kernel<<<dim3(bx, rg.n), MU_THREADS, 0, st>>>(p, g, m, v, rg, sc);
  return cudaGetLastError();
}

cudaError_t muon_update_group(TcGemm *tc, const MuonGroup &grp, const MuonStepArgs &a,
                              const MuonScratch &s, cudaStream_t st, int *launches) {
  const int r = grp.rows, c = grp.cols, L = grp.count;
  const size_t n = (size_t)r * c;
  const bool tall = r > c;
  const int d = tall ? c : r, nl = tall ? r : c;
  const int bx = blocks_for(n / 4, MUON_MAX_BLOCKS);
  // 1. momentum, bf16 update, its norm
  muon_momentum_kernel<<<dim3(bx, L), MU_THREADS, 0, st>>>(a.grads, a.mom, s.X[0], grp, a.mu, a.sc,
                                                            s.partials, s.counters, s.scale);
  CUDA_TRY(cudaGetLastError());
  muon_scale_kernel<<<dim3(bx, L), MU_THREADS, 0, st>>>(s.X[0], n, s.scale);
  CUDA_TRY(cudaGetLastError());
  *launches += 2;
  // 2. Polar Express: batched GEMMs over the L matrices of the group
  int cur = 0;
  for (int it = 0; it < a.ns; ++it) {
    const float ca = a.coeffs[3 * it], cb = a.coeffs[3 * it + 1], cc = a.coeffs[3 * it + 2];
    const bf16 *Xc = s.X[cur];
    bf16 *Xn = s.X[cur ^ 1];
    const long xs = (long)n, as = (long)d * d;
    // A = X X^T (wide) or X^T X (tall): d x d
    GemmDesc g1 = tall ? bdesc(d, d, r, Xc, c, 0, xs, Xc, c, 0, xs, L)
                       : bdesc(d, d, c, Xc, c, 1, xs, Xc, c, 1, xs, L);
    g1.epi.kind = EPI_STORE; g1.epi.out = s.A; g1.epi.ldo = d; g1.out_bstride = as;
    g1.err = a.err;
    CUDA_TRY(tc_gemm_launch(tc, g1, st, launches));
    // B = c A A + b A  (A . A with the right operand read MN-major: exact without symmetry)
    GemmDesc g2 = bdesc(d, d, d, s.A, d, 1, as, s.A, d, 0, as, L);
    g2.epi.kind = EPI_AXPBY; g2.epi.out = s.Bm; g2.epi.ldo = d; g2.out_bstride = as;
    g2.epi.aux = s.A; g2.epi.ld_aux = d; g2.epi.aux_bstride = as;
    g2.epi.alpha = cc; g2.epi.beta = cb;
    g2.err = a.err;
    CUDA_TRY(tc_gemm_launch(tc, g2, st, launches));
    // X' = a X + X B (tall: r x c times c x c) or a X + B X (wide: r x r times r x c)
    GemmDesc g3 = tall ? bdesc(r, c, c, Xc, c, 1, xs, s.Bm, d, 0, as, L)
                       : bdesc(r, c, r, s.Bm, d, 1, as, Xc, c, 0, xs, L);
    g3.epi.kind = EPI_AXPBY; g3.epi.out = Xn; g3.epi.ldo = c; g3.out_bstride = xs;
    g3.epi.aux = Xc; g3.epi.ld_aux = c; g3.epi.aux_bstride = xs;
    g3.epi.alpha = 1.f; g3.epi.beta = ca;
    g3.err = a.err;
    CUDA_TRY(tc_gemm_launch(tc, g3, st, launches));
    *launches += 3;
    cur ^= 1;
  }
  // 3. factored second moment and the norm-preserving rescale
  const int lb = tall ? (r + (MU_THREADS / 32) - 1) / (MU_THREADS / 32) : (c + 255) / 256;
  muon_lines_kernel<<<dim3(lb < 1 ? 1 : lb, L), MU_THREADS, 0, st>>>(s.X[cur], a.sv, grp, a.beta2,
                                                                   a.eps, a.sc, s.q, s.qh, s.rs);
  CUDA_TRY(cudaGetLastError());
  muon_gamma_kernel<<<L, MU_THREADS, 0, st>>>(s.q, s.qh, nl, s.gamma);
  CUDA_TRY(cudaGetLastError());
  // 4. cautious update
  muon_update_kernel<<<dim3(bx, L), MU_THREADS, 0, st>>>(a.params, s.X[cur], grp, s.rs, s.gamma,
                                                         a.lr, a.wd, a.sc);
  *launches += 3;
  return cudaGetLastError();
}
