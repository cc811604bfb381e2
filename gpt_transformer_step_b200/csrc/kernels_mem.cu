// Memory-bound kernels of the step: embedding (K1, K13), LayerNorm (K2, K12),
// cross-entropy combine, global grad norm (K14), AdamW (K15). All reductions run in a fixed
// order, so results are bitwise reproducible run to run.
#include "kernels.cuh"

namespace {

// 16-byte vectors: 8 bf16 or 4 float.
template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; typedef float4 type; };
template <> struct Vec<bf16> { static constexpr int N = 8; typedef uint4 type; };

template <typename T>
__device__ __forceinline__ void load_vec(const T *p, float (&f)[Vec<T>::N]);
template <>
__device__ __forceinline__ void load_vec<float>(const float *p, float (&f)[4]) {
  float4 v = *reinterpret_cast<const float4 *>(p);
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void load_vec<bf16>(const bf16 *p, float (&f)[8]) {
  uint4 v = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x; f[2 * i + 1] = t.y;
  }
}
template <typename T>
__device__ __forceinline__ void store_vec(T *p, const float (&f)[Vec<T>::N]);
template <>
__device__ __forceinline__ void store_vec<float>(float *p, const float (&f)[4]) {
  *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
template <>
__device__ __forceinline__ void store_vec<bf16>(bf16 *p, const float (&f)[8]) {
  uint4 v;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = v;
}

template <typename T>
__device__ __forceinline__ void unpack_vec(const typename Vec<T>::type &v, float (&f)[Vec<T>::N]);
template <>
__device__ __forceinline__ void unpack_vec<float>(const float4 &v, float (&f)[4]) {
  f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
}
template <>
__device__ __forceinline__ void unpack_vec<bf16>(const uint4 &v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ------------------------------------------------------------------------------------------
// K1 embedding forward
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void embed_fwd_kernel(const int *__restrict__ tok, const int *__restrict__ tgt,
                                 const T *__restrict__ wte, const T *__restrict__ wpe,
                                 T *__restrict__ x, int M, int Tlen, int C, int V,
                                 DevScalars *sc) {
  constexpr int VN = Vec<T>::N;
  const int vpr = C / VN;  // vectors per row
  long total = (long)M * vpr;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total;
       i += (long)gridDim.x * blockDim.x) {
    int m = (int)(i / vpr), c = (int)(i % vpr) * VN;
    int id = tok[m];
    if (c == 0) {
      if (id < 0 || id >= V) atomicOr(&sc->err, GPT_DEVERR_BAD_TOKEN);
      int t = tgt[m];
      if (t < 0 || t >= V) atomicOr(&sc->err, GPT_DEVERR_BAD_TARGET);
    }
    if (id < 0 || id >= V) id = 0;
    float a[VN], b[VN];
    load_vec<T>(wte + (long)id * C + c, a);
    load_vec<T>(wpe + (long)(m % Tlen) * C + c, b);
#pragma unroll
    for (int k = 0; k < VN; ++k) a[k] += b[k];
    store_vec<T>(x + (long)m * C + c, a);
  }
}

// ------------------------------------------------------------------------------------------
// K2 LayerNorm forward: one warp per row, the row kept in registers (two-pass variance).
// ------------------------------------------------------------------------------------------
constexpr int LN_MAXV = 8;  // vectors per lane: C <= 32*8*VN

// NV = 16-byte vectors per lane (ceil(C / (32*VN))), a compile-time bound on the row slice
// each lane keeps in registers.
template <typename T, int NV>
__global__ void layernorm_fwd_kernel(const T *__restrict__ x, const T *__restrict__ g,
                                     T *__restrict__ y, float *__restrict__ mean,
                                     float *__restrict__ rstd, int M, int C, float eps) {
  constexpr int VN = Vec<T>::N;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= M) return;
  const int nv = C / VN;
  float v[NV][VN];
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    int c = (lane + 32 * j) * VN;
    if (lane + 32 * j < nv) {
      load_vec<T>(x + (long)row * C + c, v[j]);
#pragma unroll
      for (int k = 0; k < VN; ++k) s += v[j][k];
    }
  }
  const float mu = warp_sum(s) / (float)C;
  float q = 0.f;
#pragma unroll
  for (int j = 0; j < NV; ++j)
    if (lane + 32 * j < nv) {
#pragma unroll
      for (int k = 0; k < VN; ++k) {
        float d = v[j][k] - mu;
        q += d * d;
      }
    }
  const float var = warp_sum(q) / (float)C;
  const float rs = 1.0f / sqrtf(var + eps);
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    int c = (lane + 32 * j) * VN;
    if (lane + 32 * j < nv) {
      float gg[VN], o[VN];
      load_vec<T>(g + c, gg);
#pragma unroll
      for (int k = 0; k < VN; ++k) o[k] = (v[j][k] - mu) * rs * gg[k];
      store_vec<T>(y + (long)row * C + c, o);
    }
  }
  if (lane == 0) {
    mean[row] = mu;
    rstd[row] = rs;
  }
}

// ------------------------------------------------------------------------------------------
// K12 LayerNorm backward (+ residual-gradient add, + per-block dgamma partials)
// ------------------------------------------------------------------------------------------
constexpr int LNB_WARPS = 8;
constexpr int LNB_MAX_BLOCKS = 296;

// Each warp walks its rows with the next row's x, dy and residual gradient in flight while the
// current row is reduced; x-hat and g*dy are recomputed from the raw vectors in the second
// pass instead of being kept, which leaves room for two blocks of 8 warps per SM.
template <typename T, int NV>
__global__ void __launch_bounds__(LNB_WARPS * 32, 2)
layernorm_bwd_kernel(const T *__restrict__ x, const T *__restrict__ g,
                     const float *__restrict__ mean, const float *__restrict__ rstd,
                     const T *__restrict__ dy, T *__restrict__ dres,
                     float *__restrict__ dg_partial, int M, int C, int rows_per_block,
                     int res_in) {
  using VT = typename Vec<T>::type;
  constexpr int VN = Vec<T>::N;
  extern __shared__ float sm_dg[];  // [LNB_WARPS][C]
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nv = C / VN;
  float dgacc[NV][VN];
#pragma unroll
  for (int j = 0; j < NV; ++j)
#pragma unroll
    for (int k = 0; k < VN; ++k) dgacc[j][k] = 0.f;
  const int r0 = blockIdx.x * rows_per_block;
  const int r1 = min(M, r0 + rows_per_block);
  VT xr[NV], dr[NV], rr[NV];
  float mu = 0.f, rs = 0.f;
  auto load_row = [&](int row, VT (&xa)[NV], VT (&da)[NV], VT (&ra)[NV], float &m, float &s) {
    m = mean[row];
    s = rstd[row];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      if (lane + 32 * j < nv) {
        const long off = (long)row * C + (lane + 32 * j) * VN;
        xa[j] = *reinterpret_cast<const VT *>(x + off);
        da[j] = *reinterpret_cast<const VT *>(dy + off);
        if (res_in) ra[j] = *reinterpret_cast<const VT *>(dres + off);
        else ra[j] = VT{};  // dres starts at zero: written, not accumulated
      }
    }
  };
  int row = r0 + w;
  if (row < r1) load_row(row, xr, dr, rr, mu, rs);
  for (; row < r1; row += LNB_WARPS) {
    VT xn[NV], dn[NV], rn[NV];
    float mun = 0.f, rsn = 0.f;
    if (row + LNB_WARPS < r1) load_row(row + LNB_WARPS, xn, dn, rn, mun, rsn);
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      if (lane + 32 * j < nv) {
        float xv[VN], dv[VN], gv[VN];
        unpack_vec<T>(xr[j], xv);
        unpack_vec<T>(dr[j], dv);
        unpack_vec<T>(__ldg(reinterpret_cast<const VT *>(g + (lane + 32 * j) * VN)), gv);
#pragma unroll
        for (int k = 0; k < VN; ++k) {
          const float xh = (xv[k] - mu) * rs;
          const float dxh = dv[k] * gv[k];
          a += dxh;
          b += dxh * xh;
          dgacc[j][k] += dv[k] * xh;
        }
      }
    }
    a = warp_sum(a) / (float)C;
    b = warp_sum(b) / (float)C;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      if (lane + 32 * j < nv) {
        float xv[VN], dv[VN], gv[VN], rv[VN], o[VN];
        unpack_vec<T>(xr[j], xv);
        unpack_vec<T>(dr[j], dv);
        unpack_vec<T>(__ldg(reinterpret_cast<const VT *>(g + (lane + 32 * j) * VN)), gv);
        unpack_vec<T>(rr[j], rv);
#pragma unroll
        for (int k = 0; k < VN; ++k) {
          const float xh = (xv[k] - mu) * rs;
          const float dxh = dv[k] * gv[k];
          o[k] = rv[k] + rs * (dxh - a - xh * b);
        }
        store_vec<T>(dres + (long)row * C + (lane + 32 * j) * VN, o);
      }
    }
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      xr[j] = xn[j];
      dr[j] = dn[j];
      rr[j] = rn[j];
    }
    mu = mun;
    rs = rsn;
  }
#pragma unroll
  for (int j = 0; j < NV; ++j) {
    int c = (lane + 32 * j) * VN;
    if (lane + 32 * j < nv)
#pragma unroll
      for (int k = 0; k < VN; ++k) sm_dg[w * C + c + k] = dgacc[j][k];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float s = 0.f;
    for (int ww = 0; ww < LNB_WARPS; ++ww) s += sm_dg[ww * C + c];
    dg_partial[(long)blockIdx.x * C + c] = s;
  }
}

// out[c] = sum_r partial[r][c]: block = 32 columns x 32 row groups; each thread sums rows
// g, g+32, ... in order (four loads in flight), then the 32 group sums are added in group
// order (deterministic).
__global__ void __launch_bounds__(1024) colsum_kernel(const float *__restrict__ partial, int nrows,
                                                      int C, float *__restrict__ out,
                                                      int accumulate) {
  __shared__ float sh[32][33];
  const int cx = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + cx;
  float s = 0.f;
  if (c < C) {
#pragma unroll 4
    for (int r = g; r < nrows; r += 32) s += partial[(long)r * C + c];
  }
  sh[g][cx] = s;
  __syncthreads();
  if (g == 0 && c < C) {
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) t += sh[i][cx];
    out[c] = accumulate ? out[c] + t : t;
  }
}

// ------------------------------------------------------------------------------------------
// K13 embedding backward
//   dwpe[t] = sum_b dx[b, t]                      (b in order)
//   dwte[v] += sum_{m : tok[m] = v} dx[m]          (m in increasing order)
// The token ids are sorted stably (LSD radix sort, 9-bit digits, several CTAs per pass), so
// the positions of one id end up in increasing order; windows of EW sorted entries then sum
// their runs, and runs that cross a window boundary are finished by a merge in window order.
// Every sum has a fixed order: the result is bitwise reproducible.
// ------------------------------------------------------------------------------------------
template <typename T>
__global__ void dwpe_kernel(const T *__restrict__ dx, float *__restrict__ dwpe, int Bn,
                            int Tlen, int maxT, int C, int accumulate) {
  constexpr int VN = Vec<T>::N;
  const int nvec = C / VN;
  const long total = (long)maxT * nvec;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total;
       i += (long)gridDim.x * blockDim.x) {
    const int t = (int)(i / nvec), c = (int)(i % nvec) * VN;
    float s[VN];
#pragma unroll
    for (int k = 0; k < VN; ++k) s[k] = 0.f;
    if (t < Tlen)
      for (int b = 0; b < Bn; ++b) {
        float v[VN];
        load_vec<T>(dx + ((long)b * Tlen + t) * C + c, v);
#pragma unroll
        for (int k = 0; k < VN; ++k) s[k] += v[k];
      }
    float *o = dwpe + (long)t * C + c;
#pragma unroll
    for (int k = 0; k < VN; k += 4) {
      float4 r = make_float4(s[k], s[k + 1], s[k + 2], s[k + 3]);
      if (accumulate) {
        const float4 a = *reinterpret_cast<const float4 *>(o + k);
        r.x += a.x; r.y += a.y; r.z += a.z; r.w += a.w;
      }
      *reinterpret_cast<float4 *>(o + k) = r;
    }
  }
}

constexpr int RS_BITS = 9;
constexpr int RS_BUCKETS = 1 << RS_BITS;
constexpr int RS_TILE = 2048;   // entries per CTA and pass
constexpr int RS_WARPS = 8;     // each warp ranks RS_TILE / RS_WARPS consecutive entries

// Digit histogram of one tile: hist[digit * ntiles + tile] (digit-major, so an exclusive scan
// gives every (digit, tile) its first output slot in stable order).
__global__ void __launch_bounds__(256) rs_hist_kernel(const int *__restrict__ ids, int M, int shift,
                                                      unsigned *__restrict__ hist, int ntiles) {
  __shared__ unsigned cnt[RS_BUCKETS];
  for (int i = threadIdx.x; i < RS_BUCKETS; i += blockDim.x) cnt[i] = 0u;
  __syncthreads();
  const int e0 = blockIdx.x * RS_TILE, e1 = min(M, e0 + RS_TILE);
  for (int i = e0 + threadIdx.x; i < e1; i += blockDim.x)
    atomicAdd(&cnt[((unsigned)ids[i] >> shift) & (RS_BUCKETS - 1)], 1u);
  __syncthreads();
  for (int d = threadIdx.x; d < RS_BUCKETS; d += blockDim.x) hist[(long)d * ntiles + blockIdx.x] = cnt[d];
}

// Exclusive prefix sum of n counts in place (one CTA of 1024 threads, contiguous chunks).
__global__ void __launch_bounds__(1024) rs_scan_kernel(unsigned *__restrict__ a, int n) {
  __shared__ unsigned part[1024];
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int b0 = threadIdx.x * per, b1 = min(n, b0 + per);
  unsigned s = 0;
  for (int i = b0; i < b1; ++i) s += a[i];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {  // Hillis-Steele inclusive scan
    const unsigned v = threadIdx.x >= (unsigned)off ? part[threadIdx.x - off] : 0u;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  unsigned run = part[threadIdx.x] - s;  // exclusive base of this chunk
  for (int i = b0; i < b1; ++i) {
    const unsigned c = a[i];
    a[i] = run;
    run += c;
  }
}

// Stable scatter of one tile by digit: an entry's slot is its (digit, tile) base plus the
// number of earlier entries of the tile with the same digit. pos_in == NULL: positions are
// the entry indices (first pass).
__global__ void __launch_bounds__(RS_WARPS * 32)
rs_scatter_kernel(const int *__restrict__ ids_in, const int *__restrict__ pos_in,
                  int *__restrict__ ids_out, int *__restrict__ pos_out, int M, int shift,
                  const unsigned *__restrict__ offs, int ntiles) {
  __shared__ unsigned wbase[RS_WARPS][RS_BUCKETS];  // per-warp counts, then per-warp bases
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int PER_WARP = RS_TILE / RS_WARPS;
  for (int i = threadIdx.x; i < RS_WARPS * RS_BUCKETS; i += blockDim.x) (&wbase[0][0])[i] = 0u;
  __syncthreads();
  const int t0 = blockIdx.x * RS_TILE;
  const int w0 = t0 + warp * PER_WARP, w1 = min(M, w0 + PER_WARP);
  for (int i = w0 + lane; i < w1; i += 32)
    atomicAdd(&wbase[warp][((unsigned)ids_in[i] >> shift) & (RS_BUCKETS - 1)], 1u);
  __syncthreads();
  for (int d = threadIdx.x; d < RS_BUCKETS; d += blockDim.x) {
    unsigned run = offs[(long)d * ntiles + blockIdx.x];
    for (int w = 0; w < RS_WARPS; ++w) {
      const unsigned c = wbase[w][d];
      wbase[w][d] = run;
      run += c;
    }
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int c0 = w0; c0 < w1; c0 += 32) {  // chunks of 32 in entry order
    const int i = c0 + lane;
    const bool valid = i < w1;
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    if (valid) {
      const int id = ids_in[i];
      const int pos = pos_in ? pos_in[i] : i;
      const unsigned d = ((unsigned)id >> shift) & (RS_BUCKETS - 1);
      const unsigned peers = __match_any_sync(vmask, d);
      const unsigned dst = wbase[warp][d] + __popc(peers & lt);
      ids_out[dst] = id;
      pos_out[dst] = pos;
      __syncwarp(vmask);
      if ((peers & lt) == 0u) wbase[warp][d] += __popc(peers);  // the run's first lane
    }
    __syncwarp();
  }
}

constexpr int EW = 64;  // sorted entries per window

// Window w covers sorted entries [w*EW, (w+1)*EW). Runs of one id that lie wholly inside the
// window are added to dwte here; a run that starts before the window goes to slot 0, a run
// that continues past it (and did not start before) to slot 1, for the merge kernel. The
// block's warps take the window's runs in turn (run r to warp r mod 4), so short runs do not
// wait on one another; a lane owns 16-byte column vectors, and the entries of a run are summed
// in sorted (position) order.
template <typename T>
__global__ void __launch_bounds__(128) embed_seg_kernel(const int *__restrict__ sid,
                                                        const int *__restrict__ spos,
                                                        const T *__restrict__ dx,
                                                        float *__restrict__ dwte,
                                                        float *__restrict__ partial, int M, int C) {
  static_assert(EW == 64, "a window is two 32-entry ballots");
  constexpr int VN = Vec<T>::N;
  const int w = blockIdx.x;
  const int e0 = w * EW, e1 = min(M, e0 + EW);
  const int n = e1 - e0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int s_id[EW], s_pos[EW];
  __shared__ unsigned s_start[2];  // bit t: entry t starts a run
  if (threadIdx.x < EW && (int)threadIdx.x < n) {
    s_id[threadIdx.x] = sid[e0 + threadIdx.x];
    s_pos[threadIdx.x] = spos[e0 + threadIdx.x];
  }
  __syncthreads();
  if (warp < 2) {
    const int t = warp * 32 + lane;
    const bool st = t < n && (t == 0 || s_id[t] != s_id[t - 1]);
    const unsigned b = __ballot_sync(0xffffffffu, st);
    if (lane == 0) s_start[warp] = b;
  }
  __syncthreads();
  const unsigned long long starts =
      (unsigned long long)s_start[0] | ((unsigned long long)s_start[1] << 32);
  const int id_before = e0 > 0 ? sid[e0 - 1] : -1;
  const int id_after = e1 < M ? sid[e1] : -1;
  const int nvec = C / VN;
  unsigned long long rest = starts;
  for (int r = 0; rest != 0ull; ++r) {
    const int s = __ffsll((long long)rest) - 1;  // this run: entries [s, e)
    rest &= rest - 1ull;
    const int e = rest ? __ffsll((long long)rest) - 1 : n;
    if ((r & 3) != warp) continue;
    const int id = s_id[s];
    const bool before = (s == 0) && (id == id_before);
    const bool after = (e == n) && (id == id_after);
    for (int v = lane; v < nvec; v += 32) {
      const int c = v * VN;
      float acc[VN];
#pragma unroll
      for (int k = 0; k < VN; ++k) acc[k] = 0.f;
      int k0 = s;
      for (; k0 + 4 <= e; k0 += 4) {  // four rows in flight, added in order
        float a[4][VN];
#pragma unroll
        for (int u = 0; u < 4; ++u) load_vec<T>(dx + (long)s_pos[k0 + u] * C + c, a[u]);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int k = 0; k < VN; ++k) acc[k] += a[u][k];
      }
      for (; k0 < e; ++k0) {
        float a[VN];
        load_vec<T>(dx + (long)s_pos[k0] * C + c, a);
#pragma unroll
        for (int k = 0; k < VN; ++k) acc[k] += a[k];
      }
      float *dst = (!before && !after) ? dwte + (long)id * C + c
                                       : partial + ((long)w * 2 + (before ? 0 : 1)) * C + c;
#pragma unroll
      for (int k = 0; k < VN; k += 4) {
        float4 q = make_float4(acc[k], acc[k + 1], acc[k + 2], acc[k + 3]);
        if (!before && !after) {
          const float4 o = *reinterpret_cast<const float4 *>(dst + k);
          q.x += o.x; q.y += o.y; q.z += o.z; q.w += o.w;
        }
        *reinterpret_cast<float4 *>(dst + k) = q;
      }
    }
  }
}

// For each run that continues past window w (and started inside it): sum slot 1 of w and
// slot 0 of the following windows while the run goes on, in window order; add to dwte.
__global__ void __launch_bounds__(128) embed_merge_kernel(const int *__restrict__ sid,
                                                          const float *__restrict__ partial,
                                                          float *__restrict__ dwte, int M, int C,
                                                          int nwin) {
  const int w = blockIdx.x;
  const int e0 = w * EW, e1 = min(M, e0 + EW);
  if (e1 >= M) return;
  const int id = sid[e1 - 1];
  if (sid[e1] != id) return;  // does not continue
  // the run must not have started before the window
  int s = e1 - 1;
  while (s > e0 && sid[s - 1] == id) --s;
  if (s == e0 && e0 > 0 && sid[e0 - 1] == id) return;
  // windows the run covers after w: up to the one where it ends
  int wl = w + 1;
  while (wl + 1 < nwin && sid[min(M, (wl + 1) * EW) - 1] == id && sid[(wl + 1) * EW] == id) ++wl;
  for (int c = threadIdx.x * 4; c < C; c += blockDim.x * 4) {
    float4 acc = *reinterpret_cast<const float4 *>(partial + ((long)w * 2 + 1) * C + c);
    for (int ww = w + 1; ww <= wl; ++ww) {
      const float4 p = *reinterpret_cast<const float4 *>(partial + ((long)ww * 2 + 0) * C + c);
      acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
    }
    float4 *o = reinterpret_cast<float4 *>(dwte + (long)id * C + c);
    float4 r = *o;
    r.x += acc.x; r.y += acc.y; r.z += acc.z; r.w += acc.w;
    *o = r;
  }
}

// ------------------------------------------------------------------------------------------
// Cross-entropy combine and mean loss
// ------------------------------------------------------------------------------------------
__global__ void ce_combine_kernel(const float *__restrict__ stats,
                                  const float *__restrict__ tgt_logit, float *__restrict__ lse,
                                  float *__restrict__ per_token, int M, int ntiles) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= M) return;
  const float *s = stats + (long)row * ntiles * 2;
  float mx = -INFINITY;
  for (int t = lane; t < ntiles; t += 32) mx = fmaxf(mx, s[2 * t]);
  mx = warp_max(mx);
  float sum = 0.f;
  for (int t = lane; t < ntiles; t += 32) {
    float m = s[2 * t];
    if (m > -INFINITY) sum += s[2 * t + 1] * expf(m - mx);
  }
  sum = warp_sum(sum);
  if (lane == 0) {
    float l = mx + logf(sum);
    lse[row] = l;
    per_token[row] = l - tgt_logit[row];
  }
}

__global__ void mean_loss_kernel(const float *__restrict__ per_token, int M, DevScalars *sc) {
  __shared__ double sh[32];
  double s = 0.0;
  for (int i = threadIdx.x; i < M; i += blockDim.x) s += (double)per_token[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += sh[w];
    float loss = (float)(t / (double)M);
    sc->loss = loss;
    sc->loss_sum += loss;  // cleared with the other device results at the first micro-batch
    if (!isfinite(loss)) sc->nonfinite = 1;
  }
}

// ------------------------------------------------------------------------------------------
// K14 global grad norm: fixed partition into GN_BLOCKS contiguous ranges, last-arriving
// block sums the partials in index order.
// ------------------------------------------------------------------------------------------
constexpr int GN_BLOCKS = 592;
constexpr int GN_THREADS = 512;

__global__ void __launch_bounds__(GN_THREADS)
grad_norm_kernel(const float *__restrict__ g, size_t n, double *__restrict__ partials,
                 DevScalars *sc) {
  __shared__ double sh[GN_THREADS / 32];
  __shared__ bool last;
  const size_t n4 = n / 4;
  const size_t per = (n4 + gridDim.x - 1) / gridDim.x;
  const size_t b0 = blockIdx.x * per, b1 = min(n4, b0 + per);
  float s = 0.f;
  const float4 *g4 = reinterpret_cast<const float4 *>(g);
  for (size_t i = b0 + threadIdx.x; i < b1; i += blockDim.x) {
    float4 v = g4[i];
    s += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  if (blockIdx.x == gridDim.x - 1)  // tail elements
    for (size_t i = n4 * 4 + threadIdx.x; i < n; i += blockDim.x) s += g[i] * g[i];
  double d = (double)s;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = d;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < GN_THREADS / 32; ++w) t += sh[w];
    partials[blockIdx.x] = t;
    __threadfence();
    unsigned prev = atomicAdd(&sc->counter, 1u);
    last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    double t = 0.0;
    for (int b = 0; b < (int)gridDim.x; ++b) t += ((volatile double *)partials)[b];
    sc->sumsq = t;
    float nrm = (float)sqrt(t);
    sc->norm = nrm;
    float coef = (float)((double)sc->clip / (sqrt(t) + 1e-6));
    sc->coef = coef > 1.f ? 1.f : coef;
    if (!isfinite(nrm)) sc->nonfinite = 1;
    sc->counter = 0u;
  }
}

// ------------------------------------------------------------------------------------------
// K15 AdamW (order of the nanochat fused step: decay, first moment, bias correction, update)
// ------------------------------------------------------------------------------------------
// Every operation rounds on its own (no contraction into fused multiply-adds), so the result
// does not depend on the kernel this is inlined into: the whole-step update and the ranged
// update of the data-parallel step give the same bits.
__device__ __forceinline__ void adamw_one(float &p, float g, float &m, float &v, float lr,
                                          float wd, float b1, float b2, float eps, float bias1,
                                          float bias2, float coef) {
  g = __fmul_rn(g, coef);
  p = __fmul_rn(p, __fsub_rn(1.f, __fmul_rn(lr, wd)));
  m = __fadd_rn(m, __fmul_rn(__fsub_rn(1.f, b1), __fsub_rn(g, m)));
  v = __fadd_rn(__fmul_rn(b2, v), __fmul_rn(__fmul_rn(__fsub_rn(1.f, b2), g), g));
  const float denom = __fadd_rn(__fsqrt_rn(__fdiv_rn(v, bias2)), eps);
  p = __fsub_rn(p, __fdiv_rn(__fmul_rn(__fdiv_rn(lr, bias1), m), denom));
}

__global__ void adamw_kernel(float *__restrict__ p, const float *__restrict__ g,
                             float *__restrict__ m, float *__restrict__ v,
                             bf16 *__restrict__ shadow, size_t n, const DevScalars *sc) {
  // a failed step leaves the caller's state untouched: a non-finite loss or norm, an id out
  // of range or a device wait that gave up (partial gradients) all skip the update
  if (sc->nonfinite || sc->err) return;
  const float lr = sc->lr, wd = sc->wd, b1 = sc->beta1, b2 = sc->beta2, eps = sc->eps;
  const float bias1 = sc->bias1, bias2 = sc->bias2, coef = sc->coef;
  const size_t n4 = n / 4;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 P = reinterpret_cast<float4 *>(p)[i];
    float4 G = reinterpret_cast<const float4 *>(g)[i];
    float4 Mm = reinterpret_cast<float4 *>(m)[i];
    float4 Vv = reinterpret_cast<float4 *>(v)[i];
    adamw_one(P.x, G.x, Mm.x, Vv.x, lr, wd, b1, b2, eps, bias1, bias2, coef);
    adamw_one(P.y, G.y, Mm.y, Vv.y, lr, wd, b1, b2, eps, bias1, bias2, coef);
    adamw_one(P.z, G.z, Mm.z, Vv.z, lr, wd, b1, b2, eps, bias1, bias2, coef);
    adamw_one(P.w, G.w, Mm.w, Vv.w, lr, wd, b1, b2, eps, bias1, bias2, coef);
    reinterpret_cast<float4 *>(p)[i] = P;
    reinterpret_cast<float4 *>(m)[i] = Mm;
    reinterpret_cast<float4 *>(v)[i] = Vv;
    if (shadow) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(P.x, P.y), hi = __floats2bfloat162_rn(P.z, P.w);
      uint2 u;
      u.x = *reinterpret_cast<unsigned *>(&lo);
      u.y = *reinterpret_cast<unsigned *>(&hi);
      reinterpret_cast<uint2 *>(shadow)[i] = u;
    }
  }
  if (blockIdx.x == 0)
    for (size_t i = n4 * 4 + threadIdx.x; i < n; i += blockDim.x) {
      float pp = p[i], mm = m[i], vv = v[i];
      adamw_one(pp, g[i], mm, vv, lr, wd, b1, b2, eps, bias1, bias2, coef);
      p[i] = pp; m[i] = mm; v[i] = vv;
      if (shadow) shadow[i] = __float2bfloat16_rn(pp);
    }
}

// ------------------------------------------------------------------------------------------
// Sharded optimizer pieces (data parallelism with the optimizer state split across ranks)
// ------------------------------------------------------------------------------------------
// out = sum of x[i]^2 over [0, n): the same fixed partition and in-order combine of the
// partials as grad_norm_kernel, into a caller-owned device double.
__global__ void __launch_bounds__(GN_THREADS)
sumsq_kernel(const float *__restrict__ x, size_t n, double *__restrict__ partials,
             unsigned *__restrict__ counter, double *__restrict__ out) {
  __shared__ double sh[GN_THREADS / 32];
  __shared__ bool last;
  const size_t n4 = n / 4;
  const size_t per = (n4 + gridDim.x - 1) / gridDim.x;
  const size_t b0 = blockIdx.x * per, b1 = min(n4, b0 + per);
  float s = 0.f;
  const float4 *x4 = reinterpret_cast<const float4 *>(x);
  for (size_t i = b0 + threadIdx.x; i < b1; i += blockDim.x) {
    float4 v = x4[i];
    s += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
  }
  if (blockIdx.x == gridDim.x - 1)
    for (size_t i = n4 * 4 + threadIdx.x; i < n; i += blockDim.x) s += x[i] * x[i];
  double d = (double)s;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
  if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = d;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < GN_THREADS / 32; ++w) t += sh[w];
    partials[blockIdx.x] = t;
    __threadfence();
    last = atomicAdd(counter, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (last && threadIdx.x == 0) {
    __threadfence();
    double t = 0.0;
    for (int b = 0; b < (int)gridDim.x; ++b) t += ((volatile double *)partials)[b];
    *out = t;
    *counter = 0u;
  }
}

// AdamW over a list of parameter ranges whose gradients and moments are stored compactly
// (range k at compact offset base[k]); the clip coefficient comes from the global sum of
// squares in device memory. Same arithmetic as adamw_kernel.
__global__ void adamw_ranges_kernel(float *__restrict__ p, const float *__restrict__ g,
                                    float *__restrict__ m, float *__restrict__ v,
                                    AdamRanges rg, const double *__restrict__ sumsq) {
  const int k = blockIdx.y;
  const double t = *sumsq;
  float coef = (float)((double)rg.clip / (sqrt(t) + 1e-6));
  coef = coef > 1.f ? 1.f : coef;
  if (!isfinite(t)) return;
  const size_t n4 = (size_t)rg.count[k] / 4;
  float4 *p4 = reinterpret_cast<float4 *>(p + rg.offset[k]);
  const float4 *g4 = reinterpret_cast<const float4 *>(g + rg.base[k]);
  float4 *m4 = reinterpret_cast<float4 *>(m + rg.base[k]);
  float4 *v4 = reinterpret_cast<float4 *>(v + rg.base[k]);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    float4 P = p4[i], G = g4[i], Mm = m4[i], Vv = v4[i];
    adamw_one(P.x, G.x, Mm.x, Vv.x, rg.lr, rg.wd, rg.beta1, rg.beta2, rg.eps, rg.bias1, rg.bias2, coef);
    adamw_one(P.y, G.y, Mm.y, Vv.y, rg.lr, rg.wd, rg.beta1, rg.beta2, rg.eps, rg.bias1, rg.bias2, coef);
    adamw_one(P.z, G.z, Mm.z, Vv.z, rg.lr, rg.wd, rg.beta1, rg.beta2, rg.eps, rg.bias1, rg.bias2, coef);
    adamw_one(P.w, G.w, Mm.w, Vv.w, rg.lr, rg.wd, rg.beta1, rg.beta2, rg.eps, rg.bias1, rg.bias2, coef);
    p4[i] = P;
    m4[i] = Mm;
    v4[i] = Vv;
  }
}

__global__ void to_bf16_kernel(const float *__restrict__ p, bf16 *__restrict__ out, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(p[i]);
}

int grid_for(long work, int threads, int cap = 148 * 16) {
  long b = (work + threads - 1) / threads;
  if (b < 1) b = 1;
  if (b > cap) b = cap;
  return (int)b;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// launchers
// ------------------------------------------------------------------------------------------
template <typename T>
cudaError_t launch_embed_fwd(const int *tok, const int *tgt, const T *wte, const T *wpe, T *x,
                             int M, int Tlen, int C, int V, DevScalars *sc, cudaStream_t st) {
  long work = (long)M * (C / Vec<T>::N);
  embed_fwd_kernel<T><<<grid_for(work, 256), 256, 0, st>>>(tok, tgt, wte, wpe, x, M, Tlen, C, V, sc);
  return cudaGetLastError();
}

size_t embed_bwd_ws_bytes(int maxM, int C) {
  const size_t ntiles = (maxM + RS_TILE - 1) / RS_TILE;
  const size_t nwin = (maxM + EW - 1) / EW;
  return 4 * (size_t)maxM * sizeof(int) + (size_t)RS_BUCKETS * ntiles * sizeof(unsigned) + 256 +
         nwin * 2 * (size_t)C * sizeof(float) + 256;
}

template <typename T>
cudaError_t launch_embed_bwd(const int *tok, const T *dx, float *dwte, float *dwpe, int M,
                             int Tlen, int maxT, int C, int Vp, EmbedBwdWs ws, cudaStream_t st,
                             bool accumulate) {
  const int Bn = M / Tlen;
  dwpe_kernel<T><<<grid_for((long)maxT * (C / Vec<T>::N), 256), 256, 0, st>>>(
      dx, dwpe, Bn, Tlen, maxT, C, accumulate ? 1 : 0);
  CUDA_TRY(cudaGetLastError());
  // carve the workspace: ids and positions (two buffers each), digit histogram, partials
  const int ntiles = (M + RS_TILE - 1) / RS_TILE;
  char *w = (char *)ws.base;
  int *ids[2] = {(int *)w, (int *)w + M};
  int *pos[2] = {(int *)w + 2 * (size_t)M, (int *)w + 3 * (size_t)M};
  unsigned *hist = (unsigned *)((int *)w + 4 * (size_t)M);
  float *partial = (float *)(((uintptr_t)(hist + (size_t)RS_BUCKETS * ntiles) + 255) & ~(uintptr_t)255);
  // LSD radix passes over the id bits (a pass per 9 bits of Vp - 1)
  int bits = 1;
  while ((1 << bits) < Vp) ++bits;
  const int passes = (bits + RS_BITS - 1) / RS_BITS;
  const int *cur_id = tok;
  const int *cur_pos = nullptr;
  for (int p = 0; p < passes; ++p) {
    const int shift = p * RS_BITS;
    rs_hist_kernel<<<ntiles, 256, 0, st>>>(cur_id, M, shift, hist, ntiles);
    CUDA_TRY(cudaGetLastError());
    rs_scan_kernel<<<1, 1024, 0, st>>>(hist, RS_BUCKETS * ntiles);
    CUDA_TRY(cudaGetLastError());
    rs_scatter_kernel<<<ntiles, RS_WARPS * 32, 0, st>>>(cur_id, cur_pos, ids[p & 1], pos[p & 1], M,
                                                        shift, hist, ntiles);
    CUDA_TRY(cudaGetLastError());
    cur_id = ids[p & 1];
    cur_pos = pos[p & 1];
  }
  const int nwin = (M + EW - 1) / EW;
  embed_seg_kernel<T><<<nwin, 128, 0, st>>>(cur_id, cur_pos, dx, dwte, partial, M, C);
  CUDA_TRY(cudaGetLastError());
  embed_merge_kernel<<<nwin, 128, 0, st>>>(cur_id, partial, dwte, M, C, nwin);
  return cudaGetLastError();
}

int embed_bwd_launches(int Vp) {
  int bits = 1;
  while ((1 << bits) < Vp) ++bits;
  return 3 + 3 * ((bits + RS_BITS - 1) / RS_BITS);
}

#define LN_DISPATCH(NVV, CALL)                    \
  switch (NVV) {                                  \
    case 1: CALL(1); break;                       \
    case 2: CALL(2); break;                       \
    case 3: CALL(3); break;                       \
    case 4: CALL(4); break;                       \
    case 5: case 6: CALL(6); break;               \
    default: CALL(8); break;                      \
  }

template <typename T>
int ln_nv(int C) {
  const int per = 32 * Vec<T>::N;
  return (C + per - 1) / per;
}

template <typename T>
cudaError_t launch_layernorm_fwd(const T *x, const T *g, T *y, float *mean, float *rstd, int M,
                                 int C, float eps, cudaStream_t st) {
  const int warps = 8;
  const int grid = (M + warps - 1) / warps;
#define LNF(NVC) layernorm_fwd_kernel<T, NVC><<<grid, warps * 32, 0, st>>>(x, g, y, mean, rstd, M, C, eps)
  LN_DISPATCH(ln_nv<T>(C), LNF)
#undef LNF
  return cudaGetLastError();
}

int layernorm_bwd_blocks(int M) {
  int b = (M + LNB_WARPS - 1) / LNB_WARPS;
  return b < LNB_MAX_BLOCKS ? b : LNB_MAX_BLOCKS;
}

template <typename T>
cudaError_t launch_layernorm_bwd(const T *x, const T *g, const float *mean, const float *rstd,
                                 const T *dy, T *dres, float *dg_partial, float *dg, int M,
                                 int C, cudaStream_t st, bool accumulate, bool dres_in,
                                 bool colsum) {
  const int nb = layernorm_bwd_blocks(M);
  const int rpb = (M + nb - 1) / nb;
  const size_t smem = (size_t)LNB_WARPS * C * sizeof(float);
#define LNB(NVC)                                                                              \
  layernorm_bwd_kernel<T, NVC><<<nb, LNB_WARPS * 32, smem, st>>>(x, g, mean, rstd, dy, dres, \
                                                                 dg_partial, M, C, rpb,     \
                                                                 dres_in ? 1 : 0)
  LN_DISPATCH(ln_nv<T>(C), LNB)
#undef LNB
  CUDA_TRY(cudaGetLastError());
  if (!colsum) return cudaSuccess;
  colsum_kernel<<<(C + 31) / 32, 1024, 0, st>>>(dg_partial, nb, C, dg, accumulate ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_ln_colsum(const float *dg_partial, int M, int C, float *dg, bool accumulate,
                             cudaStream_t st) {
  colsum_kernel<<<(C + 31) / 32, 1024, 0, st>>>(dg_partial, layernorm_bwd_blocks(M), C, dg,
                                                accumulate ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_ce_combine(const float *stats, const float *tgt_logit, float *lse,
                              float *per_token, int M, int ntiles, DevScalars *sc,
                              cudaStream_t st) {
  ce_combine_kernel<<<(M + 7) / 8, 256, 0, st>>>(stats, tgt_logit, lse, per_token, M, ntiles);
  CUDA_TRY(cudaGetLastError());
  mean_loss_kernel<<<1, 1024, 0, st>>>(per_token, M, sc);
  return cudaGetLastError();
}

int grad_norm_blocks() { return GN_BLOCKS; }

cudaError_t launch_grad_norm(const float *g, size_t n, double *partials, DevScalars *sc,
                             cudaStream_t st) {
  grad_norm_kernel<<<GN_BLOCKS, GN_THREADS, 0, st>>>(g, n, partials, sc);
  return cudaGetLastError();
}

cudaError_t launch_adamw(float *p, const float *g, float *m, float *v, bf16 *shadow, size_t n,
                         const DevScalars *sc, cudaStream_t st) {
  adamw_kernel<<<grid_for((long)(n / 4), 256, 148 * 8), 256, 0, st>>>(p, g, m, v, shadow, n, sc);
  return cudaGetLastError();
}

cudaError_t launch_sumsq(const float *x, size_t n, double *partials, unsigned *counter,
                         double *out, cudaStream_t st) {
  sumsq_kernel<<<GN_BLOCKS, GN_THREADS, 0, st>>>(x, n, partials, counter, out);
  return cudaGetLastError();
}

cudaError_t launch_adamw_ranges(float *p, const float *g, float *m, float *v,
                                const AdamRanges &rg, const double *sumsq, cudaStream_t st) {
  long most = 1;
  for (int k = 0; k < rg.n; ++k) most = rg.count[k] > most ? rg.count[k] : most;
  int bx = grid_for(most / 4, 256, 148 * 8);
  const int per_range = (148 * 8 + rg.n - 1) / rg.n;
  if (bx > per_range) bx = per_range < 1 ? 1 : per_range;
  adamw_ranges_kernel<<<dim3(bx, rg.n), 256, 0, st>>>(p, g, m, v, rg, sumsq);
  return cudaGetLastError();
}

cudaError_t launch_to_bf16(const float *p, bf16 *out, size_t n, cudaStream_t st) {
  to_bf16_kernel<<<grid_for((long)n, 256, 148 * 8), 256, 0, st>>>(p, out, n);
  return cudaGetLastError();
}

#define INST(T)                                                                              \
  template cudaError_t launch_embed_fwd<T>(const int *, const int *, const T *, const T *, T *, \
                                           int, int, int, int, DevScalars *, cudaStream_t);    \
  template cudaError_t launch_embed_bwd<T>(const int *, const T *, float *, float *, int, int,  \
                                           int, int, int, EmbedBwdWs, cudaStream_t, bool);     \
  template cudaError_t launch_layernorm_fwd<T>(const T *, const T *, T *, float *, float *, int, \
                                               int, float, cudaStream_t);                      \
  template cudaError_t launch_layernorm_bwd<T>(const T *, const T *, const float *,             \
                                               const float *, const T *, T *, float *, float *, \
                                               int, int, cudaStream_t, bool, bool, bool);
INST(float)
INST(bf16)
