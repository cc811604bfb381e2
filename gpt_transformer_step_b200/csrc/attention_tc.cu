// Causal (optionally left-windowed) attention, head_dim 64, on the sm_100a tensor cores.
//
// Semantics (nanochat architecture page, "Modellarchitektur und FLOPs-Berechnung": causal
// attention with a per-layer left window; reading: window w >= 0 admits keys i-w <= j <= i):
//   s_ij = q_i . k_j / sqrt(64);  P = softmax_j(s) over admitted j;  o_i = sum_j P_ij v_j;
//   lse_i = log sum_j exp(s_ij) (natural log) is kept for the backward pass.
//
// All three kernels use 128x128 tiles, TMA loads of 128x64 bf16 tiles (128-byte swizzle) from
// the fused qkv buffer [B*T, 3C], tcgen05.mma with fp32 accumulators in TMEM, and "row" warps
// in which each thread owns one row (or half a row) of the 128x128 score tile:
//   forward  (CTA = b, h, 128 queries; two CTAs per SM): S = Q K^T -> TMEM; online softmax in
//            the log2 domain with a conditional rescale of O (only when the running max grows
//            by > 8); P (bf16) -> TMEM; O += P V with P read from TMEM.
//   dQ       (persistent; item = b, h, 128 queries): D_i = dO_i . O_i (also written out),
//            S = Q K^T, dP = dO V^T, dS = P o (dP - D) -> TMEM, dQ += dS K.
//   dK / dV  (persistent; item = b, h, 128 keys): S^T = K Q^T, dP^T = V dO^T, P^T and dS^T ->
//            TMEM, dV += P^T dO, dK += dS^T Q.
// No atomics: every output element is written by exactly one work item, so results are bitwise
// reproducible. Tiles entirely outside the causal/window band are skipped; edge tiles are
// masked element by element. Every wait is bounded (device error word on timeout).
#include <atomic>
#include <type_traits>

#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace {
using namespace tc;

constexpr int HD = 64;
constexpr int TILE = 128;
constexpr int TILE_BYTES = TILE * HD * 2;  // 16 KB: 128 rows x 64 bf16, K-major SW128
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct AttnParams {
  int B, T, C, H, window;
  float scale_log2;  // log2(e) / sqrt(64)
  float scale;       // 1 / sqrt(64)
  bf16 *o;           // forward output [B*T, C]
  float *lse;        // forward output [B, H, T]
  const bf16 *O;     // backward inputs
  const bf16 *dO;    // [B*T, C]
  const float *lse_in;
  float *Dbuf;       // [B, H, T]
  bf16 *dqkv;        // [B*T, 3C]
  unsigned *err;
};

__host__ __device__ constexpr uint32_t idesc_bf16(int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TILE >> 4) << 24);
}

// A global load issued where it stands: the compiler may not sink it towards its first use
// (the value is wanted a whole tile later, and its latency must pass in the meantime).
__device__ __forceinline__ float ldg_early(const float *p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// Packed two-lane fp32 arithmetic (sm_100): one instruction for two independent elements.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// One warp-collective bounded wait: lane 0 polls, the result is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned *err) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag, err) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  return (uint8_t *)(((uintptr_t)p + 1023) & ~(uintptr_t)1023);
}

// A = 128 x K (K-major, SW128, K-blocks of 64 at stride 16 KB); B K-major N x 64 tile.
// S[128 x N] (+)= A[:, 0:64] * B^T  with 4 MMAs of K = 16.
__device__ __forceinline__ void mma_qk(uint32_t d, uint32_t sA, uint32_t sB, int n) {
  const uint32_t id = idesc_bf16(n, 0, 0);
  const uint64_t a0 = sdesc(sA, 16, 1024), b0 = sdesc(sB, 16, 1024);
#pragma unroll
  for (int k = 0; k < HD / 16; ++k)
    umma_bf16(d, a0 + (uint64_t)(2 * k), b0 + (uint64_t)(2 * k), id, k > 0 ? 1u : 0u);  // +32 B
}
// O[128 x 64] (+)= A[128 x 128] * V with A in TMEM (64 columns of packed bf16 pairs, the
// tcgen05 "A from tensor memory" form) and V the 128(k) x 64(n) MN-major smem tile.
__device__ __forceinline__ void mma_pv_ts(uint32_t d, uint32_t a_tmem, uint32_t sV, bool accumulate) {
  const uint32_t id = idesc_bf16(HD, 0, 1);
  const uint64_t b0 = sdesc(sV, 8192, 1024);
#pragma unroll
  for (int k = 0; k < TILE / 16; ++k)  // K = 16 per MMA: 8 TMEM columns of A, 16 rows of V
    umma_bf16_ts(d, a_tmem + 8 * k, b0 + (uint64_t)((k * 2048) >> 4), id,
                 (accumulate || k > 0) ? 1u : 0u);
}

// The same product over keys [64 half, 64 half + 64) only: P's TMEM columns and V's rows of
// that half.
__device__ __forceinline__ void mma_pv_ts_half(uint32_t d, uint32_t a_tmem, uint32_t sV, int half,
                                               bool accumulate) {
  const uint32_t id = idesc_bf16(HD, 0, 1);
  const uint64_t b0 = sdesc(sV, 8192, 1024);
#pragma unroll
  for (int kk = 0; kk < TILE / 32; ++kk) {
    const int k = half * (TILE / 32) + kk;
    umma_bf16_ts(d, a_tmem + 8 * k, b0 + (uint64_t)((k * 2048) >> 4), id,
                 (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Packs 32 fp32 values into 16 bf16 pairs and stores them to 16 TMEM columns.
__device__ __forceinline__ void st_tmem_bf16x32(uint32_t taddr, const uint32_t (&pk)[16]) {
  tmem_st16_nw(taddr, pk);
}

// ------------------------------------------------------------------------------------------
// persistent schedule
// ------------------------------------------------------------------------------------------
// The two backward kernels are persistent: a CTA loops over work items (one 128-row tile of one
// (batch, head)) numbered heavy-first, taking item r*G + c in even rounds r and
// r*G + G-1-c in odd rounds (G CTAs, this is CTA c), so heavy and light items pair up. Every
// warp role walks the same sequence, and the loads of the next item overlap the last tiles of
// the current one. Each output element is still written by exactly one item.
__device__ __forceinline__ int item_index(int r) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  return r * G + ((r & 1) ? G - 1 - c : c);
}

// A query tile of one (batch, head) and the key tiles it sees.
struct QTile { int q0, b, h, kt0, n; };
__device__ __forceinline__ bool query_item(const AttnParams &P, int r, QTile &it) {
  const int BH = P.B * P.H, nqt = (P.T + TILE - 1) / TILE;
  const int u = item_index(r);
  if (u >= nqt * BH) return false;
  const int bh = u % BH;
  it.q0 = (nqt - 1 - u / BH) * TILE;  // the last query tiles see the most keys: first
  it.b = bh / P.H;
  it.h = bh % P.H;
  const int w = P.window;
  it.kt0 = (w >= 0 ? max(0, it.q0 - w) : 0) / TILE;
  it.n = (min(P.T, it.q0 + TILE) + TILE - 1) / TILE - it.kt0;
  return true;
}
struct QCursor {  // (item, key tile) walk of this CTA
  QTile it;
  int i, j;
  bool valid;
  __device__ __forceinline__ void start(const AttnParams &P) { i = 0; j = 0; valid = query_item(P, 0, it); }
  __device__ __forceinline__ void next(const AttnParams &P) {
    if (++j == it.n) { j = 0; ++i; valid = query_item(P, i, it); }
  }
};

// A key tile of one (batch, head) and the query tiles that see it.
struct KTile { int k0, b, h, qt0, n; };
__device__ __forceinline__ bool key_item(const AttnParams &P, int r, KTile &it) {
  const int BH = P.B * P.H, nkt = (P.T + TILE - 1) / TILE;
  const int u = item_index(r);
  if (u >= nkt * BH) return false;
  const int bh = u % BH, kt = u / BH;  // the first key tiles are seen by the most queries
  it.k0 = kt * TILE;
  it.b = bh / P.H;
  it.h = bh % P.H;
  it.qt0 = kt;
  const int w = P.window;
  const int qhi = w >= 0 ? min(P.T - 1, it.k0 + TILE - 1 + w) : P.T - 1;
  it.n = qhi / TILE + 1 - kt;
  return true;
}
struct KCursor {  // (item, query tile) walk of this CTA
  KTile it;
  int i, j;
  bool valid;
  __device__ __forceinline__ void start(const AttnParams &P) { i = 0; j = 0; valid = key_item(P, 0, it); }
  __device__ __forceinline__ void next(const AttnParams &P) {
    if (++j == it.n) { j = 0; ++i; valid = key_item(P, i, it); }
  }
};

// ------------------------------------------------------------------------------------------
// forward
// ------------------------------------------------------------------------------------------
// K and V tiles in separate two-stage rings (a K stage frees as soon as its S MMA is done, a V
// stage after its P.V MMA); the softmax warps release S as soon as it is in registers, so the
// next tile's S = Q K^T runs on the tensor core while they compute P.
enum { F_QFULL, F_K0, F_K1, F_V0, F_V1, F_KFREE0, F_KFREE1, F_VFREE0, F_VFREE1, F_SFULL, F_SFREE,
       F_PFULL_A, F_PFULL_B, F_OFULL_A, F_OFULL_B, F_NBAR };
constexpr int FWD_SMEM = 5 * TILE_BYTES + 1024 + 256;

__global__ void __launch_bounds__(192, 2)
attn_fwd_tc(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmO,
            const AttnParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *sQ = smem, *sK0 = smem + TILE_BYTES, *sV0 = smem + 3 * TILE_BYTES;  // 2 stages each
  uint64_t *bar = (uint64_t *)(smem + 5 * TILE_BYTES);
  uint32_t *tmem_holder = (uint32_t *)(bar + F_NBAR);
  volatile int *abort_flag = (volatile int *)(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = P.B * P.H, nqt = (P.T + TILE - 1) / TILE;
  const int qt = nqt - 1 - (int)blockIdx.x / BH;  // heaviest (last) query tiles first
  const int bh = (int)blockIdx.x % BH, b = bh / P.H, h = bh % P.H;
  const int q0 = qt * TILE, row0 = b * P.T, w = P.window;
  const int kt0 = (w >= 0 ? max(0, q0 - w) : 0) / TILE;
  const int kt1 = (min(P.T, q0 + TILE) + TILE - 1) / TILE;
  const int n = kt1 - kt0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < F_NBAR; ++i)
      mbar_init(&bar[i], (i == F_PFULL_A || i == F_PFULL_B || i == F_SFREE) ? 4 : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;  // S: columns [0,128), O: [128,192), P (bf16): [192,256)

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(&bar[F_QFULL], TILE_BYTES);
      tma_load_2d(sQ, &tmQKV, &bar[F_QFULL], h * HD, row0 + q0);
      for (int j = 0; j < n; ++j) {
        const int s = j & 1, use = j >> 1, k0 = (kt0 + j) * TILE;
        if (use > 0 && !mbar_wait(&bar[F_KFREE0 + s], (use - 1) & 1, abort_flag, P.err)) break;
        mbar_expect_tx(&bar[F_K0 + s], TILE_BYTES);
        tma_load_2d(sK0 + s * TILE_BYTES, &tmQKV, &bar[F_K0 + s], P.C + h * HD, row0 + k0);
        if (use > 0 && !mbar_wait(&bar[F_VFREE0 + s], (use - 1) & 1, abort_flag, P.err)) break;
        mbar_expect_tx(&bar[F_V0 + s], TILE_BYTES);
        tma_load_2d(sV0 + s * TILE_BYTES, &tmQKV, &bar[F_V0 + s], 2 * P.C + h * HD, row0 + k0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t aQ = smem_u32(sQ), aK0 = smem_u32(sK0), aV0 = smem_u32(sV0);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        if (!mbar_wait(&bar[F_K0 + s], (j >> 1) & 1, abort_flag, P.err)) return false;
        tc_fence_after();
        mma_qk(tmem, aQ, aK0 + s * TILE_BYTES, TILE);
        umma_commit(&bar[F_SFULL]);
        umma_commit(&bar[F_KFREE0 + s]);  // K_j is no longer read
        return true;
      };
      bool ok = mbar_wait(&bar[F_QFULL], 0, abort_flag, P.err) && issue_s(0);
      for (int j = 0; ok && j < n; ++j) {
        if (!mbar_wait(&bar[F_SFREE], j & 1, abort_flag, P.err)) break;  // S_j is in registers
        tc_fence_after();
        if (j + 1 < n && !issue_s(j + 1)) break;
        // O += P V in two halves of 64 keys, each as soon as its half of P is in TMEM
        if (!mbar_wait(&bar[F_PFULL_A], j & 1, abort_flag, P.err)) break;
        if (!mbar_wait(&bar[F_V0 + (j & 1)], (j >> 1) & 1, abort_flag, P.err)) break;
        tc_fence_after();
        mma_pv_ts_half(tmem + 128, tmem + 192, aV0 + (j & 1) * TILE_BYTES, 0, j > 0);
        umma_commit(&bar[F_OFULL_A]);
        if (!mbar_wait(&bar[F_PFULL_B], j & 1, abort_flag, P.err)) break;
        tc_fence_after();
        mma_pv_ts_half(tmem + 128, tmem + 192, aV0 + (j & 1) * TILE_BYTES, 1, true);
        umma_commit(&bar[F_OFULL_B]);
        umma_commit(&bar[F_VFREE0 + (j & 1)]);  // V_j is no longer read
      }
    }
    __syncwarp();
  } else {
    const int q = warp & 3, r = q * 32 + lane, qi = q0 + r;
    const uint32_t tS = tmem + ((uint32_t)(q * 32) << 16), tO = tS + 128, tP = tS + 192;
    float m2 = -INFINITY, l = 0.f;
    bool have = false, ok = true;
    // Each 128-key tile in two halves of 64 keys, each an online-softmax step of its own (a
    // thread holds 64 scores at a time): its P goes to TMEM and its half of O += P V is
    // issued while the next half is computed. S is released once both halves are loaded.
    for (int j = 0; j < n; ++j) {
      const int k0 = (kt0 + j) * TILE;
      if (!warp_wait(&bar[F_SFULL], j & 1, abort_flag, P.err)) { ok = false; break; }
      tc_fence_after();
      const bool interior = (k0 + TILE - 1 <= q0) && (w < 0 || k0 >= q0 + TILE - 1 - w);
      // keys admitted for query qi: max(0, qi-w) <= key <= qi  ->  lo <= i <= hi (tile-local)
      const int hi = qi - k0;
      const int lo = w >= 0 ? qi - w - k0 : -1;
      auto half_step = [&](auto half_c) -> bool {
        constexpr int HF = decltype(half_c)::value;
        uint32_t s0[32], s1[32];
        tmem_ld32_nw(tS + 64 * HF, s0);
        tmem_ld32_nw(tS + 64 * HF + 32, s1);
        tmem_wait_ld32(s0);
        reg_fence32(s1);
        if (HF == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar[F_SFREE]);  // the MMA warp may overwrite S now
        }
        float sv[64];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          sv[i] = __uint_as_float(s0[i]);
          sv[32 + i] = __uint_as_float(s1[i]);
        }
        if (!interior) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            sv[i] = (64 * HF + i <= hi && 64 * HF + i >= lo) ? sv[i] : -INFINITY;
        }
        // row max as a tree of independent partial maxima
        float mp[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = sv[k];
#pragma unroll
        for (int i = 8; i < 56; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mp[k] = fmax3(mp[k], sv[i + k], sv[i + 8 + k]);
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = fmaxf(mp[k], sv[56 + k]);
        const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                               fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
        const float mt = mx * P.scale_log2;  // -inf stays -inf (scale > 0)
        float mnew = m2;
        bool resc = false;
        if (mt > -INFINITY) {
          if (!have) mnew = mt;
          else if (mt > m2 + 8.f) { mnew = mt; resc = true; }
        }
        const bool have_new = have || mt > -INFINITY;
        const float mu = have_new ? mnew : 0.f;  // nothing admitted yet: every sv is -inf
        float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};  // partial sums
        uint32_t pk[2][16];                       // P of the half, packed bf16 pairs
        const float2 sc2 = make_float2(P.scale_log2, P.scale_log2), nmu2 = make_float2(-mu, -mu);
#pragma unroll
        for (int i = 0; i < 64; i += 2) {
          const float2 a2 = fma2(make_float2(sv[i], sv[i + 1]), sc2, nmu2);
          const float p0 = ex2(a2.x), p1 = ex2(a2.y);
          ls2[(i >> 1) & 1] = add2(ls2[(i >> 1) & 1], make_float2(p0, p1));
          pk[i >> 5][(i >> 1) & 15] = pack_bf16(p0, p1);
        }
        const float ls[4] = {ls2[0].x, ls2[1].x, ls2[0].y, ls2[1].y};
        const bool any_resc = __any_sync(0xffffffffu, resc);
        if (HF == 0) {
          // this half's P columns and O are free once the previous tile's P V is done
          if (j > 0) {
            if (!warp_wait(&bar[F_OFULL_B], (j - 1) & 1, abort_flag, P.err)) return false;
            tc_fence_after();
          }
        } else if (any_resc) {
          // O is rescaled below: the first half's P V of this tile must be done
          if (!warp_wait(&bar[F_OFULL_A], j & 1, abort_flag, P.err)) return false;
          tc_fence_after();
        }
        if (any_resc) {
          const float f = resc ? ex2(m2 - mnew) : 1.f;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            float v[32];
            tmem_ld32(tO + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= f;
            tmem_st32(tO + c * 32, v);
          }
          l *= f;
        }
        m2 = mnew;
        have = have_new;
        st_tmem_bf16x32(tP + 32 * HF, pk[0]);
        st_tmem_bf16x32(tP + 32 * HF + 16, pk[1]);
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[HF == 0 ? F_PFULL_A : F_PFULL_B]);
        return true;
      };
      if (!half_step(std::integral_constant<int, 0>{})) { ok = false; break; }
      if (!half_step(std::integral_constant<int, 1>{})) { ok = false; break; }
    }
    if (ok && warp_wait(&bar[F_OFULL_B], (n - 1) & 1, abort_flag, P.err)) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint32_t pk[32];
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float v[32];
        tmem_ld32(tO + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; i += 2) pk[c * 16 + (i >> 1)] = pack_bf16(v[i] * inv, v[i + 1] * inv);
      }
      // O through shared memory (this warp's 32 rows of the Q tile, free now, 128-byte
      // swizzle) and one TMA store; rows past T are clipped by the [B, T, C] tensor map
      uint8_t *stg = sQ + q * 4096;
#pragma unroll
      for (int t = 0; t < 8; ++t)
        *reinterpret_cast<uint4 *>(stg + lane * 128 + ((t ^ (lane & 7)) << 4)) =
            make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
      fence_async_smem();
      __syncwarp();
      if (lane == 0 && q0 + q * 32 < P.T) {  // (a box wholly past T is not issued)
        tma_store_3d(&tmO, stg, h * HD, q0 + q * 32, b);
        bulk_commit();
      }
      if (qi < P.T) P.lse[((size_t)b * P.H + h) * P.T + qi] = (m2 + __log2f(l)) * LN2;
      if (lane == 0) bulk_wait_read<0>();  // the staging smem must outlive the store's reads
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------------------------------
// backward kernels (one CTA per SM): 10 warps. warp 0 TMA, warp 1 TMEM + MMA issue, warps
// 2..9 "row" warps: warp w owns TMEM lane quarter (w % 4) and column half ch = (w - 2) / 4
// (64 of the 128 columns of the S / dP tiles), so every row of a tile is shared by two warps.
// A row warp loads its S and dP columns into registers, releases the accumulators at once
// (the MMA warp then computes the next tile's S and dP while the row warps do the math), and
// writes its bf16 results into tensor memory as the A operand of the next MMAs. An item's
// accumulators are read out before the row warps release the next item's first tile, so the
// next item's accumulating MMAs never overwrite them early.
// ------------------------------------------------------------------------------------------
constexpr int BWD_THREADS = 320;
constexpr int ROW_WARPS = 8;

// 64 consecutive columns (two TMEM loads of 32) of S and dP for this thread's row.
__device__ __forceinline__ void ld_s_dp64(uint32_t tS, uint32_t tdP, uint32_t (&s0)[32],
                                          uint32_t (&s1)[32], uint32_t (&d0)[32],
                                          uint32_t (&d1)[32]) {
  tmem_ld32_nw(tS, s0);
  tmem_ld32_nw(tS + 32, s1);
  tmem_ld32_nw(tdP, d0);
  tmem_ld32_nw(tdP + 32, d1);
  tmem_wait_ld32(s0);
  reg_fence32(s1);
  reg_fence32(d0);
  reg_fence32(d1);
}

// ------------------------------------------------------------------------------------------
// backward: dQ (+ D)
// ------------------------------------------------------------------------------------------
// Per item: Q, dO and O of the query tile (double-buffered); D_i = dO_i . O_i from the smem
// tiles; then for every key tile S = Q K^T, dP = dO V^T, dS = P o (dP - D), dQ += dS K.
constexpr int DQ_STAGES = 4;  // K/V tiles in flight
enum { Q_QDO0, Q_QFREE0 = Q_QDO0 + 2, Q_KV0 = Q_QFREE0 + 2, Q_FREE0 = Q_KV0 + DQ_STAGES,
       Q_SDP = Q_FREE0 + DQ_STAGES, Q_SDPFREE, Q_DS, Q_MM2, Q_NBAR };
constexpr int DQ_QBUF = 3 * TILE_BYTES;  // Q | dO | O
constexpr int DQ_SMEM = (2 * 3 + 2 * DQ_STAGES) * TILE_BYTES + 1024 + 256;
static_assert(DQ_SMEM <= 232448, "dQ kernel shared memory");

__global__ void __launch_bounds__(BWD_THREADS, 1)
attn_bwd_dq_tc(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
               const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmDQ,
               const AttnParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *sK0 = smem + 2 * DQ_QBUF;  // stage s: K at 2s, V at 2s+1 (in tiles)
  uint64_t *bar = (uint64_t *)(smem + (2 * 3 + 2 * DQ_STAGES) * TILE_BYTES);
  uint32_t *tmem_holder = (uint32_t *)(bar + Q_NBAR);
  volatile int *abort_flag = (volatile int *)(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < Q_NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == Q_DS || i == Q_SDPFREE) cnt = ROW_WARPS;
      // the item's last S/dP MMA, then every row warp once its dQ staging (in the item's O
      // tile) has been read by the TMA store
      if (i == Q_QFREE0 || i == Q_QFREE0 + 1) cnt = 1 + ROW_WARPS;
      mbar_init(&bar[i], cnt);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;  // S [0,128), dP [128,256), dQ [256,320), dS [320,384)

  if (warp == 0) {
    if (lane == 0) {
      QTile it;
      int g = 0;
      bool ok = true;
      for (int i = 0; ok && query_item(P, i, it); ++i) {
        const int qb = i & 1, row0 = it.b * P.T;
        if (i >= 2 && !mbar_wait(&bar[Q_QFREE0 + qb], ((i >> 1) - 1) & 1, abort_flag, P.err)) break;
        uint8_t *sQ = smem + qb * DQ_QBUF;
        mbar_expect_tx(&bar[Q_QDO0 + qb], 3 * TILE_BYTES);
        tma_load_2d(sQ, &tmQKV, &bar[Q_QDO0 + qb], it.h * HD, row0 + it.q0);
        tma_load_2d(sQ + TILE_BYTES, &tmDO, &bar[Q_QDO0 + qb], it.h * HD, row0 + it.q0);
        tma_load_2d(sQ + 2 * TILE_BYTES, &tmO, &bar[Q_QDO0 + qb], it.h * HD, row0 + it.q0);
        for (int j = 0; j < it.n; ++j, ++g) {
          const int s = g % DQ_STAGES, use = g / DQ_STAGES, k0 = (it.kt0 + j) * TILE;
          if (use > 0 && !mbar_wait(&bar[Q_FREE0 + s], (use - 1) & 1, abort_flag, P.err)) { ok = false; break; }
          uint8_t *sK = sK0 + s * 2 * TILE_BYTES;
          mbar_expect_tx(&bar[Q_KV0 + s], 2 * TILE_BYTES);
          tma_load_2d(sK, &tmQKV, &bar[Q_KV0 + s], P.C + it.h * HD, row0 + k0);
          tma_load_2d(sK + TILE_BYTES, &tmQKV, &bar[Q_KV0 + s], 2 * P.C + it.h * HD, row0 + k0);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t aQ0 = smem_u32(smem), aK0 = smem_u32(sK0);
      QCursor sc, mc;
      sc.start(P);
      mc.start(P);
      int gs = 0;
      auto issue_sdp = [&]() -> bool {  // S and dP of the next tile in the walk
        const int qb = sc.i & 1, s = gs % DQ_STAGES;
        if (sc.j == 0 && !mbar_wait(&bar[Q_QDO0 + qb], (sc.i >> 1) & 1, abort_flag, P.err)) return false;
        if (!mbar_wait(&bar[Q_KV0 + s], (gs / DQ_STAGES) & 1, abort_flag, P.err)) return false;
        tc_fence_after();
        const uint32_t aQ = aQ0 + qb * DQ_QBUF, adO = aQ + TILE_BYTES;
        const uint32_t aK = aK0 + s * 2 * TILE_BYTES, aV = aK + TILE_BYTES;
        mma_qk(tmem, aQ, aK, TILE);
        mma_qk(tmem + 128, adO, aV, TILE);
        umma_commit(&bar[Q_SDP]);
        if (sc.j + 1 == sc.it.n) umma_commit(&bar[Q_QFREE0 + qb]);  // Q / dO no longer read
        sc.next(P);
        ++gs;
        return true;
      };
      bool ok = !sc.valid || issue_sdp();
      for (int g = 0; ok && mc.valid; ++g, mc.next(P)) {
        if (!mbar_wait(&bar[Q_SDPFREE], g & 1, abort_flag, P.err)) break;
        tc_fence_after();
        if (sc.valid && !issue_sdp()) break;
        if (!mbar_wait(&bar[Q_DS], g & 1, abort_flag, P.err)) break;
        tc_fence_after();
        const uint32_t aK = aK0 + (g % DQ_STAGES) * 2 * TILE_BYTES;
        mma_pv_ts(tmem + 256, tmem + 320, aK, mc.j > 0);  // dQ += dS K (dS in TMEM, K MN-major)
        umma_commit(&bar[Q_MM2]);
        umma_commit(&bar[Q_FREE0 + (g % DQ_STAGES)]);
      }
    }
    __syncwarp();
  } else {
    const int q = warp & 3, ch = (warp - 2) >> 2, r = q * 32 + lane;
    const uint32_t tS = tmem + ((uint32_t)(q * 32) << 16) + ch * 64, tdP = tS + 128;
    const int w = P.window;
    // the lse of this thread's row of an item, loaded from a valid address (index 0 for a row
    // past T, whose value is never used: such a row's P is masked to zero) with no use of the
    // value until the item starts
    auto lse_of = [&](const QTile &t) -> float {
      const int qi = t.q0 + r;
      return ldg_early(P.lse_in + (qi < P.T ? ((size_t)t.b * P.H + t.h) * P.T + qi : 0));
    };
    int g = 0;
    bool ok = true;
    QTile it, nx;
    bool have_it = query_item(P, 0, it);
    float lse_cur = have_it ? lse_of(it) : 0.f;  // (no item: nothing waits on it)
    int pend_qb = -1;  // buffer whose dQ staging a TMA store may still be reading
    for (int i = 0; ok && have_it; ++i) {
      const bool have_nx = query_item(P, i + 1, nx);
      const float lse_nx = lse_of(have_nx ? nx : it);  // in flight during this item
      const int qb = i & 1, q0 = it.q0, qi = q0 + r;
      if (!warp_wait(&bar[Q_QDO0 + qb], (i >> 1) & 1, abort_flag, P.err)) { ok = false; break; }
      // D_i = dO_i . O_i (also written for the dK/dV pass) from the swizzled smem tiles
      float D = 0.f;
      {
        const uint8_t *sdO = smem + qb * DQ_QBUF + TILE_BYTES, *sO = sdO + TILE_BYTES;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int off = r * 128 + ((c ^ (r & 7)) << 4);
          const uint4 av = *reinterpret_cast<const uint4 *>(sO + off);
          const uint4 cv = *reinterpret_cast<const uint4 *>(sdO + off);
          const __nv_bfloat162 *ha = reinterpret_cast<const __nv_bfloat162 *>(&av);
          const __nv_bfloat162 *hc = reinterpret_cast<const __nv_bfloat162 *>(&cv);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float2 fa = __bfloat1622float2(ha[u]), fc = __bfloat1622float2(hc[u]);
            D += fa.x * fc.x + fa.y * fc.y;
          }
        }
      }
      // the previous item's dQ store has read its staging: that item's buffer is free
      if (pend_qb >= 0) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[Q_QFREE0 + pend_qb]);
        pend_qb = -1;
      }
      if (ch == 0 && qi < P.T) P.Dbuf[((size_t)it.b * P.H + it.h) * P.T + qi] = D;
      const float lse2 = lse_cur * LOG2E;
      for (int j = 0; j < it.n; ++j, ++g) {
        const int k0 = (it.kt0 + j) * TILE;
        if (!warp_wait(&bar[Q_SDP], g & 1, abort_flag, P.err)) { ok = false; break; }
        tc_fence_after();
        uint32_t s0[32], s1[32], d0[32], d1[32];
        ld_s_dp64(tS, tdP, s0, s1, d0, d1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[Q_SDPFREE]);  // S / dP may be overwritten now
        const bool interior = (k0 + TILE - 1 <= q0) && (w < 0 || k0 >= q0 + TILE - 1 - w);
        const int hi = qi < P.T ? qi - k0 - ch * 64 : -1;  // admitted local columns: lo..hi
        const int lo = w >= 0 ? qi - w - k0 - ch * 64 : -1;
        uint32_t pk[32];
        // two copies of the loop: interior tiles carry no per-element mask
        auto ds_math = [&](auto masked) {
          constexpr bool MASK = decltype(masked)::value;
#pragma unroll
          for (int k = 0; k < 64; k += 2) {
            const float sa = __uint_as_float(k < 32 ? s0[k] : s1[k - 32]);
            const float sb = __uint_as_float(k < 32 ? s0[k + 1] : s1[k - 31]);
            const float da = __uint_as_float(k < 32 ? d0[k] : d1[k - 32]);
            const float db = __uint_as_float(k < 32 ? d0[k + 1] : d1[k - 31]);
            float x0 = ex2(fmaf(sa, P.scale_log2, -lse2)) * (da - D);
            float x1 = ex2(fmaf(sb, P.scale_log2, -lse2)) * (db - D);
            if (MASK) {
              x0 = (k <= hi && k >= lo) ? x0 : 0.f;
              x1 = (k + 1 <= hi && k + 1 >= lo) ? x1 : 0.f;
            }
            pk[k >> 1] = pack_bf16(x0, x1);
          }
        };
        if (interior) ds_math(std::false_type{});
        else ds_math(std::true_type{});
        // dS is free once the previous dQ MMA is done (for j == 0 the epilogue waited)
        if (j > 0 && !warp_wait(&bar[Q_MM2], (g - 1) & 1, abort_flag, P.err)) { ok = false; break; }
        {
          const uint32_t tdS = tmem + ((uint32_t)(q * 32) << 16) + 320 + ch * 32;
          uint32_t lo16[16], hi16[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) { lo16[t] = pk[t]; hi16[t] = pk[16 + t]; }
          tmem_st16_nw(tdS, lo16);
          tmem_st16_nw(tdS + 16, hi16);
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[Q_DS]);
      }
      if (!ok || !warp_wait(&bar[Q_MM2], (g - 1) & 1, abort_flag, P.err)) { ok = false; break; }
      tc_fence_after();
      float v[32];
      tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + 256 + ch * 32, v);  // dQ columns ch*32..
      // dQ through shared memory (this warp's 32 rows x 32 columns in the item's O tile,
      // 64-byte swizzle) and one TMA store; rows past T are clipped by the [B, T, 3C] map
      uint8_t *stg = smem + qb * DQ_QBUF + 2 * TILE_BYTES + (warp - 2) * 2048;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        *reinterpret_cast<uint4 *>(stg + lane * 64 + ((t ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(pack_bf16(v[8 * t] * P.scale, v[8 * t + 1] * P.scale),
                       pack_bf16(v[8 * t + 2] * P.scale, v[8 * t + 3] * P.scale),
                       pack_bf16(v[8 * t + 4] * P.scale, v[8 * t + 5] * P.scale),
                       pack_bf16(v[8 * t + 6] * P.scale, v[8 * t + 7] * P.scale));
      fence_async_smem();
      __syncwarp();
      if (lane == 0 && q0 + q * 32 < P.T) {
        tma_store_3d(&tmDQ, stg, it.h * HD + ch * 32, q0 + q * 32, it.b);
        bulk_commit();
      }
      pend_qb = qb;
      it = nx;
      have_it = have_nx;
      lse_cur = lse_nx;
    }
    if (lane == 0) bulk_wait_read<0>();  // staging smem must outlive the last store's reads
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------
// backward: dK, dV
// ------------------------------------------------------------------------------------------
// Per item: K and V of the key tile (double-buffered); then for every query tile that sees it
// S^T = K Q^T, dP^T = V dO^T, P^T and dS^T -> TMEM, dV += P^T dO, dK += dS^T Q. The lse and
// D of a query tile are copied from global memory two tiles ahead.
// With WRITE_DS the kernel also writes every dS^T tile (bf16, [B*H][T keys][T queries]) for
// the tensor-core dQ pass (attn_bwd_dq_mma), through a 32 KB staging area, and keeps three
// Q/dO stages. It takes no alignment slack: the dynamic shared memory of a kernel without
// static shared memory starts 1 KB aligned, which the kernel checks (a misaligned start sets
// the error word and the kernel returns without work).
constexpr int DKV_STAGES = 4;     // Q/dO tiles in flight
constexpr int DKV_STAGES_DS = 3;  // the same with dS^T staging (shared memory)
constexpr int LSD_BUFS = 3;       // per-tile lse / D buffers: copied two tiles ahead
enum { K_KV0, K_KVFREE0 = K_KV0 + 2, K_QDO0 = K_KVFREE0 + 2, K_FREE0 = K_QDO0 + DKV_STAGES,
       K_SDP = K_FREE0 + DKV_STAGES, K_SDPFREE, K_PS, K_MM2, K_NBAR };
__host__ __device__ constexpr int dkv_smem(int nst, bool write_ds) {
  return (4 + 2 * nst + (write_ds ? 2 : 0)) * TILE_BYTES + (write_ds ? 0 : 1024) +
         LSD_BUFS * 2 * TILE * 4 + 256;
}
static_assert(dkv_smem(DKV_STAGES, false) <= 232448, "dK/dV kernel shared memory");
static_assert(dkv_smem(DKV_STAGES_DS, true) <= 232448, "dK/dV kernel shared memory");

template <int NST, bool WRITE_DS>
__global__ void __launch_bounds__(BWD_THREADS, 1)
attn_bwd_dkv_tc(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmDO,
                const __grid_constant__ CUtensorMap tmDKV, const __grid_constant__ CUtensorMap tmDST,
                const AttnParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (WRITE_DS && (smem_u32(smem_raw) & 1023u) != 0) {  // no slack for aligning (see above)
    if (threadIdx.x == 0) atomicOr(P.err, GPT_DEVERR_TIMEOUT);
    return;
  }
  uint8_t *smem = WRITE_DS ? smem_raw : align1024(smem_raw);
  uint8_t *sKV0 = smem;                  // buffer b: K at 2b, V at 2b+1 (in tiles)
  uint8_t *sQ0 = smem + 4 * TILE_BYTES;  // stage s: Q at 2s, dO at 2s+1
  uint8_t *sDS = smem + (4 + 2 * NST) * TILE_BYTES;  // dS^T staging: 4 KB per row warp
  float *s_lsd = (float *)(smem + (4 + 2 * NST + (WRITE_DS ? 2 : 0)) * TILE_BYTES);  // [3][lse | D]
  uint64_t *bar = (uint64_t *)(s_lsd + LSD_BUFS * 2 * TILE);
  uint32_t *tmem_holder = (uint32_t *)(bar + K_NBAR);
  volatile int *abort_flag = (volatile int *)(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < K_NBAR; ++i) {
      uint32_t cnt = 1;
      if (i == K_PS || i == K_SDPFREE) cnt = ROW_WARPS;
      // the item's last S/dP MMA, then every row warp once its dV/dK staging (in the item's
      // K/V buffer) has been read by the TMA store
      if (i == K_KVFREE0 || i == K_KVFREE0 + 1) cnt = 1 + ROW_WARPS;
      mbar_init(&bar[i], cnt);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384), P^T [384,448), dS^T [448,512)
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      KTile it;
      int g = 0;
      bool ok = true;
      for (int i = 0; ok && key_item(P, i, it); ++i) {
        const int kb = i & 1, row0 = it.b * P.T;
        if (i >= 2 && !mbar_wait(&bar[K_KVFREE0 + kb], ((i >> 1) - 1) & 1, abort_flag, P.err)) break;
        uint8_t *sK = sKV0 + kb * 2 * TILE_BYTES;
        mbar_expect_tx(&bar[K_KV0 + kb], 2 * TILE_BYTES);
        tma_load_2d(sK, &tmQKV, &bar[K_KV0 + kb], P.C + it.h * HD, row0 + it.k0);
        tma_load_2d(sK + TILE_BYTES, &tmQKV, &bar[K_KV0 + kb], 2 * P.C + it.h * HD, row0 + it.k0);
        for (int j = 0; j < it.n; ++j, ++g) {
          const int s = g % NST, use = g / NST, qq0 = (it.qt0 + j) * TILE;
          if (use > 0 && !mbar_wait(&bar[K_FREE0 + s], (use - 1) & 1, abort_flag, P.err)) { ok = false; break; }
          uint8_t *sQ = sQ0 + s * 2 * TILE_BYTES;
          mbar_expect_tx(&bar[K_QDO0 + s], 2 * TILE_BYTES);
          tma_load_2d(sQ, &tmQKV, &bar[K_QDO0 + s], it.h * HD, row0 + qq0);
          tma_load_2d(sQ + TILE_BYTES, &tmDO, &bar[K_QDO0 + s], it.h * HD, row0 + qq0);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t aKV0 = smem_u32(sKV0), aQ0 = smem_u32(sQ0);
      KCursor sc, mc;
      sc.start(P);
      mc.start(P);
      int gs = 0;
      auto issue_sdp = [&]() -> bool {  // S^T and dP^T of the next tile in the walk
        const int kb = sc.i & 1, s = gs % NST;
        if (sc.j == 0 && !mbar_wait(&bar[K_KV0 + kb], (sc.i >> 1) & 1, abort_flag, P.err)) return false;
        if (!mbar_wait(&bar[K_QDO0 + s], (gs / NST) & 1, abort_flag, P.err)) return false;
        tc_fence_after();
        const uint32_t aK = aKV0 + kb * 2 * TILE_BYTES, aV = aK + TILE_BYTES;
        const uint32_t aQ = aQ0 + s * 2 * TILE_BYTES, adO = aQ + TILE_BYTES;
        mma_qk(tmem, aK, aQ, TILE);         // S^T  = K Q^T
        mma_qk(tmem + 128, aV, adO, TILE);  // dP^T = V dO^T
        umma_commit(&bar[K_SDP]);
        if (sc.j + 1 == sc.it.n) umma_commit(&bar[K_KVFREE0 + kb]);  // K / V no longer read
        sc.next(P);
        ++gs;
        return true;
      };
      bool ok = !sc.valid || issue_sdp();
      for (int g = 0; ok && mc.valid; ++g, mc.next(P)) {
        if (!mbar_wait(&bar[K_SDPFREE], g & 1, abort_flag, P.err)) break;
        tc_fence_after();
        if (sc.valid && !issue_sdp()) break;
        if (!mbar_wait(&bar[K_PS], g & 1, abort_flag, P.err)) break;
        tc_fence_after();
        const uint32_t aQ = aQ0 + (g % NST) * 2 * TILE_BYTES, adO = aQ + TILE_BYTES;
        mma_pv_ts(tmem + 256, tmem + 384, adO, mc.j > 0);  // dV += P^T dO   (P^T in TMEM)
        mma_pv_ts(tmem + 320, tmem + 448, aQ, mc.j > 0);   // dK += dS^T Q  (dS^T in TMEM)
        umma_commit(&bar[K_MM2]);
        umma_commit(&bar[K_FREE0 + (g % NST)]);
      }
    }
    __syncwarp();
  } else {
    const int q = warp & 3, ch = (warp - 2) >> 2, r = q * 32 + lane;
    const int t = threadIdx.x - 64;  // 0..255 among the row warps
    const uint32_t tS = tmem + ((uint32_t)(q * 32) << 16) + ch * 64, tdP = tS + 128;
    const int w = P.window;
    // This thread's share of a query tile's (lse | D): t < 128 lse, else D. It is copied two
    // tiles ahead straight into that tile's shared buffer (cp.async: no register holds it, so
    // nothing waits on the load's latency, which under the dS^T write stream can exceed a
    // tile), always from a valid address; whether it counts (a query past T, or no tile) and
    // the scaling of lse to the log2 domain are applied in place when that tile starts.
    auto fetch = [&](const KCursor &k, float *dst) -> bool {
      const int qi = k.valid ? (k.it.qt0 + k.j) * TILE + (t & 127) : P.T;
      const bool valid = qi < P.T;
      const size_t li = valid ? ((size_t)k.it.b * P.H + k.it.h) * P.T + qi : 0;
      cp_async4(dst, (t < 128 ? P.lse_in : P.Dbuf) + li);
      return valid;
    };
    const float lsd_scale = t < 128 ? LOG2E : 1.f;
    bool ok = true;
    KCursor cur, c1;  // this tile and the next one
    cur.start(P);
    c1 = cur;
    c1.next(P);
    bool ok0 = fetch(cur, s_lsd + t);  // validity of this tile's value and the next one's
    cp_async_commit();
    bool ok1 = fetch(c1, s_lsd + 2 * TILE + t);
    cp_async_commit();
    int lb = 0;  // this tile's buffer (g mod 3)
    int pend_kb = -1;  // buffer whose dV/dK staging a TMA store may still be reading
    for (int g = 0; cur.valid; ++g) {
      const KTile it = cur.it;
      const int j = cur.j, kb = cur.i & 1, k0 = it.k0, ki = k0 + r, qq0 = (it.qt0 + j) * TILE;
      // this query tile's lse and D are in buffer g & 1; one barrier per tile (the other
      // buffer may still be read by a warp finishing the previous tile)
      float *lsd = s_lsd + lb * 2 * TILE;
      cp_async_wait_group<1>();  // this tile's copy has landed (the next tile's may not have)
      lsd[t] = ok0 ? lsd[t] * lsd_scale : 0.f;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      // the previous item's dV/dK store has read its staging: that K/V buffer is free
      if (pend_kb >= 0) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[K_KVFREE0 + pend_kb]);
        pend_kb = -1;
      }
      const KCursor nx = c1;
      c1.next(P);
      // every row warp is past the barrier, so done with the previous tile and its buffer,
      // which now takes the values of the tile after the next one
      const int lb2 = lb == 0 ? 2 : lb - 1;  // (g + 2) mod 3
      ok0 = ok1;
      ok1 = fetch(c1, s_lsd + lb2 * 2 * TILE + t);
      cp_async_commit();
      lb = lb == 2 ? 0 : lb + 1;
      cur = nx;
      // after an abort every row warp still passes the named barrier of each tile
      if (ok) ok = warp_wait(&bar[K_SDP], g & 1, abort_flag, P.err);
      if (!ok) continue;
      tc_fence_after();
      const bool interior = (k0 + TILE - 1 <= qq0) && (w < 0 || k0 >= qq0 + TILE - 1 - w) &&
                            (qq0 + TILE <= P.T);
      // queries admitted for key ki: ki <= q <= ki + w, q < T  ->  local columns lo..hi
      const int lo = ki - qq0 - ch * 64;
      const int hi = min(P.T - 1, w >= 0 ? ki + w : P.T - 1) - qq0 - ch * 64;
      const float4 *L4 = reinterpret_cast<const float4 *>(lsd + ch * 64);
      const float4 *D4 = reinterpret_cast<const float4 *>(lsd + TILE + ch * 64);
      const uint32_t tPT = tmem + ((uint32_t)(q * 32) << 16) + 384 + ch * 32, tdST = tPT + 64;
      // P^T and dS^T of this thread's 64 columns, packed bf16 pairs, in registers first; the
      // tensor-memory copies wait for the previous tile's dV / dK MMAs (which read P^T / dS^T)
      // only after the math, so those MMAs run under it. The 64 columns are taken in two
      // halves of 32 (S and dP of one half in registers at a time, which keeps the row warps
      // within their registers); the accumulators are released after the second half's loads.
      uint32_t pp[32], pd[32];
      uint32_t sv[32], dv[32];
      // two copies of the loop: interior tiles carry no per-element mask
      auto pds_math = [&](auto masked, auto half_c) {
      constexpr bool MASK = decltype(masked)::value;
      constexpr int half = decltype(half_c)::value;
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const int c = 32 * half + i;  // column within this thread's 64
        const float4 L = L4[c >> 2], Dv = D4[c >> 2];
        const float lv[4] = {L.x, L.y, L.z, L.w}, dl[4] = {Dv.x, Dv.y, Dv.z, Dv.w};
        float pr[4], dr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float pv = ex2(fmaf(__uint_as_float(sv[i + e]), P.scale_log2, -lv[e]));
          if (MASK) pv = (c + e <= hi && c + e >= lo) ? pv : 0.f;
          pr[e] = pv;
          dr[e] = pv * (__uint_as_float(dv[i + e]) - dl[e]);
        }
        pp[c >> 1] = pack_bf16(pr[0], pr[1]);
        pp[(c >> 1) + 1] = pack_bf16(pr[2], pr[3]);
        pd[c >> 1] = pack_bf16(dr[0], dr[1]);
        pd[(c >> 1) + 1] = pack_bf16(dr[2], dr[3]);
      }
      };
      tmem_ld32_nw(tS, sv);
      tmem_ld32_nw(tdP, dv);
      tmem_wait_ld32(sv);
      reg_fence32(dv);
      if (interior) pds_math(std::false_type{}, std::integral_constant<int, 0>{});
      else pds_math(std::true_type{}, std::integral_constant<int, 0>{});
      tmem_ld32_nw(tS + 32, sv);
      tmem_ld32_nw(tdP + 32, dv);
      tmem_wait_ld32(sv);
      reg_fence32(dv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[K_SDPFREE]);  // S^T / dP^T may be overwritten now
      if (interior) pds_math(std::false_type{}, std::integral_constant<int, 1>{});
      else pds_math(std::true_type{}, std::integral_constant<int, 1>{});
      // P^T / dS^T in tensor memory are free once the previous dV / dK MMAs are done (for
      // j == 0 the previous item's epilogue waited for them)
      if (j > 0) {
        ok = warp_wait(&bar[K_MM2], (g - 1) & 1, abort_flag, P.err);
        if (!ok) continue;
      }
      tmem_st16_nw(tPT, *reinterpret_cast<const uint32_t(*)[16]>(&pp[0]));
      tmem_st16_nw(tPT + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pp[16]));
      tmem_st16_nw(tdST, *reinterpret_cast<const uint32_t(*)[16]>(&pd[0]));
      tmem_st16_nw(tdST + 16, *reinterpret_cast<const uint32_t(*)[16]>(&pd[16]));
      if (WRITE_DS) {
        // this warp's dS^T staging slot must have been read by its last store; then the same
        // bf16 dS^T row goes into it (128-byte swizzle)
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        uint8_t *slot = sDS + (warp - 2) * 4096;
#pragma unroll
        for (int c = 0; c < 8; ++c)  // 16-byte chunk c of the 128-byte row
          *reinterpret_cast<uint4 *>(slot + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_uint4(pd[4 * c], pd[4 * c + 1], pd[4 * c + 2], pd[4 * c + 3]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[K_PS]);
      if (WRITE_DS) {  // dS^T rows k0+q*32.. (keys) x queries qq0+ch*64.. to [B*H][T][T]
        fence_async_smem();
        __syncwarp();
        if (lane == 0 && qq0 + ch * 64 < P.T && k0 + q * 32 < P.T) {
          tma_store_3d(&tmDST, sDS + (warp - 2) * 4096, qq0 + ch * 64, k0 + q * 32,
                       it.b * P.H + it.h);
          bulk_commit();
        }
      }
      if (j + 1 < it.n) continue;
      // the item's last query tile: dV / dK out (column half 0 writes dV, half 1 writes dK
      // times the softmax scale)
      ok = warp_wait(&bar[K_MM2], g & 1, abort_flag, P.err);
      if (!ok) continue;
      tc_fence_after();
      const float f = ch ? P.scale : 1.f;
      // through shared memory (this warp's 32 rows in the item's K/V buffer, free now,
      // 128-byte swizzle) and one TMA store; rows past T are clipped by the [B, T, 3C] map
      uint8_t *stg = sKV0 + kb * 2 * TILE_BYTES + (warp - 2) * 4096;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + 256 + ch * 64 + c * 32, v);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4 *>(stg + lane * 128 + (((4 * c + u) ^ (lane & 7)) << 4)) =
              make_uint4(pack_bf16(v[8 * u] * f, v[8 * u + 1] * f),
                         pack_bf16(v[8 * u + 2] * f, v[8 * u + 3] * f),
                         pack_bf16(v[8 * u + 4] * f, v[8 * u + 5] * f),
                         pack_bf16(v[8 * u + 6] * f, v[8 * u + 7] * f));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0 && k0 + q * 32 < P.T) {
        tma_store_3d(&tmDKV, stg, (ch ? P.C : 2 * P.C) + it.h * HD, k0 + q * 32, it.b);
        bulk_commit();
      }
      pend_kb = kb;
    }
    cp_async_wait_all();  // the last (unused) lse / D copy has landed
    if (lane == 0) bulk_wait_all();  // every store of this warp (dK/dV, dS^T) has completed
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}
// ------------------------------------------------------------------------------------------
// backward, dQ from the stored dS^T (used with attn_bwd_dkv_tc<.., true>)
// ------------------------------------------------------------------------------------------
// D_i = dO_i . O_i for every row (b, t) and head: a warp per row, 16-byte loads across the
// row; the 8 lanes that hold one head's 64 columns combine their partial dots (fixed order).
__global__ void __launch_bounds__(256)
attn_bwd_prep_d(const bf16 *__restrict__ O, const bf16 *__restrict__ dO, float *__restrict__ D,
                int B, int T, int C, int H) {
  const int lane = threadIdx.x & 31;
  const long rows = (long)B * T;
  for (long m = blockIdx.x * 8L + (threadIdx.x >> 5); m < rows; m += gridDim.x * 8L) {
    const int b = (int)(m / T), t = (int)(m % T);
    for (int c0 = 0; c0 < C; c0 += 256) {  // 256 columns = 4 heads per pass
      const int col = c0 + lane * 8;
      float acc = 0.f;
      if (col < C) {
        const uint4 av = *reinterpret_cast<const uint4 *>(O + m * C + col);
        const uint4 cv = *reinterpret_cast<const uint4 *>(dO + m * C + col);
        const __nv_bfloat162 *ha = reinterpret_cast<const __nv_bfloat162 *>(&av);
        const __nv_bfloat162 *hc = reinterpret_cast<const __nv_bfloat162 *>(&cv);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 fa = __bfloat1622float2(ha[u]), fc = __bfloat1622float2(hc[u]);
          acc += fa.x * fc.x + fa.y * fc.y;
        }
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      acc += __shfl_xor_sync(0xffffffffu, acc, 4);
      const int h = col / HD;
      if ((lane & 7) == 0 && col < C) D[((long)b * H + h) * T + t] = acc;
    }
  }
}

// dQ_i = scale * sum_j dS_ij K_j over the key tiles a query tile sees, on the tensor cores:
// persistent CTAs over query tiles (the heavy-first snake schedule of the other passes); per
// 64-key block a TMA load of the dS^T block (MN-major A: 64 keys x 128 queries) and of the K
// block (MN-major B: 64 keys x 64 head dims), 4 MMAs of 128x64x16 into a TMEM accumulator
// (double-buffered across items); 4 epilogue warps scale, round and TMA-store dQ.
constexpr int DQM_STAGES = 6;
constexpr int DQM_A = TILE * 64 * 2;  // 16 KB
constexpr int DQM_B = 64 * 64 * 2;    // 8 KB
constexpr int DQM_STAGE = DQM_A + DQM_B;
constexpr int DQM_THREADS = 192;      // TMA, MMA, 4 epilogue warps
enum { M_FULL0, M_EMPTY0 = M_FULL0 + DQM_STAGES, M_TFULL0 = M_EMPTY0 + DQM_STAGES,
       M_TEMPTY0 = M_TFULL0 + 2, M_NBAR = M_TEMPTY0 + 2 };
constexpr int DQM_SMEM = DQM_STAGES * DQM_STAGE + 4 * 4096 + 1024 + 256;
static_assert(DQM_SMEM <= 232448, "dQ kernel shared memory");

__global__ void __launch_bounds__(DQM_THREADS, 1)
attn_bwd_dq_mma(const __grid_constant__ CUtensorMap tmDST, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmDQ, const AttnParams P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *stg = smem + DQM_STAGES * DQM_STAGE;  // 4 x 4 KB output staging
  uint64_t *bar = (uint64_t *)(stg + 4 * 4096);
  uint32_t *tmem_holder = (uint32_t *)(bar + M_NBAR);
  volatile int *abort_flag = (volatile int *)(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < M_NBAR; ++i)
      mbar_init(&bar[i], (i == M_TEMPTY0 || i == M_TEMPTY0 + 1) ? 4 : 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;  // dQ accumulators: columns [0,64) and [64,128)

  if (warp == 0) {
    if (lane == 0) {  // TMA producer
      QTile it;
      int g = 0;
      bool ok = true;
      for (int i = 0; ok && query_item(P, i, it); ++i) {
        const int bh = it.b * P.H + it.h;
        for (int j = 0; ok && j < it.n; ++j) {
          const int k0 = (it.kt0 + j) * TILE;
          for (int kb = 0; kb < 2; ++kb, ++g) {
            const int s = g % DQM_STAGES, use = g / DQM_STAGES;
            if (use > 0 && !mbar_wait(&bar[M_EMPTY0 + s], (use - 1) & 1, abort_flag, P.err)) {
              ok = false;
              break;
            }
            uint8_t *sA = smem + s * DQM_STAGE;
            mbar_expect_tx(&bar[M_FULL0 + s], DQM_STAGE);
            // dS^T[bh][keys k0+64kb..][queries q0..q0+127]: two 64-query boxes
            tma_load_3d(sA, &tmDST, &bar[M_FULL0 + s], it.q0, k0 + 64 * kb, bh);
            tma_load_3d(sA + DQM_A / 2, &tmDST, &bar[M_FULL0 + s], it.q0 + 64, k0 + 64 * kb, bh);
            // K[keys][head dims] of head h, batch b
            tma_load_2d(sA + DQM_A, &tmK, &bar[M_FULL0 + s], P.C + it.h * HD,
                        it.b * P.T + k0 + 64 * kb);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      const uint32_t id = idesc_bf16(HD, 1, 1);  // M = 128, N = 64, both operands MN-major
      QTile it;
      int g = 0;
      bool ok = true;
      for (int i = 0; ok && query_item(P, i, it); ++i) {
        const int acc = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (!mbar_wait(&bar[M_TEMPTY0 + acc], (use & 1u) ^ 1u, abort_flag, P.err)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * 64);
        for (int j = 0; ok && j < it.n; ++j)
          for (int kb = 0; kb < 2; ++kb, ++g) {
            const int s = g % DQM_STAGES;
            if (!mbar_wait(&bar[M_FULL0 + s], (g / DQM_STAGES) & 1, abort_flag, P.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sA = smem_u32(smem + s * DQM_STAGE);
            const uint64_t ad = sdesc(sA, 8192u, 1024u), bd = sdesc(sA + DQM_A, 8192u, 1024u);
#pragma unroll
            for (int k = 0; k < 4; ++k)  // 16 keys per MMA: 16 rows of 128 bytes
              umma_bf16(d, ad + (uint64_t)((k * 2048) >> 4), bd + (uint64_t)((k * 2048) >> 4), id,
                        (j > 0 || kb > 0 || k > 0) ? 1u : 0u);
            umma_commit(&bar[M_EMPTY0 + s]);
          }
        if (!ok) break;
        umma_commit(&bar[M_TFULL0 + acc]);
      }
    }
    __syncwarp();
  } else {  // epilogue: warp w reads TMEM lane quarter w % 4
    const int q = warp & 3;
    uint8_t *ws = stg + (warp - 2) * 4096;
    QTile it;
    for (int i = 0; query_item(P, i, it); ++i) {
      const int acc = i & 1;
      const uint32_t use = (uint32_t)(i >> 1);
      if (!warp_wait(&bar[M_TFULL0 + acc], use & 1u, abort_flag, P.err)) break;
      tc_fence_after();
      float v0[32], v1[32];
      const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 64);
      tmem_ld32(ta, v0);
      tmem_ld32(ta + 32, v1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[M_TEMPTY0 + acc]);  // the MMA may reuse it
      if (lane == 0) bulk_wait_read<0>();                  // the staging slot is free
      __syncwarp();
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const float *v = t < 4 ? v0 : v1;
        const int b8 = (t & 3) * 8;
        *reinterpret_cast<uint4 *>(ws + lane * 128 + ((t ^ (lane & 7)) << 4)) =
            make_uint4(pack_bf16(v[b8] * P.scale, v[b8 + 1] * P.scale),
                       pack_bf16(v[b8 + 2] * P.scale, v[b8 + 3] * P.scale),
                       pack_bf16(v[b8 + 4] * P.scale, v[b8 + 5] * P.scale),
                       pack_bf16(v[b8 + 6] * P.scale, v[b8 + 7] * P.scale));
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0 && it.q0 + q * 32 < P.T) {
        tma_store_3d(&tmDQ, ws, it.h * HD, it.q0 + q * 32, it.b);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// [rows, cols] bf16 matrix with row stride ld elements; box 64 columns x box_rows rows, SW128.
bool map_rows(CUtensorMap *m, const void *base, long cols, long rows, long ld, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (void *)base, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map over a [B, T, cols] bf16 tensor (row stride ld elements) for the epilogue TMA
// stores: box {box_cols, 32 rows, 1}; rows t >= T of a batch are outside the map, so a store
// of a ragged last tile is clipped at the batch boundary.
bool map_btc(CUtensorMap *m, const void *base, long cols, long T, long B, long ld, int box_cols,
             CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)(ld * 2 * T)};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, 32u, 1u};
  cuuint32_t es[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void *)base, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// dS^T [B*H][T keys][T queries] bf16: box {64 queries, box_keys keys, 1}, SW128.
bool map_dst(CUtensorMap *m, const void *base, long T, long BH, int box_keys) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)T, (cuuint64_t)T, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)T * 2, (cuuint64_t)(T * T * 2)};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_keys, 1u};
  cuuint32_t es[3] = {1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void *)base, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

AttnParams make_params(int B, int T, int C, int H, int window, unsigned *err) {
  AttnParams p;
  memset(&p, 0, sizeof(p));
  p.B = B; p.T = T; p.C = C; p.H = H; p.window = window;
  p.scale = 1.0f / sqrtf((float)HD);
  p.scale_log2 = p.scale * LOG2E;
  p.err = err;
  return p;
}

int attn_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

bool smem_attrs_set = false;
cudaError_t set_attrs() {
  if (smem_attrs_set) return cudaSuccess;
  CUDA_TRY(cudaFuncSetAttribute(attn_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, FWD_SMEM));
  CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, DQ_SMEM));
  CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkv_tc<DKV_STAGES, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                dkv_smem(DKV_STAGES, false)));
  CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dkv_tc<DKV_STAGES_DS, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                dkv_smem(DKV_STAGES_DS, true)));
  CUDA_TRY(cudaFuncSetAttribute(attn_bwd_dq_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, DQM_SMEM));
  smem_attrs_set = true;
  return cudaSuccess;
}

}  // namespace

bool attention_tc_supported(int C, int H) { return C / H == HD && C % H == 0 && (C % 8) == 0; }

cudaError_t launch_attention_fwd_tc(const bf16 *qkv, bf16 *o, float *lse, int B, int T, int C,
                                    int H, int window, unsigned *err, cudaStream_t st) {
  CUDA_TRY(set_attrs());
  CUtensorMap m, mo;
  if (!map_rows(&m, qkv, 3L * C, (long)B * T, 3L * C) ||
      !map_btc(&mo, o, C, T, B, C, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  AttnParams p = make_params(B, T, C, H, window, err);
  p.o = o;
  p.lse = lse;
  const int nqt = (T + TILE - 1) / TILE;
  attn_fwd_tc<<<B * H * nqt, 192, FWD_SMEM, st>>>(m, mo, p);  // two CTAs per SM
  return cudaGetLastError();
}

cudaError_t launch_attention_bwd_tc(const bf16 *qkv, const bf16 *o, const bf16 *dout,
                                    const float *lse, float *Dbuf, bf16 *dqkv, int B, int T,
                                    int C, int H, int window, unsigned *err, cudaStream_t st,
                                    bf16 *dst, bool d_ready) {
  CUDA_TRY(set_attrs());
  CUtensorMap mq, md, mo, mdq, mdkv;
  if (!map_rows(&mq, qkv, 3L * C, (long)B * T, 3L * C) ||
      !map_rows(&md, dout, (long)C, (long)B * T, (long)C) ||
      !map_rows(&mo, o, (long)C, (long)B * T, (long)C) ||
      !map_btc(&mdq, dqkv, 3L * C, T, B, 3L * C, 32, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !map_btc(&mdkv, dqkv, 3L * C, T, B, 3L * C, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  AttnParams p = make_params(B, T, C, H, window, err);
  p.O = o;
  p.dO = dout;
  p.lse_in = lse;
  p.Dbuf = Dbuf;
  p.dqkv = dqkv;
  const int items = B * H * ((T + TILE - 1) / TILE);
  const int grid = items < attn_sms() ? items : attn_sms();  // one CTA per SM
  if (dst) {
    // D, then dK/dV writing dS^T, then dQ = dS K from the stored dS^T on the tensor cores
    CUtensorMap mst, mld, mk, mdq64;
    if (!map_dst(&mst, dst, T, (long)B * H, 32) || !map_dst(&mld, dst, T, (long)B * H, 64) ||
        !map_rows(&mk, qkv, 3L * C, (long)B * T, 3L * C, 64) ||
        !map_btc(&mdq64, dqkv, 3L * C, T, B, 3L * C, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    if (!d_ready) {  // D = rowsum(dO * O), unless the producer of dO wrote it alongside
      const long rows = (long)B * T;
      const int pb = (int)((rows + 7) / 8 < 148 * 16 ? (rows + 7) / 8 : 148 * 16);
      attn_bwd_prep_d<<<pb, 256, 0, st>>>(o, dout, Dbuf, B, T, C, H);
      CUDA_TRY(cudaGetLastError());
    }
    attn_bwd_dkv_tc<DKV_STAGES_DS, true><<<grid, BWD_THREADS, dkv_smem(DKV_STAGES_DS, true), st>>>(
        mq, md, mdkv, mst, p);
    CUDA_TRY(cudaGetLastError());
    attn_bwd_dq_mma<<<grid, DQM_THREADS, DQM_SMEM, st>>>(mld, mk, mdq64, p);
    return cudaGetLastError();
  }
  attn_bwd_dq_tc<<<grid, BWD_THREADS, DQ_SMEM, st>>>(mq, md, mo, mdq, p);
  CUDA_TRY(cudaGetLastError());
  attn_bwd_dkv_tc<DKV_STAGES, false><<<grid, BWD_THREADS, dkv_smem(DKV_STAGES, false), st>>>(
      mq, md, mdkv, mdkv, p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Attention backward that allocates nothing.
//
// For callers that cannot call cudaMalloc (for example code running inside a memory pool
// or an allocator hook that must not re-enter the allocator, or a host that only owns the
// tensors it passes in): the backward's per-row scratch D = rowsum(dO * O) lives in this
// file-scope device array instead of a caller buffer. Every GPU that loads the library
// keeps NOALLOC_D_MAX floats (4 MiB) of it until the process exits. The kernels below write
// D for every row before reading it, so nothing has to be cleared between calls. All calls
// on a device share the array: calls that overlap on the GPU (different streams, no
// ordering) race on it.
// ------------------------------------------------------------------------------------------
constexpr size_t NOALLOC_D_MAX = 1u << 20;  // B * n_head * T rows
static __device__ __align__(256) float g_noalloc_D[NOALLOC_D_MAX];

namespace {
constexpr int NOALLOC_MAX_DEVICES = 64;
// device address of g_noalloc_D per device ordinal; filled at most once per slot (host
// threads that race on a first call all look up the same address, one store wins)
std::atomic<float *> g_noalloc_D_addr[NOALLOC_MAX_DEVICES];

// Device address of g_noalloc_D on the current device, looked up on the first call there. In
// host code the symbol itself is only a host-side stand-in, never a device address. The
// cached address belongs to the device's current context: cudaDeviceReset invalidates it.
cudaError_t noalloc_D_address(float **out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= NOALLOC_MAX_DEVICES) return cudaErrorInvalidDevice;
  float *a = g_noalloc_D_addr[dev].load(std::memory_order_acquire);
  if (!a) {
    void *ptr = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&ptr, g_noalloc_D));
    float *expected = nullptr;
    g_noalloc_D_addr[dev].compare_exchange_strong(expected, (float *)ptr,
                                                  std::memory_order_acq_rel);
    a = g_noalloc_D_addr[dev].load(std::memory_order_acquire);
  }
  *out = a;
  return cudaSuccess;
}
}  // namespace

size_t attention_bwd_noalloc_max_rows() { return NOALLOC_D_MAX; }

cudaError_t launch_attention_bwd_tc_noalloc(const bf16 *qkv, const bf16 *o, const bf16 *dout,
                                            const float *lse, bf16 *dqkv, int B, int T, int C,
                                            int H, int window, unsigned *err, cudaStream_t st) {
  if ((size_t)B * H * T > NOALLOC_D_MAX) return cudaErrorInvalidValue;
  float *D = nullptr;
  CUDA_TRY(noalloc_D_address(&D));
  return launch_attention_bwd_tc(qkv, o, dout, lse, D, dqkv, B, T, C, H, window, err, st,
                                 nullptr);
}
