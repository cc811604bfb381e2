// bf16 GEMM on the 5th-generation tensor cores (sm_100a): tcgen05.mma with operands staged
// in shared memory by TMA (128-byte swizzle) and fp32 accumulators in tensor memory (TMEM).
//
//   acc[m][n] = sum_k A[m][k] * B[n][k]
//
// A and B may each be K-major (k contiguous) or MN-major (m / n contiguous); the MMA reads
// both layouts directly (instruction-descriptor transpose bits), so the weight-gradient and
// data-gradient GEMMs of the backward pass need no transposed copies.
//
// Structure: persistent CTAs (one per SM), 10 warps.
//   warp 0      TMA producer: fills a ring of shared-memory stages (A 128x128, B 256x128 or,
//               for CTA pairs, this CTA's 128x128 half of B), K as two 64-element chunks
//   warp 1      TMEM allocator and MMA issuer (one thread): 8 MMAs of K = 16 per stage
//               (128x256 per CTA, or 256x256 per CTA pair with cta_group::2);
//               tcgen05.commit frees the stage; a second commit marks the accumulator full
//   warps 2..9  epilogue: tcgen05.ld of the fp32 accumulator (one row per thread, two warps
//               per TMEM lane quarter, 128 columns each), the fused epilogue, staging in
//               swizzled shared memory and TMA tensor stores (fp32 accumulate: TMA reduce-add)
// The launcher picks CTA pairs (256-row tiles; the pair halves each SM's shared-memory
// traffic per MMA) or single CTAs, and a K split whose fp32 partials an ordered reduce sums,
// from an estimate of the wave-quantised main loop plus the reduce traffic.
// The accumulator is double-buffered in TMEM (2 x 256 columns), so the epilogue of one tile
// overlaps the MMAs of the next. Every mbarrier wait is bounded: after ~2 s it sets the
// device error word and the CTA leaves through its normal teardown (TMEM is always freed).
#include <cuda.h>

#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace {
using namespace tc;

constexpr int BM = TC_BM, BN = TC_BN, BK = TC_BK;
constexpr int KC = BK / 64;            // 128-byte swizzle chunks per stage along K
constexpr int A_BYTES = BM * BK * 2;   // 32 KB
constexpr int A_CHUNK = BM * 64 * 2;   // 16 KB: one 64-k chunk of a K-major A tile
constexpr int NUM_THREADS = 320;  // producer, MMA, 8 epilogue warps
constexpr int EPI_WARPS = 8;
constexpr int EPI_COLS = BN / 2;  // columns per epilogue warp
constexpr int TMEM_COLS = 512;

enum TcEpi {
  TE_STORE = 0, TE_STORE_GELU, TE_RESID, TE_DGELU, TE_F32_STORE, TE_F32_ACCUM, TE_CE_STATS,
  TE_CE_DS, TE_PARTIAL, TE_STORE_PRE_GELU, TE_DGELU_RECOMP, TE_AXPBY, TE_STORE_DOT
};
// epilogues that read an auxiliary bf16 input of the output's shape
__host__ __device__ constexpr bool epi_has_aux(int e) {
  return e == TE_RESID || e == TE_DGELU || e == TE_DGELU_RECOMP || e == TE_AXPBY ||
         e == TE_STORE_DOT;
}

struct TcParams {
  int M, N, K;
  int num_mt, num_nt, splits, kblocks_per_split, total_kblocks;
  int units;
  int batch;       // independent products (batched GEMM); units = tiles * splits * batch
  int n_fast;      // 1: units walk the N tiles of one M tile first (see unit_coords)
  int a_mn, b_mn;  // 1 = MN-major
  // 1: the operand's map views its contiguous dimension as 64-element chunks, so one TMA
  // load brings a stage's whole operand tile (32 KB per CTA); 0: one load per chunk
  int a_wide, b_wide;
  uint32_t idesc;
  Epi epi;
  float *partial;
  unsigned *err;
};

// Tile coordinates of work unit u. Units are numbered M tile fastest, so that CTAs running at
// the same time share the B tile; when A is the larger operand and does not fit in L2 (the
// lm_head backward's dS chunk, read by the dX and dwte GEMMs) they are numbered N tile
// fastest instead, so that the CTAs reading one A tile run together and A crosses HBM once.
// z is the K split of the unit and bz its product of a batched GEMM.
__device__ __forceinline__ void unit_coords(const TcParams &P, int u, int &mt, int &nt, int &z,
                                            int &bz) {
  if (P.n_fast) {
    nt = u % P.num_nt;
    mt = (u / P.num_nt) % P.num_mt;
  } else {
    mt = u % P.num_mt;
    nt = (u / P.num_mt) % P.num_nt;
  }
  const int zz = u / (P.num_mt * P.num_nt);
  z = zz % P.splits;
  bz = zz / P.splits;
}

// ---------------------------------------------------------------------------------------
// epilogue helpers (one thread = one row, 32 consecutive columns per call)
// ---------------------------------------------------------------------------------------
constexpr float LOG2E_F = 1.4426950408889634f;

// Per-row epilogue operands that do not depend on the accumulators; they are fetched before
// the epilogue waits for a tile, so their latency overlaps the MMAs.
struct EpiRow {
  float lse;  // cross-entropy dS: lse of the row (natural log; scaled where it is used, so
              // that nothing waits on the load before the accumulators are ready)
  float s;    // cross-entropy dS: 1 / (number of loss terms)
  int t;      // cross-entropy: target column of the row (-1 for rows past M)
};
template <int EPI>
__device__ __forceinline__ EpiRow epi_row(const TcParams &P, int row) {
  EpiRow r{0.f, 0.f, -1};
  const Epi &e = P.epi;
  // Loaded unconditionally from a valid row (a row past M reads row M-1: nothing of such a row
  // is stored or written), so that no select on the loaded values makes the warp wait for
  // them before the accumulators are ready.
  const int rr = row < P.M ? row : P.M - 1;
  if (EPI == TE_CE_DS || EPI == TE_CE_STATS) r.t = e.targets[e.row_offset + rr];
  if (EPI == TE_CE_DS) {
    r.lse = e.lse[e.row_offset + rr];
    r.s = e.sc->inv_M;
  }
  return r;
}

// 32 bf16 of the auxiliary input (residual stream, or gelu' stored by the forward) of one row, packed;
// zeros past M or N.
__device__ __forceinline__ void load_aux_chunk(const TcParams &P, int row, int col0, int bz,
                                               uint4 (&a)[4]) {
  const Epi &e = P.epi;
  const bf16 *src = (const bf16 *)e.aux + (long)bz * e.aux_bstride + (long)row * e.ld_aux + col0;
  if (row < P.M && col0 + 32 <= P.N) {
#pragma unroll
    for (int q = 0; q < 4; ++q) a[q] = reinterpret_cast<const uint4 *>(src)[q];
  } else {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t lo = (row < P.M && col0 + 2 * i < P.N) ? __bfloat16_as_ushort(src[2 * i]) : 0u;
      const uint32_t hi = (row < P.M && col0 + 2 * i + 1 < P.N) ? __bfloat16_as_ushort(src[2 * i + 1]) : 0u;
      w[i] = lo | (hi << 16);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) a[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}
__device__ __forceinline__ void unpack_bf16x32(const uint4 (&a)[4], float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w[4] = {a[q].x, a[q].y, a[q].z, a[q].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
}

// Cross-entropy statistics of one 32-column chunk of a row: the running (max, sum of
// exp(logit - max)) over the valid vocabulary columns, and the target logit when the chunk
// holds it.
__device__ __forceinline__ void ce_stats_chunk(const TcParams &P, int row, int col0, const EpiRow &er,
                                               const float (&v)[32], float &ce_max, float &ce_sum) {
  const Epi &e = P.epi;
  const int lim = min(P.N, e.V) - col0;  // valid columns in this chunk
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (i < lim) mx = fmaxf(mx, v[i]);
  const float mnew = fmaxf(ce_max, mx);
  if (mnew > -INFINITY) {
    const float m2 = mnew * LOG2E_F;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      if (i < lim) s0 += ex2(fmaf(v[i], LOG2E_F, -m2));
      if (i + 1 < lim) s1 += ex2(fmaf(v[i + 1], LOG2E_F, -m2));
    }
    ce_sum = ce_sum * ex2(fmaf(ce_max, LOG2E_F, -m2)) + (s0 + s1);
    ce_max = mnew;
  }
  const int t = er.t - col0;
  if (t >= 0 && t < 32 && t < lim) {
    float tv = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) tv = (i == t) ? v[i] : tv;
    e.tgt_logit[e.row_offset + row] = tv;
  }
}

// ---------------------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------------------
// CG = 1: one CTA per 128x256 tile. CG = 2: a cluster of two CTAs per 256x256 tile; each CTA
// TMA-loads its own 128 rows of A and 128 rows (N) of B into its own shared memory, the
// leader (cluster rank 0) issues tcgen05.mma.cta_group::2, which reads both CTAs' stages and
// writes rows 0-127 to the leader's TMEM and rows 128-255 to the peer's. Both CTAs' TMA
// loads complete on the leader's stage barrier; the leader's commits arrive on both CTAs'
// barriers (commit multicast); the peer's epilogue releases the accumulator with a remote
// arrive on the leader's barrier. No TMA load uses cluster multicast.
template <int CG>
struct TcCfg {
  static constexpr int B_ROWS = BN / CG;                 // rows of B each CTA loads
  static constexpr int B_CTA_BYTES = B_ROWS * BK * 2;    // 64 KB / 32 KB
  static constexpr int B_CHUNK = B_ROWS * 64 * 2;        // one 64-element chunk of B
  static constexpr int STAGE = A_BYTES + B_CTA_BYTES;    // 96 KB / 64 KB
  // 192 KB of stages in flight, 4 KB of epilogue staging per warp (two bf16 chunk slots, or
  // one for two outputs / fp32). A stage's operands arrive in one 32 KB TMA load each: a
  // producer thread's loads complete at a rate set per load more than per byte, so 128-wide
  // K stages (one load per operand) feed the MMAs faster than 64-wide ones (one 16 KB load
  // per operand).
  static constexpr int NSTAGE = CG == 1 ? 2 : 3;
  static constexpr int WARP_STAGE = 4096;  // epilogue staging per warp
  static constexpr int SMEM = NSTAGE * STAGE + EPI_WARPS * WARP_STAGE + 1024 + 256;
  static_assert(SMEM <= 232448, "GEMM shared memory");
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t nclusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// Relaxed: it only tells the MMA issuer that this warp's accumulator reads are done, and those
// have completed (tcgen05.wait::ld) before the tcgen05 fence that precedes it; a release would
// also wait for this thread's earlier writes, which nothing on the other side reads.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx_addr(uint32_t addr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(addr), "r"(bytes)
               : "memory");
}
// TMA tile load whose completion is counted on mbarrier `mbar_cluster` (a shared::cluster
// address, possibly in the peer CTA of the pair).
template <int CG>
__device__ __forceinline__ void tma_load_pair(void *dst, const CUtensorMap *map,
                                              uint32_t mbar_cluster, int c0, int c1, int c2) {
  if (CG == 2)
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(mbar_cluster), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
  else
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(mbar_cluster), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}
// The same with a 4D map (an operand whose contiguous dimension is viewed as 64-element chunks).
template <int CG>
__device__ __forceinline__ void tma_load_pair4(void *dst, const CUtensorMap *map,
                                               uint32_t mbar_cluster, int c0, int c1, int c2,
                                               int c3) {
  if (CG == 2)
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(mbar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
  else
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"((uint64_t)map), "r"(mbar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
template <int CG>
__device__ __forceinline__ void umma_issue(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  if (CG == 2)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    umma_bf16(d_tmem, adesc, bdesc, idesc, accumulate);
}
// Arrive on `bar` (same offset) in every CTA of the pair once all prior MMAs complete.
template <int CG>
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
  if (CG == 2)
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"((uint16_t)3)
        : "memory");
  else
    umma_commit(bar);
}

// Epilogue math for one 32-column chunk of one row (everything but the store): v holds the
// fp32 accumulators on entry and the values to store on exit; v2 the second output (GELU);
// aux the chunk's auxiliary input (residual / dGELU).
template <int EPI>
__device__ __forceinline__ void epi_math(const TcParams &P, int col0, const EpiRow &er,
                                         const uint4 (&aux)[4], float (&v)[32], float (&v2)[32]) {
  if (EPI == TE_CE_DS) {
    // dS = (softmax - onehot(target)) / n over the valid vocabulary columns, 0 past V
    const int V = P.epi.V;
    const float L2 = er.lse * LOG2E_F;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int c = col0 + i;
      float p = ex2(fmaf(v[i], LOG2E_F, -L2));
      p = (c == er.t) ? p - 1.f : p;
      v[i] = c < V ? p * er.s : 0.f;
    }
  } else if (EPI == TE_RESID || EPI == TE_DGELU) {
    // residual: aux + acc; dGELU: acc * gelu'(pre), the derivative stored by the forward
    float a[32];
    unpack_bf16x32(aux, a);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = EPI == TE_RESID ? a[i] + v[i] : v[i] * a[i];
  } else if (EPI == TE_AXPBY) {
    float a[32];
    unpack_bf16x32(aux, a);
    const float al = P.epi.alpha, be = P.epi.beta;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = fmaf(al, v[i], be * a[i]);
  } else if (EPI == TE_STORE_GELU) {
    // out = gelu'(acc) (kept for the backward instead of the pre-activation), out2 = gelu(acc)
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float g;
      v2[i] = gelu_and_grad_fast(v[i], g);
      v[i] = g;
    }
  } else if (EPI == TE_STORE_PRE_GELU) {
    // out = bf16(acc) (the pre-activation, kept for the backward), out2 = gelu of that same
    // bf16 value, so that the backward's recomputed activation is bitwise the forward's
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      v[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
      v2[i] = gelu_fast(v[i]);
    }
  } else if (EPI == TE_DGELU_RECOMP) {
    // out = acc * gelu'(pre), out2 = gelu(pre): both from the kept pre-activation
    float a[32];
    unpack_bf16x32(aux, a);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float g;
      v2[i] = gelu_and_grad_fast(a[i], g);
      v[i] *= g;
    }
  }
}

// Writes row `r` (this lane) of a 32x32 chunk into a staging slot laid out for a TMA store:
// bf16 rows of 64 bytes with the 64-byte swizzle, fp32 rows of 128 bytes with the 128-byte one.
__device__ __forceinline__ void stage_bf16_row(uint8_t *slot, int r, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 u = make_uint4(pack_bf16(v[8 * c], v[8 * c + 1]), pack_bf16(v[8 * c + 2], v[8 * c + 3]),
                         pack_bf16(v[8 * c + 4], v[8 * c + 5]), pack_bf16(v[8 * c + 6], v[8 * c + 7]));
    *reinterpret_cast<uint4 *>(slot + r * 64 + ((c ^ ((r >> 1) & 3)) << 4)) = u;
  }
}
__device__ __forceinline__ void stage_f32_row(uint8_t *slot, int r, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<float4 *>(slot + r * 128 + ((c ^ (r & 7)) << 4)) =
        make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}

template <int EPI, int CG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
               const TcParams P) {
  using Cf = TcCfg<CG>;
  constexpr int NS = Cf::NSTAGE;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *epi_stage = smem + NS * Cf::STAGE;  // EPI_WARPS x WARP_STAGE bytes
  uint64_t *full_bar = (uint64_t *)(epi_stage + EPI_WARPS * Cf::WARP_STAGE);
  uint64_t *empty_bar = full_bar + NS;
  uint64_t *tfull_bar = empty_bar + NS;
  uint64_t *tempty_bar = tfull_bar + 2;
  uint32_t *tmem_holder = (uint32_t *)(tempty_bar + 2);
  volatile int *abort_flag = (volatile int *)(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const int unit0 = CG == 2 ? (int)cluster_id_x() : (int)blockIdx.x;
  const int ustride = CG == 2 ? (int)nclusters_x() : (int)gridDim.x;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], EPI_WARPS * CG);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    if (CG == 2) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_holder)),
                   "r"(TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      tmem_alloc(tmem_holder, TMEM_COLS);
    }
  }
  tc_fence_before();
  if (CG == 2) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------ TMA producer (each CTA) ------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t issued = 0, last_par = 0;
      for (int u = unit0; u < P.units && ok; u += ustride) {
        int mt, nt, z, bz;
        unit_coords(P, u, mt, nt, z, bz);
        const int m0 = mt * BM * CG + (int)rank * BM;
        const int n0 = nt * BN + (int)rank * Cf::B_ROWS;
        const int kb0 = z * P.kblocks_per_split;
        const int kb1 = min(P.total_kblocks, kb0 + P.kblocks_per_split);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, P.err)) { ok = false; break; }
          uint8_t *sA = smem + stage * Cf::STAGE;
          uint8_t *sB = sA + A_BYTES;
          const uint32_t fb = smem_u32(&full_bar[stage]);
          const uint32_t fbl = CG == 2 ? mapa_shared(fb, 0) : fb;  // the leader's barrier
          if (rank == 0) mbar_expect_tx_addr(fb, Cf::STAGE * CG);
          // smem layout of an operand tile: its 64-element chunks one after the other, each
          // 128-byte swizzled (K-major: [k chunk][row][64 k]; MN-major: [mn chunk][k][64 mn])
          const int k0 = kb * BK;
          if (P.a_wide) {
            if (!P.a_mn) tma_load_pair4<CG>(sA, &tmA, fbl, 0, m0, k0 / 64, bz);
            else tma_load_pair4<CG>(sA, &tmA, fbl, 0, k0, m0 / 64, bz);
          } else if (!P.a_mn) {
#pragma unroll
            for (int j = 0; j < KC; ++j)
              tma_load_pair<CG>(sA + j * A_CHUNK, &tmA, fbl, k0 + 64 * j, m0, bz);
          } else {
#pragma unroll
            for (int j = 0; j < BM / 64; ++j)  // MN-major chunks: 64 m by BK k rows of 128 B
              tma_load_pair<CG>(sA + j * (BK * 128), &tmA, fbl, m0 + 64 * j, k0, bz);
          }
          if (P.b_wide) {
            if (!P.b_mn) tma_load_pair4<CG>(sB, &tmB, fbl, 0, n0, k0 / 64, bz);
            else tma_load_pair4<CG>(sB, &tmB, fbl, 0, k0, n0 / 64, bz);
          } else if (!P.b_mn) {
#pragma unroll
            for (int j = 0; j < KC; ++j)
              tma_load_pair<CG>(sB + j * Cf::B_CHUNK, &tmB, fbl, k0 + 64 * j, n0, bz);
          } else {
#pragma unroll
            for (int j = 0; j < Cf::B_ROWS / 64; ++j)
              tma_load_pair<CG>(sB + j * (BK * 128), &tmB, fbl, n0 + 64 * j, k0, bz);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == NS) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag && rank == 0) {
        // leave no bulk copy in flight: wait (bounded) for the last fill of every stage
        const uint64_t t0 = globaltimer();
        for (int s2 = 0; s2 < NS; ++s2) {
          if (!(issued >> s2 & 1u)) continue;
          while (!mbar_try_wait(&full_bar[s2], (last_par >> s2) & 1u) &&
                 globaltimer() - t0 < 200000000ull) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------ MMA issuer (leader CTA) ------------------------------
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int i = 0;
      // byte offset of MMA k-step k (16 k) in an operand tile: K-major, chunk k / 4 and 32 B
      // per step inside it; MN-major, 16 k rows of 128 B per step. MN-major chunks (64 m or n)
      // are BK rows of 128 B apart (the descriptor's leading byte offset).
      const uint32_t a_lbo = P.a_mn ? (uint32_t)(BK * 128) : 16u;
      const uint32_t b_lbo = P.b_mn ? (uint32_t)(BK * 128) : 16u;
      for (int u = unit0; u < P.units && ok; u += ustride, ++i) {
        const int z = (u / (P.num_mt * P.num_nt)) % P.splits;
        const int kb0 = z * P.kblocks_per_split;
        const int kb1 = min(P.total_kblocks, kb0 + P.kblocks_per_split);
        const int acc = i & 1;
        const uint32_t use = (uint32_t)(i >> 1);
        if (!mbar_wait(&tempty_bar[acc], (use & 1u) ^ 1u, abort_flag, P.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, abort_flag, P.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sA = smem_u32(smem + stage * Cf::STAGE);
          const uint64_t ad0 = sdesc(sA, a_lbo, 1024u), bd0 = sdesc(sA + A_BYTES, b_lbo, 1024u);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t ao = P.a_mn ? (uint32_t)k * 2048u
                                       : (uint32_t)(k >> 2) * A_CHUNK + (uint32_t)(k & 3) * 32u;
            const uint32_t bo = P.b_mn ? (uint32_t)k * 2048u
                                       : (uint32_t)(k >> 2) * Cf::B_CHUNK + (uint32_t)(k & 3) * 32u;
            umma_issue<CG>(d_tmem, ad0 + (uint64_t)(ao >> 4), bd0 + (uint64_t)(bo >> 4), P.idesc,
                           (kb > kb0 || k > 0) ? 1u : 0u);
          }
          umma_commit_pair<CG>(&empty_bar[stage]);
          if (++stage == NS) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair<CG>(&tfull_bar[acc]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------ epilogue (each CTA) ------------------------------
    // 8 warps: warp w reads TMEM lane quarter (w % 4) and columns [half*128, half*128+128)
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int OUT_BYTES = (EPI == TE_F32_STORE || EPI == TE_F32_ACCUM || EPI == TE_PARTIAL) ? 4 : 2;
    constexpr int SLOT_BYTES = 32 * 32 * OUT_BYTES;
    constexpr int NOUT = (EPI == TE_STORE_GELU || EPI == TE_STORE_PRE_GELU || EPI == TE_DGELU_RECOMP) ? 2 : 1;
    constexpr int CHUNK_SLOTS = Cf::WARP_STAGE / (SLOT_BYTES * NOUT) >= 4 ? 4
                              : Cf::WARP_STAGE / (SLOT_BYTES * NOUT);
    static_assert(CHUNK_SLOTS >= 1, "epilogue staging too small");
    uint8_t *wstage = epi_stage + (warp - 2) * Cf::WARP_STAGE;
    int chunk_seq = 0;
    int i = 0;
    for (int u = unit0; u < P.units; u += ustride, ++i) {
      int mt, nt, z, bz;
      unit_coords(P, u, mt, nt, z, bz);
      const int acc = i & 1;
      const uint32_t use = (uint32_t)(i >> 1);
      const int row0 = mt * BM * CG + (int)rank * BM + q * 32;  // this warp's 32 rows
      const int row = row0 + lane;
      const int c0 = half * EPI_COLS;
      // operands that do not depend on the accumulators: loaded before the wait
      const EpiRow er = epi_row<EPI>(P, row);
      uint4 aux[4];
      if (epi_has_aux(EPI) && c0 < min(BN, P.N - nt * BN))
        load_aux_chunk(P, row, nt * BN + c0, bz, aux);
      int okw = 1;
      if (lane == 0) okw = mbar_wait(&tfull_bar[acc], use & 1u, abort_flag, P.err) ? 1 : 0;
      okw = __shfl_sync(0xffffffffu, okw, 0);
      if (!okw) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + c0);
      float ce_max = -INFINITY, ce_sum = 0.f;
      float dot_part = 0.f;  // TE_STORE_DOT: the first half of a head's dot
      const int ncols = min(BN, P.N - nt * BN) - c0;
      // the accumulator load of chunk c + 1 (and its auxiliary input) is in flight during
      // chunk c's math and store
      uint32_t raw[32];
      if (ncols > 0) tmem_ld32_nw(tbase, raw);
#pragma unroll
      for (int c = 0; c < EPI_COLS / 32; ++c) {
        if (c * 32 >= ncols) break;  // uniform across the warp
        const int col0 = nt * BN + c0 + c * 32;
        const bool more = (c + 1) * 32 < ncols && c + 1 < EPI_COLS / 32;
        tmem_wait_ld32(raw);
        float v[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(raw[k]);
        if (more) tmem_ld32_nw(tbase + (uint32_t)((c + 1) * 32), raw);
        uint4 aux_nx[4];
        if (epi_has_aux(EPI) && more) load_aux_chunk(P, row, col0 + 32, bz, aux_nx);
        if (EPI == TE_CE_STATS) {
          if (row < P.M) ce_stats_chunk(P, row, col0, er, v, ce_max, ce_sum);
          continue;
        }
        float v2[32];
        epi_math<EPI>(P, col0, er, aux, v, v2);
        if (EPI == TE_STORE_DOT) {
          // the head's dot of the stored (bf16) dO row with O, over its two 32-column chunks
          float a[32];
          unpack_bf16x32(aux, a);
          float sdot = 0.f;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            sdot = fmaf(__bfloat162float(__float2bfloat16_rn(v[k])), a[k], sdot);
          if ((col0 & 63) == 0) {
            dot_part = sdot;
          } else if (row < P.M) {
            const int b = row / P.epi.dot_T, t = row - b * P.epi.dot_T;
            P.epi.outf[((long)b * (P.N / 64) + col0 / 64) * P.epi.dot_T + t] = dot_part + sdot;
          }
        }
        if (epi_has_aux(EPI)) {
#pragma unroll
          for (int q = 0; q < 4; ++q) aux[q] = aux_nx[q];
        }
        // staging slot of this chunk (round robin); wait until its previous store has read it
        if (lane == 0) {
          if (CHUNK_SLOTS == 1) bulk_wait_read<0>();
          else if (CHUNK_SLOTS == 2) bulk_wait_read<1>();
          else bulk_wait_read<3>();
        }
        __syncwarp();
        uint8_t *slot = wstage + (chunk_seq % CHUNK_SLOTS) * SLOT_BYTES * NOUT;
        if (OUT_BYTES == 4) stage_f32_row(slot, lane, v);
        else stage_bf16_row(slot, lane, v);
        if (NOUT == 2) stage_bf16_row(slot + SLOT_BYTES, lane, v2);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (EPI == TE_PARTIAL) tma_store_3d(&tmO, slot, col0, row0, z);
          else if (EPI == TE_F32_ACCUM) tma_reduce_add_3d(&tmO, slot, col0, row0, bz);
          else tma_store_3d(&tmO, slot, col0, row0, bz);
          if (NOUT == 2) tma_store_3d(&tmO2, slot + SLOT_BYTES, col0, row0, bz);
          bulk_commit();
        }
        ++chunk_seq;
      }
      if (EPI == TE_CE_STATS && row < P.M && ncols > 0) {
        const Epi &e = P.epi;
        float *st = e.stats + ((long)(e.row_offset + row) * e.ntiles + nt * 2 + half) * 2;
        st[0] = ce_max;
        st[1] = ce_sum;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty_bar[acc]), 0));
        else mbar_arrive(&tempty_bar[acc]);
      }
    }
    if (lane == 0) bulk_wait_all();  // every TMA store of this warp has completed
    __syncwarp();
  }
  tc_fence_before();
  if (CG == 2) cluster_sync_all(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (CG == 2)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(TMEM_COLS)
                   : "memory");
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------
int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// 2-D bf16 tensor map: inner dimension `inner` (contiguous), outer `outer`, row stride `ld`
// elements, box {64, box_outer}, 128-byte swizzle.
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up at run time so the library loads without libcuda.
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

// Output tensor map for the TMA-store epilogue: [depth][rows][cols] with row stride `ld` and
// `plane` elements between planes (the products of a batched GEMM, or the split-K partials),
// box 32 x 32 x 1, bf16 with the 64-byte swizzle or fp32 with the 128-byte one.
bool make_out_map(CUtensorMap *m, const void *base, bool f32, long cols, long rows, long ld,
                  long depth = 1, long plane = 0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int es = f32 ? 4 : 2;
  if (depth <= 1) { depth = 1; plane = ld * rows; }
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)depth};
  cuuint64_t strides[2] = {(cuuint64_t)ld * es, (cuuint64_t)plane * es};
  cuuint32_t box[3] = {32u, 32u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
             (void *)base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Operand map: bf16 [batch][outer][inner] (inner contiguous, row stride ld, `bstride`
// elements between batches), box {64, box_outer, 1}, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *base, long inner, long outer, long ld, int box_outer,
              long batch = 1, long bstride = 0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  if (batch <= 1) { batch = 1; bstride = ld * outer; }
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)outer, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)ld * 2, (cuuint64_t)bstride * 2};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_outer, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void *)base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The same operand viewed as [batch][inner / 64][outer][64] (inner % 64 == 0): box
// {64, box_outer, box_chunks, 1} brings box_chunks 64-element chunks of box_outer rows,
// one chunk after the other in shared memory.
bool make_map_chunked(CUtensorMap *m, const void *base, long inner, long outer, long ld,
                      int box_outer, int box_chunks, long batch = 1, long bstride = 0) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || inner % 64 != 0) return false;
  if (batch <= 1) { batch = 1; bstride = ld * outer; }
  cuuint64_t dims[4] = {64u, (cuuint64_t)outer, (cuuint64_t)(inner / 64), (cuuint64_t)batch};
  cuuint64_t strides[3] = {(cuuint64_t)ld * 2, 128u, (cuuint64_t)bstride * 2};
  cuuint32_t box[4] = {64u, (cuuint32_t)box_outer, (cuuint32_t)box_chunks, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, (void *)base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int EPI, int CG>
cudaError_t launch_kind(const CUtensorMap &a, const CUtensorMap &b, const CUtensorMap &o,
                        const CUtensorMap &o2, const TcParams &P, int grid, cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel<EPI, CG>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         TcCfg<CG>::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = TcCfg<CG>::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CG;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_gemm_kernel<EPI, CG>, a, b, o, o2, P);
}

template <int CG>
cudaError_t launch_epi(int kind, bool split, const CUtensorMap &ma, const CUtensorMap &mb,
                       const CUtensorMap &mo, const CUtensorMap &mo2, const TcParams &P, int grid,
                       cudaStream_t st) {
#define TC_L(K) launch_kind<K, CG>(ma, mb, mo, mo2, P, grid, st)
  if (split) return TC_L(TE_PARTIAL);
  switch (kind) {
    case EPI_STORE: return TC_L(TE_STORE);
    case EPI_STORE_GELU: return TC_L(TE_STORE_GELU);
    case EPI_RESID: return TC_L(TE_RESID);
    case EPI_DGELU: return TC_L(TE_DGELU);
    case EPI_F32_STORE: return TC_L(TE_F32_STORE);
    case EPI_F32_ACCUM: return TC_L(TE_F32_ACCUM);
    case EPI_CE_STATS: return TC_L(TE_CE_STATS);
    case EPI_CE_DS: return TC_L(TE_CE_DS);
    case EPI_STORE_PRE_GELU: return TC_L(TE_STORE_PRE_GELU);
    case EPI_DGELU_RECOMP: return TC_L(TE_DGELU_RECOMP);
    case EPI_AXPBY: return TC_L(TE_AXPBY);
    case EPI_STORE_DOT: return TC_L(TE_STORE_DOT);
    default: return cudaErrorInvalidValue;
  }
#undef TC_L
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

struct TcGemm {
  unsigned *err;
  size_t splitk_capacity;  // floats available at GemmDesc::partial
};

cudaError_t tc_gemm_create(TcGemm **out) {
  *out = new TcGemm();
  (*out)->err = nullptr;
  (*out)->splitk_capacity = 0;
  return cudaSuccess;
}
void tc_gemm_set_splitk_capacity(TcGemm *t, size_t floats) { t->splitk_capacity = floats; }
void tc_gemm_destroy(TcGemm *t) { delete t; }

bool tc_gemm_supported(const GemmDesc &d) {
  if (d.K <= 0 || d.M <= 0 || d.N <= 0) return false;
  if ((d.lda & 7) || (d.ldb & 7)) return false;
  if (!aligned16(d.A) || !aligned16(d.B)) return false;
  const Epi &e = d.epi;
  if (d.batch > 1) {  // batched products: bf16 outputs, 16-byte batch strides, no K split
    if (e.kind != EPI_STORE && e.kind != EPI_AXPBY) return false;
    if ((d.a_bstride & 7) || (d.b_bstride & 7) || (d.out_bstride & 7) || d.split_k > 1) return false;
  }
  switch (e.kind) {
    case EPI_STORE:
    case EPI_CE_DS:
      return (e.ldo & 7) == 0 && aligned16(e.out);
    case EPI_STORE_GELU:
    case EPI_STORE_PRE_GELU:
      return (e.ldo & 7) == 0 && (e.ldo2 & 7) == 0 && aligned16(e.out) && aligned16(e.out2);
    case EPI_DGELU_RECOMP:
      return (e.ldo & 7) == 0 && (e.ldo2 & 7) == 0 && (e.ld_aux & 7) == 0 && aligned16(e.out) &&
             aligned16(e.out2) && aligned16(e.aux);
    case EPI_RESID:
    case EPI_DGELU:
    case EPI_AXPBY:
      return (e.ldo & 7) == 0 && (e.ld_aux & 7) == 0 && (e.aux_bstride & 7) == 0 &&
             aligned16(e.out) && aligned16(e.aux);
    case EPI_STORE_DOT:  // whole 64-column heads, one sequence length for the rows
      return (e.ldo & 7) == 0 && (e.ld_aux & 7) == 0 && aligned16(e.out) && aligned16(e.aux) &&
             e.outf && e.dot_T > 0 && d.M % e.dot_T == 0 && d.N % 64 == 0 && d.split_k == 1;
    case EPI_F32_STORE:
    case EPI_F32_ACCUM:
      return (e.ldf & 3) == 0 && aligned16(e.outf);
    case EPI_CE_STATS:
      return true;
    default:
      return false;
  }
}

// The CTA group (1 or 2) and K split the launcher uses for `d` with `capacity` floats of
// partial-sum scratch on `sms` SMs (host only; split_k > 0 in d is taken as given).
void tc_gemm_plan(const GemmDesc &d, size_t capacity, int sms, int *cta_group, int *split) {
  const int nt = (d.N + BN - 1) / BN;
  const long kblocks = (d.K + BK - 1) / BK;
  const bool f32out = d.epi.kind == EPI_F32_STORE || d.epi.kind == EPI_F32_ACCUM;
  const bool elementwise = d.epi.kind != EPI_CE_STATS && d.epi.kind != EPI_CE_DS;
  const long nbatch = d.batch > 1 ? d.batch : 1;
  int CG = ((long)((d.M + 2 * BM - 1) / (2 * BM)) * nt * nbatch >= sms / 2) ? 2 : 1;
  int S = d.split_k;
  if (nbatch > 1) S = 1;  // batched products are not split
  if (S <= 0) {
    S = 1;
    if ((f32out || elementwise) && capacity > 0) {
      // automatic: the CTA group and K split with the smallest estimated time, in units of
      // one 128-wide k-block of one CTA tile (~0.8 us): the wave-quantised main loop, CTA
      // pairs credited with their smaller shared-memory traffic, plus for a split the ordered
      // reduce, which reads the s fp32 partials and writes the result (~6 TB/s), and its
      // launch (the partial stores themselves overlap the main loop)
      double best = 1e30;
      for (int cg = 1; cg <= 2; ++cg) {
        const long tiles = (long)((d.M + cg * BM - 1) / (cg * BM)) * nt * nbatch;
        const long slots = sms / cg;
        for (int s = 1; s <= 16; ++s) {
          if (s > 1 && (kblocks / s < 2 || (size_t)s * d.M * d.N > capacity)) break;
          const long units = tiles * s;
          const long waves = (units + slots - 1) / slots;
          double est = (double)waves * (double)((kblocks + s - 1) / s) * (cg == 2 ? 0.93 : 1.0);
          if (s > 1) est += ((s + 1.0) * d.M * d.N * 4.0 / 6.0e12 + 3e-6) / 0.8e-6;
          if (est < best) { best = est; CG = cg; S = s; }
        }
      }
    }
  }
  if (S > kblocks) S = (int)kblocks;
  if (S < 1) S = 1;
  if (kblocks > 0) {
    const long per = (kblocks + S - 1) / S;
    S = (int)((kblocks + per - 1) / per);  // no empty split
  }
  *cta_group = CG;
  *split = S;
}

cudaError_t tc_gemm_launch(TcGemm *t, GemmDesc &d, cudaStream_t st, int *launches) {
  (void)launches;
  TcParams P;
  memset(&P, 0, sizeof(P));
  const int sms = num_sms();
  const int nt = (d.N + BN - 1) / BN;
  const long kblocks = (d.K + BK - 1) / BK;
  int CG, S;
  tc_gemm_plan(d, d.partial ? t->splitk_capacity : 0, sms, &CG, &S);
  P.M = d.M; P.N = d.N; P.K = d.K;
  P.num_mt = (d.M + BM * CG - 1) / (BM * CG);
  P.num_nt = nt;
  P.total_kblocks = (int)kblocks;
  P.kblocks_per_split = (P.total_kblocks + S - 1) / S;
  if (S > 1 && (!d.partial || (size_t)S * d.M * d.N > t->splitk_capacity)) return cudaErrorInvalidValue;
  d.split_k = S;
  P.splits = S;
  P.batch = d.batch > 1 ? d.batch : 1;
  if (P.batch > 1 && S > 1) return cudaErrorInvalidValue;
  P.units = P.num_mt * P.num_nt * S * P.batch;
  {
    const double a_bytes = 2.0 * d.M * d.K, b_bytes = 2.0 * d.N * d.K;
    P.n_fast = (P.num_nt > 1 && a_bytes > b_bytes && a_bytes > 48e6) ? 1 : 0;
  }
  P.a_mn = d.a_kmajor ? 0 : 1;
  P.b_mn = d.b_kmajor ? 0 : 1;
  P.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)P.a_mn << 15) |
            ((uint32_t)P.b_mn << 16) | ((uint32_t)(BN >> 3) << 17) |
            ((uint32_t)((BM * CG) >> 4) << 24);
  P.epi = d.epi;
  P.partial = d.partial;
  P.err = d.err ? d.err : (d.epi.sc ? (unsigned *)&d.epi.sc->err : t->err);
  if (!P.err) return cudaErrorInvalidValue;
  CUtensorMap ma, mb;
  const int b_rows = BN / CG;
  // one load per operand and stage when the contiguous dimension is whole 64-element chunks
  // (a chunk past the end is then out of bounds and zero-filled, never part of the next row)
  P.a_wide = ((P.a_mn ? d.M : d.K) % 64 == 0) ? 1 : 0;
  P.b_wide = ((P.b_mn ? d.N : d.K) % 64 == 0) ? 1 : 0;
  bool ok;
  if (P.a_wide)
    ok = P.a_mn ? make_map_chunked(&ma, d.A, d.M, d.K, d.lda, BK, BM / 64, P.batch, d.a_bstride)
                : make_map_chunked(&ma, d.A, d.K, d.M, d.lda, BM, KC, P.batch, d.a_bstride);
  else
    ok = P.a_mn ? make_map(&ma, d.A, d.M, d.K, d.lda, BK, P.batch, d.a_bstride)
                : make_map(&ma, d.A, d.K, d.M, d.lda, BM, P.batch, d.a_bstride);
  if (P.b_wide)
    ok = ok && (P.b_mn ? make_map_chunked(&mb, d.B, d.N, d.K, d.ldb, BK, b_rows / 64, P.batch,
                                          d.b_bstride)
                       : make_map_chunked(&mb, d.B, d.K, d.N, d.ldb, b_rows, KC, P.batch,
                                          d.b_bstride));
  else
    ok = ok && (P.b_mn ? make_map(&mb, d.B, d.N, d.K, d.ldb, BK, P.batch, d.b_bstride)
                       : make_map(&mb, d.B, d.K, d.N, d.ldb, b_rows, P.batch, d.b_bstride));
  if (!ok) return cudaErrorInvalidValue;
  // output maps of the TMA-store epilogue (rows and columns past M, N are clipped by TMA)
  CUtensorMap mo, mo2;
  memset(&mo, 0, sizeof(mo));
  memset(&mo2, 0, sizeof(mo2));
  const Epi &e0 = d.epi;
  if (S > 1) {
    ok = make_out_map(&mo, d.partial, true, d.N, d.M, d.N, S, (long)d.M * d.N);
  } else {
    switch (e0.kind) {
      case EPI_STORE: case EPI_RESID: case EPI_DGELU: case EPI_CE_DS: case EPI_AXPBY:
      case EPI_STORE_DOT:
        ok = make_out_map(&mo, e0.out, false, d.N, d.M, e0.ldo, P.batch, d.out_bstride);
        break;
      case EPI_STORE_GELU: case EPI_STORE_PRE_GELU: case EPI_DGELU_RECOMP:
        ok = make_out_map(&mo, e0.out, false, d.N, d.M, e0.ldo) &&
             make_out_map(&mo2, e0.out2, false, d.N, d.M, e0.ldo2);
        break;
      case EPI_F32_STORE: case EPI_F32_ACCUM:
        ok = make_out_map(&mo, e0.outf, true, d.N, d.M, e0.ldf);
        break;
      default:
        break;
    }
  }
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e;
  if (CG == 2) {
    const int clusters = P.units < sms / 2 ? P.units : sms / 2;
    e = launch_epi<2>(d.epi.kind, S > 1, ma, mb, mo, mo2, P, 2 * clusters, st);
  } else {
    const int grid = P.units < sms ? P.units : sms;
    e = launch_epi<1>(d.epi.kind, S > 1, ma, mb, mo, mo2, P, grid, st);
  }
  if (e != cudaSuccess) return e;
  if (S > 1) return launch_splitk_reduce<bf16>(d, st);
  return cudaSuccess;
}
