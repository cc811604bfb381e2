// C ABI and step schedule of the GPT-2 training-step library.
//
// One gpt_train_step enqueues, on the caller's stream: token staging, the embedding, n_layer
// forward blocks, final LayerNorm, lm_head cross-entropy statistics, the chunked lm_head
// backward, the block backward in reverse, the embedding backward, the global grad norm
// and AdamW. The whole sequence for one (B, T) and one set of buffers is captured once into
// a CUDA graph and replayed; lr / wd / clip / step live in device memory (nanochat
// architecture page, "AdamW Fused Step": hyper-parameters held as tensors so that a
// compiled step is reused when lr changes). The only host synchronisation is the read-back
// of the loss, the grad norm and the device error word at the end of the call.
// gpt_train_step_accum runs the same schedule once per micro-batch (one graph per phase:
// gradients stored, accumulated, accumulated + clip and AdamW).
#include <cuda.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <map>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/gpt_step.h"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "muon.cuh"

namespace {

constexpr int ALIGN = 256;
constexpr int SIMT_TILE_N = 64;

struct Layer {
  size_t ln1, wqkv, wap, ln2, wfc, wmp;
};

struct Acts {  // per-layer saved activations
  // dgelu = gelu'(pre-activation), or with GELU recompute the pre-activation itself; h =
  // gelu(pre-activation), one buffer shared by all layers with GELU recompute
  void *x_in, *a, *qkv, *o, *x_mid, *c, *dgelu, *h;
  float *lse, *mu1, *rs1, *mu2, *rs2;
};

// Phases of a training call: a whole step, or the first / a middle / the last micro-batch of
// a gradient-accumulated step (gradients stored, accumulated, accumulated + update).
enum StepPhase { PH_STEP = 0, PH_FIRST = 1, PH_MIDDLE = 2, PH_LAST = 3 };

struct GraphKey {
  int B, T, train, phase;
  const void *p, *g, *m, *v, *ptl;
  bool operator<(const GraphKey &o) const {
    return std::tie(B, T, train, phase, p, g, m, v, ptl) <
           std::tie(o.B, o.T, o.train, o.phase, o.p, o.g, o.m, o.v, o.ptl);
  }
};

}  // namespace

struct gpt_handle {
  gpt_config cfg;
  std::vector<int> windows;
  int C, H, hd, mC, V, Vp, L, maxT, maxB, maxM;
  bool use_bf16;
  size_t nparams;
  size_t off_wte, off_wpe, off_lnf;
  std::vector<Layer> layer;
  std::vector<gpt_tensor_desc> descs;
  int device;
  cudaStream_t stream;
  // workspace
  char *ws;
  size_t ws_bytes;
  DevScalars *sc;
  DevScalars *sc_host;  // pinned
  int *tok, *tgt;
  std::vector<Acts> acts;
  void *x_final, *yf;
  float *muf, *rsf;
  float *stats, *tgt_logit, *lse_ce, *per_token;
  int ce_tile_n, ce_ntiles;
  void *dS;
  long ldS;
  int chunk_rows;
  void *dx, *dh, *dc, *dqkv, *dout, *dyf;
  float *Dbuf, *dg_partial;
  bf16 *dst;  // attention backward: dS^T of one layer [B*H][T][T] (NULL: the two-pass backward)
  double *gn_partials;
  float *splitk;
  size_t splitk_elems;
  // The weight-gradient GEMMs of the backward run on a second stream beside the chain of
  // data-gradient kernels (they fill its GEMM wave tails and memory-bound stretches), with
  // their own split-K scratch; events order them against the buffers they share.
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_wmp, ev_wfc, ev_wap, ev_wqkv, ev_wte, ev_side_done, ev_cs[2];
  float *splitk2;
  float *dg_partial2;  // LayerNorm backward: the dgamma partials alternate between two buffers
  void *emb_ws;  // embedding backward: sort buffers, digit histogram, window partials
  bf16 *shadow;
  // state
  long step;
  float last_norm;
  const float *shadow_src;
  bool shadow_valid;
  bool use_graphs;
  struct Captured {
    cudaGraphExec_t exec;
    int launches;
  };
  std::map<GraphKey, Captured> graphs;
  int launches;
  std::string cuda_err;
  // kernel timing
  bool time_kernels;
  std::vector<cudaEvent_t> ev;
  std::vector<double> ev_work;  // algorithmic FLOPs or bytes of the launch
  std::vector<int> ev_kind;     // GPT_KSTAT_* class of the launch
  int ev_used;
  long long stat_launches[GPT_KSTAT_COUNT];
  double stat_ms[GPT_KSTAT_COUNT], stat_work[GPT_KSTAT_COUNT];
  TcGemm *tc;
  void *muon_ws;  // Muon scratch, allocated by the first gpt_muon_update
};

namespace {

size_t align_up(size_t x) { return (x + ALIGN - 1) / ALIGN * ALIGN; }

int fail(gpt_handle *h, cudaError_t e) {
  if (h) h->cuda_err = cudaGetErrorString(e);
  return e == cudaErrorMemoryAllocation ? GPT_ERR_OOM : GPT_ERR_CUDA;
}

#define TRY(x)                                  \
  do {                                          \
    cudaError_t e__ = (x);                      \
    if (e__ != cudaSuccess) return fail(h, e__); \
  } while (0)

bool misaligned(const void *p) { return ((uintptr_t)p & 15u) != 0; }

bool is_device_ptr(const void *p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

// --------------------------------------------------------------------------------------
// per-launch timing (GPT_OPT_TIME_KERNELS): CUDA events on the step's stream around a launch,
// with the launch's algorithmic work, accumulated per kernel class by finish()
// --------------------------------------------------------------------------------------
int tbegin(gpt_handle *h, int kind, double work) {
  if (!h->time_kernels || h->ev_used + 2 > (int)h->ev.size()) return -1;
  const int k = h->ev_used;
  h->ev_used += 2;
  h->ev_work[k / 2] = work;
  h->ev_kind[k / 2] = kind;
  return cudaEventRecord(h->ev[k], h->stream) == cudaSuccess ? k : -1;
}
cudaError_t tend(gpt_handle *h, int k) {
  return k >= 0 ? cudaEventRecord(h->ev[k + 1], h->stream) : cudaSuccess;
}
#define TIMED(h, kind, work, call)                 \
  do {                                             \
    const int tk__ = tbegin((h), (kind), (work));  \
    CUDA_TRY(call);                                \
    CUDA_TRY(tend((h), tk__));                     \
  } while (0)
// the same in a C-ABI function (returns a GPT_ERR_* status)
#define TIMED_S(h, kind, work, call)               \
  do {                                             \
    const int tk__ = tbegin((h), (kind), (work));  \
    TRY(call);                                     \
    TRY(tend((h), tk__));                          \
  } while (0)

// --------------------------------------------------------------------------------------
// GEMM dispatch
// --------------------------------------------------------------------------------------
int choose_split(const gpt_handle *h, int M, int N, int K, int tm, int tn) {
  long tiles = (long)((M + tm - 1) / tm) * ((N + tn - 1) / tn);
  int s = 1;
  while (tiles * s < 2 * 148 && K / (s * 2) >= 256) s *= 2;
  while (s > 1 && (size_t)s * M * N > h->splitk_elems) s /= 2;
  return s;
}

// on_side: launch on the weight-gradient stream (only when side_ok: not while timing kernels,
// which needs every launch on the main stream)
bool side_ok(const gpt_handle *h) { return h->side != nullptr && !h->time_kernels; }

cudaError_t gemm(gpt_handle *h, GemmDesc d, bool on_side = false) {
  if (d.M <= 0 || d.N <= 0) return cudaSuccess;
  on_side = on_side && side_ok(h);
  cudaStream_t gst = on_side ? h->side : h->stream;
  float *scratch = on_side ? h->splitk2 : h->splitk;
  d.epi.sc = h->sc;  // device error word and 1/M for every epilogue
  const double flops = 2.0 * d.M * d.N * d.K;
  const int k = tbegin(h, d.epi.kind == EPI_CE_DS ? GPT_KSTAT_GEMM_RECOMPUTE : GPT_KSTAT_GEMM,
                       flops);
  cudaError_t e;
  const bool f32out = d.epi.kind == EPI_F32_STORE || d.epi.kind == EPI_F32_ACCUM;
  const bool elementwise = d.epi.kind != EPI_CE_STATS && d.epi.kind != EPI_CE_DS;
  if (!h->use_bf16) {
    if (d.epi.kind == EPI_CE_STATS) {
      d.epi.tile_n = SIMT_TILE_N;
      d.epi.ntiles = (d.N + SIMT_TILE_N - 1) / SIMT_TILE_N;
      h->ce_ntiles = d.epi.ntiles;
    }
    if (d.split_k == 0) d.split_k = f32out ? choose_split(h, d.M, d.N, d.K, 64, 64) : 1;
    d.partial = scratch;
    e = launch_gemm_simt<float>(d, gst);
  } else if (h->tc && tc_gemm_supported(d)) {
    if (d.epi.kind == EPI_CE_STATS) {
      d.epi.tile_n = TC_CE_TILE;
      d.epi.ntiles = (d.N + TC_CE_TILE - 1) / TC_CE_TILE;
      h->ce_ntiles = d.epi.ntiles;
    }
    // the launcher picks the CTA group and, for elementwise epilogues, the K split
    d.partial = scratch;
    e = tc_gemm_launch(h->tc, d, gst, &h->launches);
  } else {
    if (d.epi.kind == EPI_CE_STATS) {
      d.epi.tile_n = SIMT_TILE_N;
      d.epi.ntiles = (d.N + SIMT_TILE_N - 1) / SIMT_TILE_N;
      h->ce_ntiles = d.epi.ntiles;
    }
    if (d.split_k == 0) d.split_k = f32out ? choose_split(h, d.M, d.N, d.K, 64, 64) : 1;
    d.partial = scratch;
    e = launch_gemm_simt<bf16>(d, gst);
  }
  h->launches += 1 + (d.split_k > 1 ? 1 : 0);
  if (e != cudaSuccess) return e;
  return tend(h, k);
}

GemmDesc gdesc(int M, int N, int K, const void *A, long lda, int ak, const void *B, long ldb,
               int bk) {
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.M = M; d.N = N; d.K = K;
  d.A = A; d.lda = lda; d.a_kmajor = ak;
  d.B = B; d.ldb = ldb; d.b_kmajor = bk;
  d.split_k = 0;
  return d;
}

// Attention: tensor-core kernels for bf16 with head_dim 64, CUDA-core kernels otherwise.
template <typename T>
cudaError_t attention_fwd(gpt_handle *h, const T *qkv, T *o, float *lse, int B, int Tlen, int w) {
  return launch_attention_fwd<T>(qkv, o, lse, B, Tlen, h->C, h->H, w, h->stream);
}
template <>
cudaError_t attention_fwd<bf16>(gpt_handle *h, const bf16 *qkv, bf16 *o, float *lse, int B,
                                int Tlen, int w) {
  if (attention_tc_supported(h->C, h->H))
    return launch_attention_fwd_tc(qkv, o, lse, B, Tlen, h->C, h->H, w, &h->sc->err, h->stream);
  return launch_attention_fwd<bf16>(qkv, o, lse, B, Tlen, h->C, h->H, w, h->stream);
}
// The dS^T scratch when the call's T gives it 16-byte rows (else the two-pass backward).
bf16 *attn_dst(const gpt_handle *h, int Tlen) { return (Tlen % 8 == 0) ? h->dst : nullptr; }

template <typename T>
cudaError_t attention_bwd(gpt_handle *h, const T *qkv, const T *o, const T *dout,
                          const float *lse, T *dqkv, int B, int Tlen, int w) {
  return launch_attention_bwd<T>(qkv, o, dout, lse, h->Dbuf, dqkv, B, Tlen, h->C, h->H, w,
                                 h->stream);
}
// The attention backward of the bf16 step takes D = rowsum(dO * O) from the epilogue of the
// GEMM that forms dO (EPI_STORE_DOT) when it runs the stored-dS form on the tensor cores.
bool fused_d(const gpt_handle *h, int Tlen) {
  return h->use_bf16 && h->tc && attention_tc_supported(h->C, h->H) && attn_dst(h, Tlen);
}
template <>
cudaError_t attention_bwd<bf16>(gpt_handle *h, const bf16 *qkv, const bf16 *o, const bf16 *dout,
                                const float *lse, bf16 *dqkv, int B, int Tlen, int w) {
  if (attention_tc_supported(h->C, h->H))
    return launch_attention_bwd_tc(qkv, o, dout, lse, h->Dbuf, dqkv, B, Tlen, h->C, h->H, w,
                                   &h->sc->err, h->stream, attn_dst(h, Tlen), fused_d(h, Tlen));
  return launch_attention_bwd<bf16>(qkv, o, dout, lse, h->Dbuf, dqkv, B, Tlen, h->C, h->H, w,
                                    h->stream);
}

// Admitted (query, key) pairs of one head's causal attention over T positions with left
// window w (w < 0: full causal): sum over queries of min(i, w) + 1.
double admitted_scores(long T, long w) {
  if (w < 0 || w >= T - 1) return (double)T * (T + 1) / 2.0;
  return (double)(w + 1) * T - (double)w * (w + 1) / 2.0;
}

// --------------------------------------------------------------------------------------
// the step schedule
// --------------------------------------------------------------------------------------
template <typename T>
cudaError_t enqueue(gpt_handle *h, const float *params, float *grads, float *adam_m,
                    float *adam_v, int B, int Tlen, bool train, float *per_token_out,
                    int phase) {
  cudaStream_t st = h->stream;
  const int C = h->C, H = h->H, mC = h->mC, V = h->V, M = B * Tlen;
  const T *W = h->use_bf16 ? (const T *)h->shadow : (const T *)params;
  DevScalars *sc = h->sc;
  int &nl = h->launches;

  // algorithmic work per launch (kernel timing): bytes of the memory-bound kernels, FLOPs
  // of the contractions (4 hd per admitted score forward, 8 hd backward; the backward's
  // recompute of the scores is not counted)
  const double es = h->use_bf16 ? 2.0 : 4.0;
  const double ln_fwd_bytes = (double)M * (2.0 * C * es + 8.0) + C * es;
  const double ln_bwd_bytes = (double)M * (4.0 * C * es + 8.0) + C * es + 4.0 * C;
  auto attn_flops = [&](int w, double per_score) {
    return per_score * h->hd * admitted_scores(Tlen, w) * B * H;
  };

  // ---------------- forward ----------------
  T *x0 = (T *)h->acts[0].x_in;
  TIMED(h, GPT_KSTAT_EMBED_FWD, (double)M * 3.0 * C * es + 8.0 * M,
        (launch_embed_fwd<T>(h->tok, h->tgt, W + h->off_wte, W + h->off_wpe, x0, M, Tlen, C, V,
                             sc, st))); nl++;
  for (int l = 0; l < h->L; ++l) {
    Acts &A = h->acts[l];
    const Layer &P = h->layer[l];
    T *xnext = (T *)(l + 1 < h->L ? h->acts[l + 1].x_in : h->x_final);
    TIMED(h, GPT_KSTAT_LN_FWD, ln_fwd_bytes,
          launch_layernorm_fwd<T>((T *)A.x_in, W + P.ln1, (T *)A.a, A.mu1, A.rs1, M, C,
                                  h->cfg.ln_eps, st)); nl++;
    GemmDesc d = gdesc(M, 3 * C, C, A.a, C, 1, W + P.wqkv, C, 1);
    d.epi.kind = EPI_STORE; d.epi.out = A.qkv; d.epi.ldo = 3 * C;
    CUDA_TRY(gemm(h, d));
    TIMED(h, GPT_KSTAT_ATTN_FWD, attn_flops(h->windows[l], 4.0),
          attention_fwd<T>(h, (T *)A.qkv, (T *)A.o, A.lse, B, Tlen, h->windows[l])); nl++;
    d = gdesc(M, C, C, A.o, C, 1, W + P.wap, C, 1);
    d.epi.kind = EPI_RESID; d.epi.out = A.x_mid; d.epi.ldo = C; d.epi.aux = A.x_in; d.epi.ld_aux = C;
    CUDA_TRY(gemm(h, d));
    TIMED(h, GPT_KSTAT_LN_FWD, ln_fwd_bytes,
          launch_layernorm_fwd<T>((T *)A.x_mid, W + P.ln2, (T *)A.c, A.mu2, A.rs2, M, C,
                                  h->cfg.ln_eps, st)); nl++;
    d = gdesc(M, mC, C, A.c, C, 1, W + P.wfc, C, 1);
    d.epi.kind = h->cfg.recompute_gelu ? EPI_STORE_PRE_GELU : EPI_STORE_GELU;
    d.epi.out = A.dgelu; d.epi.ldo = mC; d.epi.out2 = A.h; d.epi.ldo2 = mC;
    CUDA_TRY(gemm(h, d));
    d = gdesc(M, C, mC, A.h, mC, 1, W + P.wmp, mC, 1);
    d.epi.kind = EPI_RESID; d.epi.out = xnext; d.epi.ldo = C; d.epi.aux = A.x_mid; d.epi.ld_aux = C;
    CUDA_TRY(gemm(h, d));
  }
  TIMED(h, GPT_KSTAT_LN_FWD, ln_fwd_bytes,
        launch_layernorm_fwd<T>((T *)h->x_final, W + h->off_lnf, (T *)h->yf, h->muf, h->rsf, M, C,
                                h->cfg.ln_eps, st)); nl++;
  // lm_head statistics (the logits stay on chip)
  {
    GemmDesc d = gdesc(M, V, C, h->yf, C, 1, W + h->off_wte, C, 1);
    d.split_k = 1;
    Epi &e = d.epi;
    e.kind = EPI_CE_STATS; e.targets = h->tgt; e.stats = h->stats; e.tgt_logit = h->tgt_logit;
    e.V = V; e.row_offset = 0; e.sc = sc;
    CUDA_TRY(gemm(h, d));
    TIMED(h, GPT_KSTAT_CE, (double)M * (h->ce_ntiles * 8.0 + 16.0),
          launch_ce_combine(h->stats, h->tgt_logit, h->lse_ce, h->per_token, M, h->ce_ntiles, sc,
                            st)); nl += 2;
  }
  if (per_token_out) {
    CUDA_TRY(cudaMemcpyAsync(per_token_out, h->per_token, sizeof(float) * M,
                             cudaMemcpyDeviceToDevice, st));
  }
  if (!train) return cudaSuccess;

  // ---------------- backward ----------------
  // after the first micro-batch of an accumulated step every gradient write adds
  const bool acc = phase == PH_MIDDLE || phase == PH_LAST;
  const int wgrad = acc ? EPI_F32_ACCUM : EPI_F32_STORE;
  float *G = grads;
  // dwte: the first lm_head chunk stores (unless accumulating), later chunks and the embedding
  // backward add; the padding rows V..Vp-1 are never written by the GEMMs and are zeroed
  if (!acc && h->Vp > V)
    CUDA_TRY(cudaMemsetAsync(G + h->off_wte + (size_t)V * C, 0, sizeof(float) * (size_t)(h->Vp - V) * C, st));
  // The weight gradients (dwte here, the layers' weights below) go to the side stream (see
  // gpt_handle::side). fork: the side stream waits for all the main stream has issued; mark /
  // join: an event after side work, and the main stream waiting for it before it rewrites a
  // buffer that work reads.
  const bool sd = side_ok(h);
  auto fork = [&]() -> cudaError_t {
    if (!sd) return cudaSuccess;
    CUDA_TRY(cudaEventRecord(h->ev_fork, st));
    return cudaStreamWaitEvent(h->side, h->ev_fork, 0);
  };
  auto mark = [&](cudaEvent_t ev) { return sd ? cudaEventRecord(ev, h->side) : cudaSuccess; };
  auto join = [&](cudaEvent_t ev) { return sd ? cudaStreamWaitEvent(st, ev, 0) : cudaSuccess; };
  // LayerNorm backward; with the side stream its dgamma column sum runs there, reading one of
  // two partial buffers, which the next-but-one LayerNorm backward reuses after that sum
  int lnbuf = 0;
  bool have_cs[2] = {false, false};
  auto ln_bwd = [&](const T *x, const T *g, const float *mu, const float *rs, const T *dy,
                    T *dres, float *dgout, bool dres_in) -> cudaError_t {
    float *part = lnbuf ? h->dg_partial2 : h->dg_partial;
    if (have_cs[lnbuf]) CUDA_TRY(join(h->ev_cs[lnbuf]));
    CUDA_TRY(launch_layernorm_bwd<T>(x, g, mu, rs, dy, dres, part, dgout, M, C, st, acc, dres_in,
                                     !sd));
    if (sd) {
      CUDA_TRY(fork());
      CUDA_TRY(launch_ln_colsum(part, M, C, dgout, acc, h->side));
      CUDA_TRY(mark(h->ev_cs[lnbuf]));
      have_cs[lnbuf] = true;
    }
    lnbuf ^= 1;
    return cudaSuccess;
  };
  bool have_wte = false;
  for (int r0 = 0; r0 < M; r0 += h->chunk_rows) {
    const int R = M - r0 < h->chunk_rows ? M - r0 : h->chunk_rows;
    const T *yf_c = (const T *)h->yf + (size_t)r0 * C;
    GemmDesc d = gdesc(R, V, C, yf_c, C, 1, W + h->off_wte, C, 1);
    d.split_k = 1;
    Epi &e = d.epi;
    e.kind = EPI_CE_DS; e.out = h->dS; e.ldo = h->ldS; e.targets = h->tgt; e.lse = h->lse_ce;
    e.V = V; e.row_offset = r0; e.sc = sc;
    if (have_wte) CUDA_TRY(join(h->ev_wte));  // dS is rewritten: the last dwte has read it
    CUDA_TRY(gemm(h, d));
    // dwte (+)= dS^T . yf, on the side stream beside dyf
    CUDA_TRY(fork());
    GemmDesc dw = gdesc(V, C, R, h->dS, h->ldS, 0, yf_c, C, 0);
    dw.epi.kind = (acc || r0 > 0) ? EPI_F32_ACCUM : EPI_F32_STORE; dw.epi.outf = G + h->off_wte;
    dw.epi.ldf = C;
    dw.split_k = 1;
    CUDA_TRY(gemm(h, dw, true));
    CUDA_TRY(mark(h->ev_wte));
    have_wte = true;
    // dyf = dS . wte
    d = gdesc(R, C, V, h->dS, h->ldS, 1, W + h->off_wte, C, 0);
    d.epi.kind = EPI_STORE; d.epi.out = (T *)h->dyf + (size_t)r0 * C; d.epi.ldo = C;
    CUDA_TRY(gemm(h, d));
  }
  T *dx = (T *)h->dx;  // the residual-stream gradient starts here (nothing to add to)
  TIMED(h, GPT_KSTAT_LN_BWD, ln_bwd_bytes - (double)M * C * es,
        ln_bwd((T *)h->x_final, W + h->off_lnf, h->muf, h->rsf, (T *)h->dyf, dx, G + h->off_lnf,
               false)); nl += 2;
  bool have_wfc = false, have_wqkv = false;
  for (int l = h->L - 1; l >= 0; --l) {
    Acts &A = h->acts[l];
    const Layer &P = h->layer[l];
    // MLP: x_out = x_mid + gelu(c Wfc^T) Wmp^T
    if (have_wfc) CUDA_TRY(join(h->ev_wfc));  // dh is rewritten: the last dWfc has read it
    GemmDesc d = gdesc(M, mC, C, dx, C, 1, W + P.wmp, mC, 0);
    d.epi.kind = EPI_DGELU; d.epi.out = h->dh; d.epi.ldo = mC; d.epi.aux = A.dgelu; d.epi.ld_aux = mC;
    if (h->cfg.recompute_gelu) {  // dh = dy * gelu'(pre), and gelu(pre) again for dWmp
      d.epi.kind = EPI_DGELU_RECOMP; d.epi.out2 = A.h; d.epi.ldo2 = mC;
    }
    CUDA_TRY(gemm(h, d));
    CUDA_TRY(fork());
    d = gdesc(C, mC, M, dx, C, 0, A.h, mC, 0);
    d.epi.kind = wgrad; d.epi.outf = G + P.wmp; d.epi.ldf = mC;
    CUDA_TRY(gemm(h, d, true));
    CUDA_TRY(mark(h->ev_wmp));
    d = gdesc(mC, C, M, h->dh, mC, 0, A.c, C, 0);
    d.epi.kind = wgrad; d.epi.outf = G + P.wfc; d.epi.ldf = C;
    CUDA_TRY(gemm(h, d, true));
    CUDA_TRY(mark(h->ev_wfc));
    have_wfc = true;
    d = gdesc(M, C, mC, h->dh, mC, 1, W + P.wfc, C, 0);
    d.epi.kind = EPI_STORE; d.epi.out = h->dc; d.epi.ldo = C;
    CUDA_TRY(gemm(h, d));
    CUDA_TRY(join(h->ev_wmp));  // dx is rewritten: dWmp has read it
    TIMED(h, GPT_KSTAT_LN_BWD, ln_bwd_bytes,
          ln_bwd((T *)A.x_mid, W + P.ln2, A.mu2, A.rs2, (T *)h->dc, dx, G + P.ln2, true)); nl += 2;
    // attention: x_mid = x_in + attn(a) Wap^T
    CUDA_TRY(fork());
    d = gdesc(C, C, M, dx, C, 0, A.o, C, 0);
    d.epi.kind = wgrad; d.epi.outf = G + P.wap; d.epi.ldf = C;
    CUDA_TRY(gemm(h, d, true));
    CUDA_TRY(mark(h->ev_wap));
    d = gdesc(M, C, C, dx, C, 1, W + P.wap, C, 0);
    d.epi.kind = EPI_STORE; d.epi.out = h->dout; d.epi.ldo = C;
    if (fused_d(h, Tlen)) {  // D = rowsum(dO * O) per head, for the attention backward
      d.epi.kind = EPI_STORE_DOT; d.epi.aux = A.o; d.epi.ld_aux = C; d.epi.outf = h->Dbuf;
      d.epi.dot_T = Tlen; d.split_k = 1;
    }
    CUDA_TRY(gemm(h, d));
    if (have_wqkv) CUDA_TRY(join(h->ev_wqkv));  // dqkv is rewritten: the last dWqkv has read it
    TIMED(h, GPT_KSTAT_ATTN_BWD, attn_flops(h->windows[l], 8.0),
          attention_bwd<T>(h, (T *)A.qkv, (T *)A.o, (T *)h->dout, A.lse, (T *)h->dqkv, B, Tlen,
                           h->windows[l])); nl += (h->use_bf16 && attn_dst(h, Tlen) && !fused_d(h, Tlen)) ? 3 : 2;
    CUDA_TRY(fork());
    d = gdesc(3 * C, C, M, h->dqkv, 3 * C, 0, A.a, C, 0);
    d.epi.kind = wgrad; d.epi.outf = G + P.wqkv; d.epi.ldf = C;
    CUDA_TRY(gemm(h, d, true));
    CUDA_TRY(mark(h->ev_wqkv));
    have_wqkv = true;
    d = gdesc(M, C, 3 * C, h->dqkv, 3 * C, 1, W + P.wqkv, C, 0);
    d.epi.kind = EPI_STORE; d.epi.out = h->dc; d.epi.ldo = C;
    CUDA_TRY(gemm(h, d));
    CUDA_TRY(join(h->ev_wap));  // dx is rewritten: dWap has read it
    TIMED(h, GPT_KSTAT_LN_BWD, ln_bwd_bytes,
          ln_bwd((T *)A.x_in, W + P.ln1, A.mu1, A.rs1, (T *)h->dc, dx, G + P.ln1, true)); nl += 2;
  }
  // the embedding backward adds into the wte gradient after the last dwte
  if (have_wte) CUDA_TRY(join(h->ev_wte));
  EmbedBwdWs ew{h->emb_ws};
  TIMED(h, GPT_KSTAT_EMBED_BWD, (double)M * C * es + 4.0 * C * h->maxT * (acc ? 2 : 1) + 8.0 * M,
        launch_embed_bwd<T>(h->tok, dx, G + h->off_wte, G + h->off_wpe, M, Tlen, h->maxT, C, h->Vp,
                            ew, st, acc)); nl += embed_bwd_launches(h->Vp);
  // every weight gradient is complete before anything reads the gradients, or the next phase
  // rewrites the activations the side stream reads (and a captured graph rejoins here)
  if (sd) {
    CUDA_TRY(mark(h->ev_side_done));
    CUDA_TRY(join(h->ev_side_done));
  }
  if (phase == PH_FIRST || phase == PH_MIDDLE) return cudaSuccess;  // update after the last
  // ---------------- clip + AdamW ----------------
  TIMED(h, GPT_KSTAT_GRAD_NORM, 4.0 * h->nparams,
        launch_grad_norm(G, h->nparams, h->gn_partials, sc, st)); nl++;
  TIMED(h, GPT_KSTAT_ADAMW, (h->use_bf16 ? 30.0 : 28.0) * h->nparams,
        launch_adamw((float *)params, G, adam_m, adam_v, h->use_bf16 ? h->shadow : nullptr,
                     h->nparams, sc, st)); nl++;
  return cudaSuccess;
}

cudaError_t run(gpt_handle *h, const float *params, float *grads, float *m, float *v, int B,
                int Tlen, bool train, float *ptl, int phase = PH_STEP) {
  if (h->use_bf16) return enqueue<bf16>(h, params, grads, m, v, B, Tlen, train, ptl, phase);
  return enqueue<float>(h, params, grads, m, v, B, Tlen, train, ptl, phase);
}

int check_common(gpt_handle *h, const void *params, const int *tokens, const int *targets, int B,
                 int Tlen) {
  if (!h || !params || !tokens || !targets) return GPT_ERR_INVALID_ARG;
  if (B <= 0 || Tlen <= 0 || B > h->maxB || Tlen > h->maxT) return GPT_ERR_SHAPE;
  if (misaligned(params)) return GPT_ERR_ALIGN;
  return GPT_OK;
}

// Copies tokens/targets (host or device) into the workspace and the hyper-parameters into
// device scalars; clear: also zero the device-written results (loss sum, flags, error word),
// done once per optimizer step (at its first micro-batch).
int stage_inputs(gpt_handle *h, const int *tokens, const int *targets, int M, bool clear = true) {
  const cudaMemcpyKind kt = is_device_ptr(tokens) ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  const cudaMemcpyKind kg = is_device_ptr(targets) ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice;
  TRY(cudaMemcpyAsync(h->tok, tokens, sizeof(int) * M, kt, h->stream));
  TRY(cudaMemcpyAsync(h->tgt, targets, sizeof(int) * M, kg, h->stream));
  TRY(cudaMemcpyAsync(h->sc, h->sc_host, offsetof(DevScalars, sumsq), cudaMemcpyHostToDevice,
                      h->stream));
  // the device-written results of the previous call are cleared
  if (clear)
    TRY(cudaMemsetAsync((char *)h->sc + offsetof(DevScalars, loss), 0,
                        offsetof(DevScalars, counter) - offsetof(DevScalars, loss), h->stream));
  return GPT_OK;
}

int launch_step(gpt_handle *h, const float *params, float *grads, float *m, float *v, int B,
                int Tlen, bool train, float *ptl, int phase = PH_STEP) {
  h->launches = 0;
  const bool capture_ok = h->use_graphs && h->stream != nullptr && !h->time_kernels;
  if (!capture_ok) {
    TRY(run(h, params, grads, m, v, B, Tlen, train, ptl, phase));
    return GPT_OK;
  }
  GraphKey key{B, Tlen, train ? 1 : 0, phase, params, grads, m, v, ptl};
  auto it = h->graphs.find(key);
  if (it == h->graphs.end()) {
    cudaGraph_t g;
    TRY(cudaStreamBeginCapture(h->stream, cudaStreamCaptureModeThreadLocal));
    cudaError_t e = run(h, params, grads, m, v, B, Tlen, train, ptl, phase);
    cudaError_t e2 = cudaStreamEndCapture(h->stream, &g);
    if (e != cudaSuccess) return fail(h, e);
    if (e2 != cudaSuccess) return fail(h, e2);
    cudaGraphExec_t ex;
    e = cudaGraphInstantiate(&ex, g, 0);
    cudaGraphDestroy(g);
    if (e != cudaSuccess) return fail(h, e);
    it = h->graphs.emplace(key, gpt_handle::Captured{ex, h->launches}).first;
  }
  h->launches = it->second.launches;
  TRY(cudaGraphLaunch(it->second.exec, h->stream));
  return GPT_OK;
}

int finish(gpt_handle *h, float *loss, int n_micro = 1) {
  TRY(cudaMemcpyAsync(h->sc_host, h->sc, sizeof(DevScalars), cudaMemcpyDeviceToHost, h->stream));
  TRY(cudaStreamSynchronize(h->stream));
  if (loss) *loss = n_micro == 1 ? h->sc_host->loss : h->sc_host->loss_sum / (float)n_micro;
  if (h->time_kernels) {
    for (int k = 0; k + 1 < h->ev_used; k += 2) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, h->ev[k], h->ev[k + 1]) == cudaSuccess) {
        const int kind = h->ev_kind[k / 2];
        h->stat_ms[kind] += ms;
        h->stat_work[kind] += h->ev_work[k / 2];
        h->stat_launches[kind]++;
      }
    }
    h->ev_used = 0;
  }
  const unsigned err = h->sc_host->err;
  if (err & GPT_DEVERR_TIMEOUT) return GPT_ERR_DEVICE_TIMEOUT;
  if (err & (GPT_DEVERR_BAD_TOKEN | GPT_DEVERR_BAD_TARGET)) return GPT_ERR_BAD_TOKEN;
  return GPT_OK;
}

// M: positions whose mean loss the step optimises (n_micro * B * T).
void set_hyper(gpt_handle *h, long M, float lr, float wd, float clip, long t) {
  DevScalars *s = h->sc_host;
  s->lr = lr; s->wd = wd; s->clip = clip;
  s->beta1 = h->cfg.beta1; s->beta2 = h->cfg.beta2; s->eps = h->cfg.adam_eps;
  s->bias1 = (float)(1.0 - pow((double)h->cfg.beta1, (double)t));
  s->bias2 = (float)(1.0 - pow((double)h->cfg.beta2, (double)t));
  s->inv_M = (float)(1.0 / (double)M);
  s->step = (int)t;
}

}  // namespace

// ======================================================================================
// C ABI
// ======================================================================================
extern "C" {

const char *gpt_strerror(int s) {
  switch (s) {
    case GPT_OK: return "ok";
    case GPT_ERR_INVALID_ARG: return "invalid argument";
    case GPT_ERR_SHAPE: return "unsupported shape";
    case GPT_ERR_ALIGN: return "pointer not 16-byte aligned";
    case GPT_ERR_OOM: return "out of device memory";
    case GPT_ERR_CUDA: return "CUDA error";
    case GPT_ERR_NONFINITE: return "non-finite loss or gradient norm; update skipped";
    case GPT_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case GPT_ERR_BAD_TOKEN: return "token or target id out of range";
    default: return "unknown status";
  }
}

gpt_handle *gpt_create(const gpt_config *cfg, int *status) {
  int dummy;
  if (!status) status = &dummy;
  *status = GPT_ERR_INVALID_ARG;
  if (!cfg) return nullptr;
  const gpt_config c = *cfg;
  if (c.precision != GPT_FP32 && c.precision != GPT_BF16) return nullptr;
  if (c.vocab <= 0 || c.vocab_padded < c.vocab || c.n_layer <= 0 || c.n_head <= 0 ||
      c.n_embd <= 0 || c.max_T <= 0 || c.max_B <= 0 || c.mlp_mult <= 0)
    return nullptr;
  if (!(c.ln_eps > 0.f) || !(c.beta1 >= 0.f && c.beta1 < 1.f) || !(c.beta2 >= 0.f && c.beta2 < 1.f) ||
      !(c.adam_eps > 0.f))
    return nullptr;
  *status = GPT_ERR_SHAPE;
  const int C = c.n_embd, H = c.n_head;
  if (C % H) return nullptr;
  const int hd = C / H;
  if (hd != 32 && hd != 64 && hd != 128) return nullptr;
  const bool bf = c.precision == GPT_BF16;
  if (bf ? (C % 64 != 0) : (C % 4 != 0)) return nullptr;
  if (C > (bf ? 2048 : 1024)) return nullptr;
  if ((long)c.max_B * c.max_T > GPT_MAX_TOKENS) return nullptr;
  if (c.vocab_padded > 131072) return nullptr;

  gpt_handle *h = new gpt_handle();
  h->cfg = c;
  h->windows.assign(c.n_layer, -1);
  if (c.window_left)
    for (int l = 0; l < c.n_layer; ++l) h->windows[l] = c.window_left[l];
  h->cfg.window_left = nullptr;
  h->C = C; h->H = H; h->hd = hd; h->mC = c.mlp_mult * C; h->V = c.vocab; h->Vp = c.vocab_padded;
  h->L = c.n_layer; h->maxT = c.max_T; h->maxB = c.max_B; h->maxM = c.max_B * c.max_T;
  h->use_bf16 = bf;
  h->stream = nullptr;
  h->step = 0;
  h->last_norm = NAN;
  h->shadow_src = nullptr;
  h->shadow_valid = false;
  h->use_graphs = true;
  h->time_kernels = false;
  h->ev_used = 0;
  for (int k = 0; k < GPT_KSTAT_COUNT; ++k) { h->stat_launches[k] = 0; h->stat_ms[k] = 0; h->stat_work[k] = 0; }
  h->tc = nullptr;
  h->muon_ws = nullptr;
  cudaGetDevice(&h->device);

  // ---- parameter layout ----
  size_t off = 0;
  auto add = [&](const char *name, int nd, long long d0, long long d1) {
    gpt_tensor_desc d;
    memset(&d, 0, sizeof(d));
    snprintf(d.name, sizeof(d.name), "%s", name);
    d.offset = (long long)off; d.ndim = nd; d.shape[0] = d0; d.shape[1] = nd > 1 ? d1 : 0;
    h->descs.push_back(d);
    size_t n = (size_t)d0 * (nd > 1 ? (size_t)d1 : 1);
    size_t o = off;
    off += n;
    return o;
  };
  char nm[32];
  h->off_wte = add("wte", 2, h->Vp, C);
  h->off_wpe = add("wpe", 2, h->maxT, C);
  for (int l = 0; l < h->L; ++l) {
    Layer P;
    snprintf(nm, 32, "h%d.ln1.g", l); P.ln1 = add(nm, 1, C, 0);
    snprintf(nm, 32, "h%d.w_qkv", l); P.wqkv = add(nm, 2, 3 * C, C);
    snprintf(nm, 32, "h%d.w_attnproj", l); P.wap = add(nm, 2, C, C);
    snprintf(nm, 32, "h%d.ln2.g", l); P.ln2 = add(nm, 1, C, 0);
    snprintf(nm, 32, "h%d.w_fc", l); P.wfc = add(nm, 2, h->mC, C);
    snprintf(nm, 32, "h%d.w_mlpproj", l); P.wmp = add(nm, 2, C, h->mC);
    h->layer.push_back(P);
  }
  h->off_lnf = add("lnf.g", 1, C, 0);
  h->nparams = off;

  // ---- workspace ----
  const size_t es = bf ? 2 : 4;
  const size_t M = h->maxM;
  h->ce_tile_n = SIMT_TILE_N;  // the stats buffer is sized for the narrowest column tile
  h->ce_ntiles = (h->V + h->ce_tile_n - 1) / h->ce_tile_n;
  h->chunk_rows = c.lmhead_chunk_rows > 0 ? c.lmhead_chunk_rows : 8192;
  if (h->chunk_rows > (int)M) h->chunk_rows = (int)M;
  h->ldS = (h->V + 7) / 8 * 8;
  h->splitk_elems = (size_t)8 * ((size_t)h->mC * C > (size_t)M * C ? (size_t)h->mC * C : (size_t)M * C);

  std::vector<std::pair<void **, size_t>> req;
  auto need = [&](void **p, size_t bytes) { req.push_back({p, bytes}); };
  h->acts.resize(h->L);
  for (int l = 0; l < h->L; ++l) {
    Acts &A = h->acts[l];
    need(&A.x_in, M * C * es); need(&A.a, M * C * es); need(&A.qkv, M * 3 * C * es);
    need(&A.o, M * C * es); need(&A.x_mid, M * C * es); need(&A.c, M * C * es);
    need(&A.dgelu, M * h->mC * es);
    if (!c.recompute_gelu || l == 0) need(&A.h, M * h->mC * es);
    need((void **)&A.lse, M * H * 4); need((void **)&A.mu1, M * 4); need((void **)&A.rs1, M * 4);
    need((void **)&A.mu2, M * 4); need((void **)&A.rs2, M * 4);
  }
  need(&h->x_final, M * C * es); need(&h->yf, M * C * es);
  need((void **)&h->muf, M * 4); need((void **)&h->rsf, M * 4);
  need((void **)&h->stats, M * h->ce_ntiles * 8); need((void **)&h->tgt_logit, M * 4);
  need((void **)&h->lse_ce, M * 4); need((void **)&h->per_token, M * 4);
  need(&h->dS, (size_t)h->chunk_rows * h->ldS * es);
  need(&h->dx, M * C * es); need(&h->dh, M * h->mC * es); need(&h->dc, M * C * es);
  need(&h->dqkv, M * 3 * C * es); need(&h->dout, M * C * es); need(&h->dyf, M * C * es);
  need((void **)&h->Dbuf, M * H * 4);
  // dS^T scratch of the attention backward: B*H*T^2 bf16 (403 MB at 124M), when it is modest
  const size_t dst_bytes = (size_t)c.max_B * H * (size_t)c.max_T * c.max_T * 2;
  const bool use_dst = bf && (c.max_T % 8 == 0) && dst_bytes <= ((size_t)4 << 30) &&
                       (C / H == 64);
  if (use_dst) need((void **)&h->dst, dst_bytes);
  else h->dst = nullptr;
  need((void **)&h->dg_partial, (size_t)layernorm_bwd_blocks((int)M) * C * 4);
  need((void **)&h->dg_partial2, (size_t)layernorm_bwd_blocks((int)M) * C * 4);
  need((void **)&h->gn_partials, (size_t)grad_norm_blocks() * 8);
  need((void **)&h->splitk, h->splitk_elems * 4);
  need((void **)&h->splitk2, h->splitk_elems * 4);
  need(&h->emb_ws, embed_bwd_ws_bytes((int)M, C));
  need((void **)&h->tok, M * 4); need((void **)&h->tgt, M * 4);
  need((void **)&h->sc, sizeof(DevScalars));
  if (bf) need((void **)&h->shadow, h->nparams * 2);
  else h->shadow = nullptr;
  size_t total = 0;
  for (auto &r : req) total += align_up(r.second);
  h->ws_bytes = total;
  cudaError_t e = cudaMalloc(&h->ws, total);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *status = e == cudaErrorMemoryAllocation ? GPT_ERR_OOM : GPT_ERR_CUDA;
    delete h;
    return nullptr;
  }
  size_t o2 = 0;
  for (auto &r : req) {
    *r.first = h->ws + o2;
    o2 += align_up(r.second);
  }
  if (c.recompute_gelu)  // one activation buffer for all layers
    for (int l = 1; l < h->L; ++l) h->acts[l].h = h->acts[0].h;
  *status = GPT_ERR_CUDA;
  if (cudaMemset(h->ws, 0, total) != cudaSuccess || cudaMallocHost(&h->sc_host, sizeof(DevScalars)) != cudaSuccess) {
    cudaGetLastError();
    cudaFree(h->ws);
    delete h;
    return nullptr;
  }
  memset(h->sc_host, 0, sizeof(DevScalars));
  if (bf) {
    if (tc_gemm_create(&h->tc) != cudaSuccess) {
      cudaGetLastError();
      h->tc = nullptr;
    } else {
      tc_gemm_set_splitk_capacity(h->tc, h->splitk_elems);
    }
  }
  // the weight-gradient stream and its events; without them everything runs on one stream
  h->side = nullptr;
  if (cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking) == cudaSuccess) {
    cudaEvent_t *evs[9] = {&h->ev_fork, &h->ev_wmp, &h->ev_wfc, &h->ev_wap, &h->ev_wqkv,
                           &h->ev_wte, &h->ev_side_done, &h->ev_cs[0], &h->ev_cs[1]};
    bool ok = true;
    for (auto *ev : evs) ok = ok && cudaEventCreateWithFlags(ev, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      cudaStreamDestroy(h->side);
      h->side = nullptr;
    }
  } else {
    cudaGetLastError();
    h->side = nullptr;
  }
  *status = GPT_OK;
  return h;
}

void gpt_destroy(gpt_handle *h) {
  if (!h) return;
  cudaSetDevice(h->device);
  for (auto &kv : h->graphs) cudaGraphExecDestroy(kv.second.exec);
  for (auto ev : h->ev) cudaEventDestroy(ev);
  if (h->side) {
    for (auto ev : {h->ev_fork, h->ev_wmp, h->ev_wfc, h->ev_wap, h->ev_wqkv, h->ev_wte,
                    h->ev_side_done, h->ev_cs[0], h->ev_cs[1]})
      cudaEventDestroy(ev);
    cudaStreamDestroy(h->side);
  }
  if (h->tc) tc_gemm_destroy(h->tc);
  if (h->muon_ws) cudaFree(h->muon_ws);
  cudaFree(h->ws);
  cudaFreeHost(h->sc_host);
  delete h;
}

size_t gpt_num_params(const gpt_handle *h) { return h ? h->nparams : 0; }

int gpt_param_layout(const gpt_handle *h, gpt_tensor_desc *out, int cap) {
  if (!h || (cap > 0 && !out)) return GPT_ERR_INVALID_ARG;
  for (int i = 0; i < (int)h->descs.size() && i < cap; ++i) out[i] = h->descs[i];
  return (int)h->descs.size();
}

int gpt_set_stream(gpt_handle *h, void *s) {
  if (!h) return GPT_ERR_INVALID_ARG;
  h->stream = (cudaStream_t)s;
  return GPT_OK;
}

int gpt_params_changed(gpt_handle *h) {
  if (!h) return GPT_ERR_INVALID_ARG;
  h->shadow_valid = false;
  return GPT_OK;
}

int gpt_forward_loss(gpt_handle *h, const float *params, const int *tokens, const int *targets,
                     int B, int T, float *loss, float *per_token_loss) {
  int s = check_common(h, params, tokens, targets, B, T);
  if (s) return s;
  if (!loss) return GPT_ERR_INVALID_ARG;
  cudaSetDevice(h->device);
  const int M = B * T;
  h->ev_used = 0;
  set_hyper(h, M, 0.f, 0.f, 1.f, h->step + 1);
  if ((s = stage_inputs(h, tokens, targets, M))) return s;
  if (h->use_bf16) {  // forward-only calls refresh the bf16 weights every time
    TRY(launch_to_bf16(params, h->shadow, h->nparams, h->stream));
    h->shadow_src = params;
    h->shadow_valid = true;
  }
  h->launches = 0;
  TRY(run(h, params, nullptr, nullptr, nullptr, B, T, false, per_token_loss));
  s = finish(h, loss);
  if (s) return s;
  return isfinite(*loss) ? GPT_OK : GPT_ERR_NONFINITE;
}

int gpt_train_step(gpt_handle *h, float *params, float *grads, float *adam_m, float *adam_v,
                   const int *tokens, const int *targets, int B, int T, float lr, float wd,
                   float clip, float *loss) {
  return gpt_train_step_accum(h, params, grads, adam_m, adam_v, tokens, targets, 1, B, T, lr, wd,
                              clip, loss);
}

int gpt_train_step_accum(gpt_handle *h, float *params, float *grads, float *adam_m,
                         float *adam_v, const int *tokens, const int *targets, int n_micro,
                         int B, int T, float lr, float wd, float clip, float *loss) {
  int s = check_common(h, params, tokens, targets, B, T);
  if (s) return s;
  if (!grads || !adam_m || !adam_v || !loss || n_micro < 1) return GPT_ERR_INVALID_ARG;
  if (misaligned(grads) || misaligned(adam_m) || misaligned(adam_v)) return GPT_ERR_ALIGN;
  if (!isfinite(lr) || !isfinite(wd) || !(clip > 0.f)) return GPT_ERR_INVALID_ARG;
  cudaSetDevice(h->device);
  const int M = B * T;
  const long t = h->step + 1;
  h->ev_used = 0;
  set_hyper(h, (long)n_micro * M, lr, wd, clip, t);
  if (h->use_bf16 && (!h->shadow_valid || h->shadow_src != params)) {
    TRY(launch_to_bf16(params, h->shadow, h->nparams, h->stream));
    h->shadow_src = params;
    h->shadow_valid = true;
  }
  int launches = 0;
  for (int i = 0; i < n_micro; ++i) {
    const int phase = n_micro == 1 ? PH_STEP : i == 0 ? PH_FIRST : i + 1 < n_micro ? PH_MIDDLE : PH_LAST;
    if ((s = stage_inputs(h, tokens + (size_t)i * M, targets + (size_t)i * M, M, i == 0))) return s;
    if ((s = launch_step(h, params, grads, adam_m, adam_v, B, T, true, nullptr, phase))) return s;
    launches += h->launches;
  }
  h->launches = launches;
  s = finish(h, loss, n_micro);
  h->last_norm = h->sc_host->norm;
  if (s) return s;
  if (h->sc_host->nonfinite) return GPT_ERR_NONFINITE;
  h->step = t;
  return GPT_OK;
}

int gpt_forward_backward(gpt_handle *h, const float *params, float *grads, const int *tokens,
                         const int *targets, int n_micro, int B, int T, float grad_scale,
                         float *loss) {
  int s = check_common(h, params, tokens, targets, B, T);
  if (s) return s;
  if (!grads || !loss || n_micro < 1 || !isfinite(grad_scale)) return GPT_ERR_INVALID_ARG;
  if (misaligned(grads)) return GPT_ERR_ALIGN;
  cudaSetDevice(h->device);
  const int M = B * T;
  h->ev_used = 0;
  // the gradient of the mean loss over all n_micro * B * T positions, times grad_scale
  set_hyper(h, (long)n_micro * M, 0.f, 0.f, 1.f, h->step + 1);
  h->sc_host->inv_M = (float)((double)grad_scale / ((double)n_micro * M));
  if (h->use_bf16 && (!h->shadow_valid || h->shadow_src != params)) {
    TRY(launch_to_bf16(params, h->shadow, h->nparams, h->stream));
    h->shadow_src = params;
    h->shadow_valid = true;
  }
  int launches = 0;
  for (int i = 0; i < n_micro; ++i) {
    // gradients stored by the first micro-batch, added by the others; no update
    const int phase = i == 0 ? PH_FIRST : PH_MIDDLE;
    if ((s = stage_inputs(h, tokens + (size_t)i * M, targets + (size_t)i * M, M, i == 0))) return s;
    if ((s = launch_step(h, params, grads, nullptr, nullptr, B, T, true, nullptr, phase))) return s;
    launches += h->launches;
  }
  h->launches = launches;
  s = finish(h, loss, n_micro);
  if (s) return s;
  return h->sc_host->nonfinite ? GPT_ERR_NONFINITE : GPT_OK;
}

int gpt_sumsq(gpt_handle *h, const float *x, size_t n, double *sumsq_dev) {
  if (!h || !x || !sumsq_dev) return GPT_ERR_INVALID_ARG;
  if (misaligned(x) || ((uintptr_t)sumsq_dev & 7u)) return GPT_ERR_ALIGN;
  cudaSetDevice(h->device);
  unsigned *counter = (unsigned *)((char *)h->sc + offsetof(DevScalars, counter2));
  TRY(launch_sumsq(x, n, h->gn_partials, counter, sumsq_dev, h->stream));
  return GPT_OK;
}

int gpt_adamw_ranges(gpt_handle *h, float *params, const float *grads, float *adam_m,
                     float *adam_v, const long long *offsets, const long long *counts,
                     int nranges, float lr, float wd, float clip, const double *sumsq_dev,
                     long step) {
  if (!h || !params || !grads || !adam_m || !adam_v || !offsets || !counts || !sumsq_dev)
    return GPT_ERR_INVALID_ARG;
  if (nranges < 0 || nranges > ADAM_MAX_RANGES || step < 1 || !isfinite(lr) || !isfinite(wd) ||
      !(clip > 0.f))
    return GPT_ERR_INVALID_ARG;
  if (misaligned(params) || misaligned(grads) || misaligned(adam_m) || misaligned(adam_v) ||
      ((uintptr_t)sumsq_dev & 7u))
    return GPT_ERR_ALIGN;
  if (nranges == 0) return GPT_OK;
  AdamRanges rg;
  memset(&rg, 0, sizeof(rg));
  rg.n = nranges;
  long long base = 0;
  for (int k = 0; k < nranges; ++k) {
    if (offsets[k] < 0 || counts[k] < 0 || offsets[k] + counts[k] > (long long)h->nparams)
      return GPT_ERR_SHAPE;
    if ((offsets[k] & 3) || (counts[k] & 3)) return GPT_ERR_ALIGN;
    rg.offset[k] = offsets[k];
    rg.count[k] = counts[k];
    rg.base[k] = base;
    base += counts[k];
  }
  rg.lr = lr; rg.wd = wd; rg.clip = clip;
  rg.beta1 = h->cfg.beta1; rg.beta2 = h->cfg.beta2; rg.eps = h->cfg.adam_eps;
  rg.bias1 = (float)(1.0 - pow((double)h->cfg.beta1, (double)step));
  rg.bias2 = (float)(1.0 - pow((double)h->cfg.beta2, (double)step));
  cudaSetDevice(h->device);
  TRY(launch_adamw_ranges(params, grads, adam_m, adam_v, rg, sumsq_dev, h->stream));
  h->shadow_valid = false;  // params changed outside the step
  return GPT_OK;
}

int gpt_muon_update(gpt_handle *h, float *params, const float *grads, float *adam_m,
                    float *adam_v, const gpt_muon_config *mc, float lr, float wd, float clip) {
  if (!h || !params || !grads || !adam_m || !adam_v || !mc || !mc->coeffs) return GPT_ERR_INVALID_ARG;
  if (misaligned(params) || misaligned(grads) || misaligned(adam_m) || misaligned(adam_v))
    return GPT_ERR_ALIGN;
  if (!isfinite(lr) || !isfinite(wd) || !(clip > 0.f) || mc->ns_steps < 0 || mc->ns_steps > 16 ||
      !isfinite(mc->matrix_lr) || !isfinite(mc->weight_decay) || !(mc->momentum >= 0.f) ||
      !(mc->momentum < 1.f) || !(mc->beta2 >= 0.f) || !(mc->beta2 < 1.f) || !(mc->eps > 0.f))
    return GPT_ERR_INVALID_ARG;
  if (!h->use_bf16 || !h->tc) return GPT_ERR_SHAPE;  // the iteration runs on the tensor cores
  cudaSetDevice(h->device);
  cudaStream_t st = h->stream;
  const int C = h->C, mC = h->mC, L = h->L;
  const size_t lstride = L > 1 ? h->layer[1].wqkv - h->layer[0].wqkv : 0;
  MuonGroup groups[4] = {{3 * C, C, L, h->layer[0].wqkv, lstride},
                         {C, C, L, h->layer[0].wap, lstride},
                         {mC, C, L, h->layer[0].wfc, lstride},
                         {C, mC, L, h->layer[0].wmp, lstride}};
  if (!h->muon_ws) {
    const size_t bytes = muon_scratch_bytes(groups, 4);
    TRY(cudaMalloc(&h->muon_ws, bytes));
    TRY(cudaMemset(h->muon_ws, 0, bytes));
  }
  const MuonScratch scr = muon_scratch_carve(h->muon_ws, groups, 4);
  const long t = h->step + 1;
  h->ev_used = 0;
  set_hyper(h, 1, lr, wd, clip, t);
  TRY(cudaMemcpyAsync(h->sc, h->sc_host, offsetof(DevScalars, sumsq), cudaMemcpyHostToDevice, st));
  TRY(cudaMemsetAsync((char *)h->sc + offsetof(DevScalars, loss), 0,
                      offsetof(DevScalars, counter) - offsetof(DevScalars, loss), st));
  int nl = 0;
  // global norm and clip coefficient of the raw gradient
  TIMED_S(h, GPT_KSTAT_GRAD_NORM, 4.0 * h->nparams,
        launch_grad_norm(grads, h->nparams, h->gn_partials, h->sc, st)); nl++;
  // AdamW: embeddings (wte is also the tied lm_head), positions, LayerNorm gains
  MuonAdamRanges rg;
  memset(&rg, 0, sizeof(rg));
  rg.lr = lr; rg.wd = wd;
  rg.beta1 = h->cfg.beta1; rg.beta2 = h->cfg.beta2; rg.eps = h->cfg.adam_eps;
  rg.bias1 = h->sc_host->bias1; rg.bias2 = h->sc_host->bias2;
  std::vector<std::pair<long long, long long>> ranges;
  ranges.push_back({(long long)h->off_wte, (long long)h->Vp * C});
  ranges.push_back({(long long)h->off_wpe, (long long)h->maxT * C});
  for (int l = 0; l < L; ++l) {
    ranges.push_back({(long long)h->layer[l].ln1, C});
    ranges.push_back({(long long)h->layer[l].ln2, C});
  }
  ranges.push_back({(long long)h->off_lnf, C});
  for (size_t k0 = 0; k0 < ranges.size(); k0 += MUON_ADAM_MAX_RANGES) {
    rg.n = 0;
    for (size_t k = k0; k < ranges.size() && rg.n < MUON_ADAM_MAX_RANGES; ++k, ++rg.n) {
      rg.offset[rg.n] = ranges[k].first;
      rg.count[rg.n] = ranges[k].second;
    }
    TIMED_S(h, GPT_KSTAT_ADAMW, 28.0 * (double)(h->off_wpe + (size_t)h->maxT * C),
          muon_adamw_ranges(params, grads, adam_m, adam_v, rg, h->sc, st)); nl++;
  }
  // Muon on the block matrices, one group of equal shapes at a time
  MuonStepArgs a;
  a.params = params; a.grads = grads; a.mom = adam_m; a.sv = adam_v;
  a.coeffs = mc->coeffs; a.ns = mc->ns_steps;
  a.lr = mc->matrix_lr; a.wd = mc->weight_decay; a.mu = mc->momentum; a.beta2 = mc->beta2;
  a.eps = mc->eps; a.sc = h->sc; a.err = &h->sc->err;
  for (int gi = 0; gi < 4; ++gi) {
    const MuonGroup &g = groups[gi];
    const double d = g.rows < g.cols ? g.rows : g.cols, big = g.rows < g.cols ? g.cols : g.rows;
    const double flops = (double)g.count * a.ns * (4.0 * d * d * big + 2.0 * d * d * d);
    TIMED_S(h, GPT_KSTAT_MUON, flops, muon_update_group(h->tc, g, a, scr, st, &nl));
  }
  h->launches = nl;
  h->shadow_valid = false;  // the bf16 weights are refreshed by the next forward
  float dummy = 0.f;
  int s = finish(h, &dummy);
  h->last_norm = h->sc_host->norm;
  if (s) return s;
  if (h->sc_host->nonfinite) return GPT_ERR_NONFINITE;
  h->step = t;
  return GPT_OK;
}

int gpt_get_step(const gpt_handle *h, long *step) {
  if (!h || !step) return GPT_ERR_INVALID_ARG;
  *step = h->step;
  return GPT_OK;
}

int gpt_set_step(gpt_handle *h, long step) {
  if (!h || step < 0) return GPT_ERR_INVALID_ARG;
  h->step = step;
  h->shadow_valid = false;
  return GPT_OK;
}

float gpt_last_grad_norm(const gpt_handle *h) { return h ? h->last_norm : NAN; }

int gpt_set_option(gpt_handle *h, int option, long value) {
  if (!h) return GPT_ERR_INVALID_ARG;
  if (option == GPT_OPT_USE_GRAPHS) {
    h->use_graphs = value != 0;
    return GPT_OK;
  }
  if (option == GPT_OPT_TIME_KERNELS) {
    h->time_kernels = value != 0;
    if (h->time_kernels && h->ev.empty()) {
      const int n = 2 * (48 * h->L + 256);
      h->ev.resize(n);
      h->ev_work.assign(n / 2, 0.0);
      h->ev_kind.assign(n / 2, 0);
      for (int i = 0; i < n; ++i)
        if (cudaEventCreate(&h->ev[i]) != cudaSuccess) return fail(h, cudaGetLastError());
    }
    return GPT_OK;
  }
  return GPT_ERR_INVALID_ARG;
}

int gpt_kernel_stats(gpt_handle *h, int kind, long long *launches, double *total_ms,
                     double *work, int reset) {
  if (!h || kind < 0 || kind >= GPT_KSTAT_COUNT) return GPT_ERR_INVALID_ARG;
  // GEMM: every GEMM launch's time with the method's own FLOPs (the recompute excluded)
  const bool all_gemm = kind == GPT_KSTAT_GEMM;
  const long long n = h->stat_launches[kind] + (all_gemm ? h->stat_launches[GPT_KSTAT_GEMM_RECOMPUTE] : 0);
  const double ms = h->stat_ms[kind] + (all_gemm ? h->stat_ms[GPT_KSTAT_GEMM_RECOMPUTE] : 0.0);
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  if (work) *work = h->stat_work[kind];
  if (reset) {
    for (int k = 0; k < GPT_KSTAT_COUNT; ++k) { h->stat_launches[k] = 0; h->stat_ms[k] = 0; h->stat_work[k] = 0; }
  }
  return GPT_OK;
}

int gpt_last_launch_count(const gpt_handle *h) { return h ? h->launches : 0; }

const char *gpt_last_cuda_error(const gpt_handle *h) { return h ? h->cuda_err.c_str() : ""; }

}  // extern "C"
