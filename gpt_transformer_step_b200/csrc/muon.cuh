// Hybrid Muon + AdamW optimizer update: launchers (muon.cu).
#pragma once
#include "common.cuh"

struct TcGemm;

constexpr int MUON_MAX_BLOCKS = 592;  // blocks per matrix of the elementwise kernels

// `count` matrices of rows x cols in the flat parameter layout: matrix l at off0 + l * stride.
struct MuonGroup {
  int rows, cols, count;
  size_t off0, stride;
};

// Device scratch for one group at a time (sized for the largest group).
struct MuonScratch {
  bf16 *X[2];          // [count][rows][cols], the iterate and the next one
  bf16 *A, *Bm;        // [count][d][d], d = min(rows, cols)
  float *q, *qh, *rs;  // [count][lines] per line: sum of X^2, that over max(s, eps), rsqrt
  double *partials;    // [count][MUON_MAX_BLOCKS]
  unsigned *counters;  // [count], zero between calls
  float *scale, *gamma;
};
size_t muon_scratch_bytes(const MuonGroup *groups, int ngroups);
MuonScratch muon_scratch_carve(void *base, const MuonGroup *groups, int ngroups);

struct MuonStepArgs {
  float *params;
  const float *grads;
  float *mom;  // momentum buffers (flat layout)
  float *sv;   // factored second moments (at each matrix's offset of a flat vector)
  const float *coeffs;  // host: ns triples (a, b, c)
  int ns;
  float lr, wd, mu, beta2, eps;
  const DevScalars *sc;  // coef (clip), nonfinite / err flags
  unsigned *err;
};

// Muon on every matrix of the group (momentum, Polar Express, factored second moment,
// cautious update). Adds the kernel launches to *launches.
cudaError_t muon_update_group(TcGemm *tc, const MuonGroup &grp, const MuonStepArgs &a,
                              const MuonScratch &s, cudaStream_t st, int *launches);

// AdamW on ranges of the flat vectors (p, g, m, v share the layout), coef from the scalars.
constexpr int MUON_ADAM_MAX_RANGES = 64;
struct MuonAdamRanges {
  int n;
  long long offset[MUON_ADAM_MAX_RANGES], count[MUON_ADAM_MAX_RANGES];
  float lr, wd, beta1, beta2, eps, bias1, bias2;
};
cudaError_t muon_adamw_ranges(float *p, const float *g, float *m, float *v,
                              const MuonAdamRanges &rg, const DevScalars *sc, cudaStream_t st);
