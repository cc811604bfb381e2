// tcgen05 / TMEM / TMA GEMM for sm_100a (bf16 operands, fp32 accumulation in TMEM).
#pragma once
#include "common.cuh"

constexpr int TC_BM = 128;  // rows per CTA tile (TMEM lanes)
constexpr int TC_BN = 256;  // columns per CTA tile (TMEM fp32 columns)
constexpr int TC_BK = 128;  // K per pipeline stage (two 64-element, 128-byte swizzle chunks of bf16)
constexpr int TC_CE_TILE = TC_BN / 2;  // column width of one cross-entropy statistics partial

struct TcGemm;
cudaError_t tc_gemm_create(TcGemm **out);
void tc_gemm_destroy(TcGemm *t);
// Floats available for split-K partials at GemmDesc::partial (0: never split).
void tc_gemm_set_splitk_capacity(TcGemm *t, size_t floats);
// True when the shape, strides and epilogue can run on the tensor-core path.
bool tc_gemm_supported(const GemmDesc &d);
// CTA group (1 or 2) and K split the launcher chooses (host only); capacity = floats of split-K
// scratch (0: no split).
void tc_gemm_plan(const GemmDesc &d, size_t capacity, int sms, int *cta_group, int *split);
// Enqueues the GEMM (and its split-K reduction, if any). d.split_k <= 0 lets the launcher
// choose the split (only for elementwise epilogues); the chosen value is written back.
cudaError_t tc_gemm_launch(TcGemm *t, GemmDesc &d, cudaStream_t st, int *launches);
