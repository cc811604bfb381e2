"""Gradient parity of the bf16 tensor-core path where only large shapes reach its code paths.

1. A medium model the oracle finishes in well under a minute, chosen so that the launch plan
   takes CTA pairs (cta_group::2) for the QKV and MLP fc GEMMs, K splits for the weight
   gradients, several (ragged) lm_head backward chunks and a left window: per-tensor gradient
   cosine >= 0.999 against the oracle, the loss within 5e-3 and the AdamW update within
   2e-2 * lr given the same gradients (the spec bf16 bounds).
2. The full workloads (GPT-2 124M B=16 x T=1024, 350M B=8 x T=1024, 124M-width T=2048 with
   alternating 512-key windows) in the launch configuration the bench times: the bf16 path's
   gradients against the fp32 validation path's (CUDA-core kernels that match the oracle token
   by token at these sizes and element by element at small ones), cosine >= 0.999 per tensor.
"""
import numpy as np
import pytest

import oracle
from gpt_transformer_step_b200 import binding as gb
from gpt_transformer_step_b200 import fixtures as fx
from tests import gpu_util as U

MEDIUM = fx.ModelShape(vocab=3000, vocab_padded=3072, n_layer=2, n_head=4, n_embd=256,
                       max_T=512, window_left=[64, -1])
MEDIUM_B, MEDIUM_T, MEDIUM_CHUNK = 2, 512, 384


def _scratch_floats(sh, M):
    # split-K scratch of the step's workspace: 8 x max(mC * C, M * C) floats
    C = sh.n_embd
    return 8 * max(sh.mlp_mult * C * C, M * C)


def _plans(sh, M):
    C, mC = sh.n_embd, sh.mlp_mult * sh.n_embd
    s = _scratch_floats(sh, M)
    return {
        "qkv": gb.gemm_plan(M, 3 * C, C, "store", s),
        "fc": gb.gemm_plan(M, mC, C, "store_gelu", s),
        "wgrad_qkv": gb.gemm_plan(3 * C, C, M, "f32_store", s),
        "wgrad_fc": gb.gemm_plan(mC, C, M, "f32_store", s),
        "wgrad_mlpproj": gb.gemm_plan(C, mC, M, "f32_store", s),
    }


def test_medium_model_takes_the_large_shape_paths():
    """Host check (no GPU) of the launch plan the parity case below runs with."""
    p = _plans(MEDIUM, MEDIUM_B * MEDIUM_T)
    assert p["qkv"][1] == 2 and p["fc"][1] == 2, p
    assert all(p[k][2] > 1 for k in ("wgrad_qkv", "wgrad_fc", "wgrad_mlpproj")), p
    assert -(-MEDIUM_B * MEDIUM_T // MEDIUM_CHUNK) >= 2 and (MEDIUM_B * MEDIUM_T) % MEDIUM_CHUNK


@pytest.mark.gpu
def test_medium_model_bf16_matches_oracle():
    sh, B, T = MEDIUM, MEDIUM_B, MEDIUM_T
    lr, wd, clip = 6e-4, 0.1, 1.0
    p = fx.init_params(sh, 5)
    tok, tgt = fx.zipf_tokens(sh.vocab, 1.05, B, T, 5)
    st = U.make_step(sh, B, T, 1, lmhead_chunk_rows=MEDIUM_CHUNK)
    try:
        r = U.gpu_train_step(st, p, tok, tgt, lr, wd, clip)
    finally:
        st.close()
    o = oracle.Oracle.from_shape(sh, dtype=np.float32)
    loss, g = o.forward_backward(p, tok, tgt)
    assert abs(r.loss - loss) <= U.BF16_LOSS_ABS, (r.loss, loss)
    U.assert_bf16_grads(sh, r.grads, g, "medium vs oracle")
    zeros = np.zeros_like(p, dtype=np.float64)
    pe, _, _, n = U.oracle_adamw_on(r.grads, p, zeros, zeros, lr, wd, clip, 1)
    assert abs(r.norm - n) <= 1e-4 * n
    assert np.abs(r.params - pe).max() <= U.BF16_UPDATE_ABS_PER_LR * lr


def test_gpt2_124m_plan_uses_pairs_splits_and_chunks():
    """Host check (no GPU) of the launch plan of the full 124M step."""
    wl = fx.WORKLOADS["gpt2_124m_bf16"]
    M = wl.B * wl.T
    p = _plans(wl.shape, M)
    assert p["qkv"][1] == 2 and p["fc"][1] == 2, p
    assert all(p[k][2] > 1 for k in ("wgrad_qkv", "wgrad_fc", "wgrad_mlpproj")), p
    assert M // 8192 == 2  # the default lm_head chunk (8192 rows): two chunks


@pytest.mark.gpu
@pytest.mark.parametrize("name,recompute", [("gpt2_124m_bf16", False), ("gpt2_350m_bf16", False),
                                            ("gpt2_124m_swa_bf16", False),
                                            ("gpt2_124m_bf16", True)])
def test_full_size_bf16_grads_match_fp32_path(name, recompute):
    """recompute: the bf16 step with GELU recomputed in the backward (activation recompute)."""
    wl = fx.WORKLOADS[name]
    sh = wl.shape
    p, tok, tgt = fx.make_inputs(wl)
    grads = {}
    for prec in (0, 1):
        st = U.make_step(sh, wl.B, wl.T, prec, recompute_gelu=recompute and prec == 1)
        try:
            r = U.gpu_train_step(st, p, tok, tgt, wl.lr, wl.wd, wl.clip)
        finally:
            st.close()
        assert np.isfinite(r.grads).all()
        grads[prec] = r
    assert abs(grads[1].loss - grads[0].loss) <= U.BF16_LOSS_ABS
    U.assert_bf16_grads(sh, grads[1].grads, grads[0].grads, f"{name} bf16 vs fp32 path")
    assert abs(grads[1].norm - grads[0].norm) <= 1e-2 * grads[0].norm
