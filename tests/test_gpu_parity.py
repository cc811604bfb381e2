"""Parity of the CUDA path (through the C ABI) with the oracle on the same seeded inputs.

Sizes the oracle finishes in seconds, spanning several tiles with ragged tails, in both the
fp32 validation mode and bf16 mode; the full GPT-2 124M configuration is checked on sampled
outputs (causal prefixes the oracle can compute) and on properties that hold at any size.
"""
import math

import numpy as np
import pytest

import oracle
from gpt_transformer_step_b200 import fixtures as fx
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

FP32, BF16 = 0, 1


def _oracle_step(sh, p, tok, tgt, lr, wd, clip):
    o = oracle.Oracle.from_shape(sh)
    pp = p.astype(np.float64)
    m, v = np.zeros_like(pp), np.zeros_like(pp)
    loss, g, n = o.train_step(pp, m, v, tok, tgt, lr, wd, clip, 1)
    return loss, g, n, pp, m, v


def check_fp32(sh, B, T, seed=0, lr=1e-3, wd=0.01, clip=1.0, s=1.1):
    p = fx.init_params(sh, seed)
    tok, tgt = fx.zipf_tokens(sh.vocab, s, B, T, seed)
    st = U.make_step(sh, B, T, FP32)
    r = U.gpu_train_step(st, p, tok, tgt, lr, wd, clip)
    loss, g, n, pp, m, v = _oracle_step(sh, p, tok, tgt, lr, wd, clip)
    assert abs(r.loss - loss) <= U.FP32_LOSS_ABS, (r.loss, loss)
    for (name, a), (_, b) in zip(U.per_tensor(sh, r.grads), U.per_tensor(sh, g)):
        if np.abs(b).max() == 0:
            assert np.abs(a).max() == 0, name
            continue
        assert U.grad_rel_err(a, b) <= U.FP32_GRAD_REL, (name, U.grad_rel_err(a, b))
    assert abs(r.norm - n) <= 1e-3 * n
    # AdamW given the same gradients
    zeros = np.zeros_like(p, dtype=np.float64)
    pe, _, _, _ = U.oracle_adamw_on(r.grads, p, zeros, zeros, lr, wd, clip, 1)
    assert np.abs(r.params - pe).max() <= U.BF16_UPDATE_ABS_PER_LR * lr
    # end to end: at t=1 the update is lr*g/(|g|+eps), well conditioned where |g| >> eps
    well = np.abs(g) >= 1e-5
    assert np.abs(r.params - pp)[well].max() <= U.BF16_UPDATE_ABS_PER_LR * lr
    st.close()


def check_bf16(sh, B, T, seed=0, lr=6e-4, wd=0.1, clip=1.0, s=1.05, **kw):
    p = fx.init_params(sh, seed)
    tok, tgt = fx.zipf_tokens(sh.vocab, s, B, T, seed)
    st = U.make_step(sh, B, T, BF16, **kw)
    r = U.gpu_train_step(st, p, tok, tgt, lr, wd, clip)
    o = oracle.Oracle.from_shape(sh)
    loss, g = o.forward_backward(p, tok, tgt)
    assert abs(r.loss - loss) <= U.BF16_LOSS_ABS, (r.loss, loss)
    for (name, a), (_, b) in zip(U.per_tensor(sh, r.grads), U.per_tensor(sh, g)):
        if np.abs(b).max() == 0:
            assert np.abs(a).max() == 0, name
            continue
        c = U.cosine(a, b)
        assert c >= U.BF16_GRAD_COS, (name, c)
    # AdamW given the same gradients
    zeros = np.zeros_like(p, dtype=np.float64)
    pe, me, ve, n = U.oracle_adamw_on(r.grads, p, zeros, zeros, lr, wd, clip, 1)
    assert abs(r.norm - n) <= 1e-4 * n
    assert np.abs(r.params - pe).max() <= U.BF16_UPDATE_ABS_PER_LR * lr
    assert np.abs(r.m - me).max() <= 1e-6 * max(np.abs(me).max(), 1e-30) + 1e-12
    st.close()
    return r


# ---------------------------------------------------------------------------------------
# fp32 validation mode
# ---------------------------------------------------------------------------------------

def test_tiny_char_fp32_workload():
    wl = fx.WORKLOADS["tiny_char_fp32"]
    check_fp32(wl.shape, wl.B, wl.T, lr=wl.lr, wd=wl.wd, clip=wl.clip, s=wl.zipf_s)


def test_fp32_ragged_tiles_and_windows():
    sh = fx.ModelShape(vocab=1000, vocab_padded=1024, n_layer=2, n_head=4, n_embd=128,
                       max_T=80, window_left=[17, -1])
    check_fp32(sh, B=3, T=70, seed=1)


def test_fp32_head_dim_64_and_clip_engaged():
    sh = fx.ModelShape(vocab=300, vocab_padded=320, n_layer=1, n_head=2, n_embd=128, max_T=40)
    check_fp32(sh, B=2, T=37, seed=2, clip=1e-3)


# ---------------------------------------------------------------------------------------
# bf16 mode
# ---------------------------------------------------------------------------------------

def test_bf16_ragged_tiles():
    sh = fx.ModelShape(vocab=1000, vocab_padded=1024, n_layer=2, n_head=4, n_embd=256,
                       max_T=200)
    check_bf16(sh, B=3, T=200, seed=3)


def test_bf16_ragged_tiles_window_and_chunked_lmhead():
    sh = fx.ModelShape(vocab=777, vocab_padded=784, n_layer=2, n_head=2, n_embd=128,
                       max_T=160, window_left=[40, -1])
    check_bf16(sh, B=2, T=150, seed=4, lmhead_chunk_rows=96)


def test_bf16_shakespeare_shape():
    wl = fx.WORKLOADS["shakespeare_char_bf16"]
    check_bf16(wl.shape, B=1, T=128, lr=wl.lr, wd=wl.wd, s=wl.zipf_s)


# ---------------------------------------------------------------------------------------
# full GPT-2 124M: sampled outputs + properties
# ---------------------------------------------------------------------------------------

@pytest.fixture(scope="module")
def gpt2():
    wl = fx.WORKLOADS["gpt2_124m_bf16"]
    p, tok, tgt = fx.make_inputs(wl)
    st = U.make_step(wl.shape, wl.B, wl.T, BF16)
    yield wl, p, tok, tgt, st
    st.close()


def test_gpt2_124m_forward_prefixes_match_oracle(gpt2):
    wl, p, tok, tgt, st = gpt2
    loss, ptl = U.gpu_forward(st, p, tok, tgt)
    assert abs(loss - math.log(wl.shape.vocab)) < 0.25
    o = oracle.Oracle.from_shape(wl.shape, dtype=np.float32)
    P = 24  # causal prefix the oracle recomputes: positions < P depend only on tokens < P
    rows = (0, wl.B - 1)
    refs = [o.forward(p, tok[b:b + 1, :P], tgt[b:b + 1, :P], per_token=True)[1][0] for b in rows]
    # the loss bound is about the mean over all B*T tokens: the fp32 validation path matches
    # the oracle token by token on the prefixes, and the bf16 loss matches the fp32 loss over
    # the full batch; single bf16 prefix tokens carry bf16 noise and are bounded directly
    st32 = U.make_step(wl.shape, wl.B, wl.T, 0)
    try:
        loss32, ptl32 = U.gpu_forward(st32, p, tok, tgt)
    finally:
        st32.close()
    for b, ref in zip(rows, refs):
        assert np.abs(ptl32[b, :P] - ref).max() <= U.FP32_LOSS_ABS
    assert abs(loss - loss32) <= U.BF16_LOSS_ABS, (loss, loss32)
    d = np.concatenate([ptl[b, :P] - ref for b, ref in zip(rows, refs)])
    assert np.abs(d).max() <= 10 * U.BF16_LOSS_ABS, np.abs(d).max()


def test_gpt2_124m_train_step_update_and_determinism(gpt2):
    wl, p, tok, tgt, st = gpt2
    r1 = U.gpu_train_step(st, p, tok, tgt, wl.lr, wl.wd, wl.clip)
    st.step = 0
    r2 = U.gpu_train_step(st, p, tok, tgt, wl.lr, wl.wd, wl.clip)
    assert np.array_equal(r1.grads, r2.grads) and np.array_equal(r1.params, r2.params)
    assert r1.loss == r2.loss
    assert np.isfinite(r1.grads).all()
    zeros = np.zeros_like(p, dtype=np.float64)
    pe, _, _, n = U.oracle_adamw_on(r1.grads, p, zeros, zeros, wl.lr, wl.wd, wl.clip, 1)
    assert abs(r1.norm - n) <= 1e-4 * n
    assert np.abs(r1.params - pe).max() <= U.BF16_UPDATE_ABS_PER_LR * wl.lr
    # padded vocab rows: zero gradient, only weight decay moves them (0 stays 0)
    V, Vp, C = wl.shape.vocab, wl.shape.vocab_padded, wl.shape.n_embd
    assert np.all(r1.grads[V * C:Vp * C] == 0)
    assert np.all(r1.params[V * C:Vp * C] == 0)
    st.step = 0


def test_gpt2_124m_causality_bitwise(gpt2):
    wl, p, tok, tgt, st = gpt2
    _, base = U.gpu_forward(st, p, tok, tgt)
    t = 500
    tok2 = tok.copy()
    tok2[:, t + 1] = (tok2[:, t + 1] + 12345) % wl.shape.vocab
    _, pert = U.gpu_forward(st, p, tok2, tgt)
    assert np.array_equal(base[:, :t + 1], pert[:, :t + 1])
    assert not np.array_equal(base[:, t + 1:], pert[:, t + 1:])


# ---------------------------------------------------------------------------------------
# activation recompute (GELU recomputed in the backward from the kept pre-activation)
# ---------------------------------------------------------------------------------------

def test_gelu_recompute_fp32_is_bitwise_the_stored_path():
    """In fp32 mode the recomputed GELU and derivative are the very values the stored path
    keeps, so the whole step is bitwise identical."""
    sh = fx.ModelShape(vocab=1000, vocab_padded=1024, n_layer=2, n_head=4, n_embd=128,
                       max_T=80, window_left=[17, -1])
    p = fx.init_params(sh, 21)
    tok, tgt = fx.zipf_tokens(sh.vocab, 1.1, 3, 70, 21)
    runs = []
    for rc in (False, True):
        st = U.make_step(sh, 3, 70, FP32, recompute_gelu=rc)
        runs.append(U.gpu_train_step(st, p, tok, tgt, 1e-3, 0.01, 1.0))
        st.close()
    a, b = runs
    assert a.loss == b.loss and np.array_equal(a.grads, b.grads)
    assert np.array_equal(a.params, b.params)


def test_gelu_recompute_bf16_matches_oracle():
    sh = fx.ModelShape(vocab=1000, vocab_padded=1024, n_layer=3, n_head=4, n_embd=256,
                       max_T=200, window_left=[50, -1, 7])
    r1 = check_bf16(sh, B=3, T=200, seed=22, recompute_gelu=True)
    st = U.make_step(sh, 3, 200, BF16, recompute_gelu=True)
    tok, tgt = fx.zipf_tokens(sh.vocab, 1.05, 3, 200, 22)
    r2 = U.gpu_train_step(st, fx.init_params(sh, 22), tok, tgt, 6e-4, 0.1, 1.0)
    st.close()
    assert r1.loss == r2.loss and np.array_equal(r1.grads, r2.grads)  # deterministic
