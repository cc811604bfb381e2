"""Gradient accumulation (gpt_train_step_accum) through the C ABI against the oracle's
accumulated step: the loss is the mean over all micro-batch positions, the gradient the mean
of the micro-batch gradients, then one clip and one AdamW update. Also: equality with one step
over the whole batch (fp32), determinism, and n_micro = 1 being gpt_train_step."""
import numpy as np
import pytest

import oracle
from gpt_transformer_step_b200 import fixtures as fx
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

FP32, BF16 = 0, 1


def _gpu_accum(st, p, tok, tgt, lr, wd, clip):
    import torch
    P = U.to_dev(p)
    G = torch.zeros_like(P)
    M = torch.zeros_like(P)
    V = torch.zeros_like(P)
    tk = U.to_dev(tok.astype(np.int32))
    tg = U.to_dev(tgt.astype(np.int32))
    st.use_current_torch_stream()
    loss = st.train_step_accum(P, G, M, V, tk, tg, lr, wd, clip)
    torch.cuda.synchronize()
    return U.GpuRun(loss, G.cpu().numpy(), P.cpu().numpy(), M.cpu().numpy(), V.cpu().numpy(),
                    st.last_grad_norm())


def _inputs(sh, n_micro, B, T, seed, s):
    p = fx.init_params(sh, seed)
    tok, tgt = fx.zipf_tokens(sh.vocab, s, n_micro * B, T, seed)
    return p, tok.reshape(n_micro, B, T), tgt.reshape(n_micro, B, T)


def _oracle_accum(sh, p, tok, tgt, lr, wd, clip):
    o = oracle.Oracle.from_shape(sh)
    pp = p.astype(np.float64)
    m, v = np.zeros_like(pp), np.zeros_like(pp)
    loss, g, n = o.train_step_accum(pp, m, v, tok, tgt, lr, wd, clip, 1)
    return loss, g, n, pp


def test_fp32_accumulated_step_matches_oracle():
    sh = fx.ModelShape(vocab=1000, vocab_padded=1024, n_layer=2, n_head=4, n_embd=128,
                       max_T=80, window_left=[17, -1])
    lr, wd, clip = 1e-3, 0.01, 1.0
    p, tok, tgt = _inputs(sh, 3, 2, 70, seed=6, s=1.1)
    st = U.make_step(sh, 2, 70, FP32)
    try:
        r = _gpu_accum(st, p, tok, tgt, lr, wd, clip)
    finally:
        st.close()
    loss, g, n, pp = _oracle_accum(sh, p, tok, tgt, lr, wd, clip)
    assert abs(r.loss - loss) <= U.FP32_LOSS_ABS, (r.loss, loss)
    for (name, a), (_, b) in zip(U.per_tensor(sh, r.grads), U.per_tensor(sh, g)):
        if np.abs(b).max() == 0:
            assert np.abs(a).max() == 0, name
            continue
        assert U.grad_rel_err(a, b) <= U.FP32_GRAD_REL, (name, U.grad_rel_err(a, b))
    assert abs(r.norm - n) <= 1e-3 * n
    zeros = np.zeros_like(p, dtype=np.float64)
    pe, _, _, _ = U.oracle_adamw_on(r.grads, p, zeros, zeros, lr, wd, clip, 1)
    assert np.abs(r.params - pe).max() <= U.BF16_UPDATE_ABS_PER_LR * lr
    well = np.abs(g) >= 1e-5
    assert np.abs(r.params - pp)[well].max() <= U.BF16_UPDATE_ABS_PER_LR * lr


def test_fp32_two_micro_batches_equal_one_step_over_both():
    """Same rows, same update: 2 micro-batches of B=2 vs one step with B=4 (fp32 mode, so the
    only difference is the summation order of the gradient reductions)."""
    sh = fx.ModelShape(vocab=300, vocab_padded=320, n_layer=2, n_head=2, n_embd=128, max_T=48)
    lr, wd, clip = 1e-3, 0.01, 1.0
    p, tok, tgt = _inputs(sh, 2, 2, 48, seed=7, s=1.1)
    st_a = U.make_step(sh, 2, 48, FP32)
    st_b = U.make_step(sh, 4, 48, FP32)
    try:
        ra = _gpu_accum(st_a, p, tok, tgt, lr, wd, clip)
        rb = U.gpu_train_step(st_b, p, tok.reshape(4, 48), tgt.reshape(4, 48), lr, wd, clip)
    finally:
        st_a.close()
        st_b.close()
    assert abs(ra.loss - rb.loss) <= 1e-5 * abs(rb.loss)
    for (name, a), (_, b) in zip(U.per_tensor(sh, ra.grads), U.per_tensor(sh, rb.grads)):
        if np.abs(b).max() == 0:
            assert np.abs(a).max() == 0, name
            continue
        assert U.grad_rel_err(a, b) <= 1e-4, (name, U.grad_rel_err(a, b))
    assert abs(ra.norm - rb.norm) <= 1e-5 * rb.norm
    # at t = 1 the update is lr*g/(|g|+eps): compared where it is well conditioned, |g| >> eps
    well = np.abs(rb.grads) >= 1e-5
    assert np.abs(ra.params - rb.params)[well].max() <= 1e-3 * lr


def test_bf16_accumulated_step_matches_oracle_and_is_deterministic():
    sh = fx.ModelShape(vocab=777, vocab_padded=784, n_layer=2, n_head=2, n_embd=128,
                       max_T=160, window_left=[40, -1])
    lr, wd, clip = 6e-4, 0.1, 1.0
    p, tok, tgt = _inputs(sh, 3, 2, 150, seed=8, s=1.05)
    st = U.make_step(sh, 2, 150, BF16, lmhead_chunk_rows=96)
    try:
        r1 = _gpu_accum(st, p, tok, tgt, lr, wd, clip)
        st.step = 0
        r2 = _gpu_accum(st, p, tok, tgt, lr, wd, clip)
    finally:
        st.close()
    assert r1.loss == r2.loss and np.array_equal(r1.grads, r2.grads)
    assert np.array_equal(r1.params, r2.params)
    o = oracle.Oracle.from_shape(sh)
    pp = p.astype(np.float64)
    loss, g, _ = o.train_step_accum(pp, np.zeros_like(pp), np.zeros_like(pp), tok, tgt, lr, wd,
                                    clip, 1)
    assert abs(r1.loss - loss) <= U.BF16_LOSS_ABS, (r1.loss, loss)
    for (name, a), (_, b) in zip(U.per_tensor(sh, r1.grads), U.per_tensor(sh, g)):
        if np.abs(b).max() == 0:
            assert np.abs(a).max() == 0, name
            continue
        c = U.cosine(a, b)
        assert c >= U.BF16_GRAD_COS, (name, c)
    zeros = np.zeros_like(p, dtype=np.float64)
    pe, _, _, n = U.oracle_adamw_on(r1.grads, p, zeros, zeros, lr, wd, clip, 1)
    assert abs(r1.norm - n) <= 1e-4 * n
    assert np.abs(r1.params - pe).max() <= U.BF16_UPDATE_ABS_PER_LR * lr


def test_one_micro_batch_is_the_plain_step_bitwise():
    sh = fx.ModelShape(vocab=500, vocab_padded=512, n_layer=1, n_head=2, n_embd=128, max_T=64)
    lr, wd, clip = 6e-4, 0.1, 1.0
    p, tok, tgt = _inputs(sh, 1, 2, 64, seed=9, s=1.05)
    st = U.make_step(sh, 2, 64, BF16)
    try:
        ra = _gpu_accum(st, p, tok, tgt, lr, wd, clip)
        st.step = 0
        rb = U.gpu_train_step(st, p, tok[0], tgt[0], lr, wd, clip)
    finally:
        st.close()
    assert ra.loss == rb.loss
    assert np.array_equal(ra.grads, rb.grads) and np.array_equal(ra.params, rb.params)
