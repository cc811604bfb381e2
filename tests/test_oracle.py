"""Pins for the oracle (CPU only). Each check rests on something other than the oracle
itself: a float64 PyTorch model built from library routines, finite differences, closed
forms, and invariants of the mathematics."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from gpt_transformer_step_b200 import fixtures as fx
from tests import torch_reference as tref

TINY = fx.WORKLOADS["tiny_char_fp32"]


def tiny_inputs(seed=0, B=None, T=None):
    return fx.make_inputs(TINY, seed, B, T)


def rel_max(a, b):
    return float(np.abs(np.asarray(a) - np.asarray(b)).max() / max(np.abs(b).max(), 1e-300))


def per_tensor(sh, arr):
    for name, off, shp, _ in fx.param_layout(sh):
        yield name, arr[off:off + int(np.prod(shp))]


# ---------------------------------------------------------------------------------------
# layout
# ---------------------------------------------------------------------------------------

def test_layout_matches_fixture_and_counts():
    for wl in fx.WORKLOADS.values():
        o = oracle.Oracle.from_shape(wl.shape)
        lay = fx.param_layout(wl.shape)
        assert o.n == fx.num_params(wl.shape)
        assert [(off, int(np.prod(s))) for _, off, s, _ in lay] == o.layout()
    # the counts in the workloads' own descriptions
    assert fx.num_params(fx.WORKLOADS["gpt2_124m_bf16"].shape) == 124_373_760
    assert fx.num_params(fx.WORKLOADS["gpt2_350m_bf16"].shape) == 354_599_936


# ---------------------------------------------------------------------------------------
# whole model vs an independent float64 torch model (library routines)
# ---------------------------------------------------------------------------------------

def _check_vs_torch(sh, p, tok, tgt, tol_loss=1e-10, tol_grad=1e-9):
    o = oracle.Oracle.from_shape(sh)
    loss, g = o.forward_backward(p, tok, tgt)
    tl, tg = tref.loss_and_grad(p, sh, tok, tgt)
    assert abs(loss - tl) <= tol_loss * max(1, abs(tl))
    for (name, a), (_, b) in zip(per_tensor(sh, g), per_tensor(sh, tg)):
        if np.abs(b).max() == 0:
            assert np.abs(a).max() == 0, name
            continue
        assert rel_max(a, b) <= tol_grad, name


def test_tiny_vs_torch_f64():
    p, tok, tgt = tiny_inputs()
    _check_vs_torch(TINY.shape, p, tok, tgt)


def test_tiny_padded_vocab_and_windows_vs_torch():
    sh = fx.ModelShape(vocab=61, vocab_padded=72, n_layer=3, n_head=4, n_embd=32, max_T=20,
                       window_left=[3, -1, 0])
    p = fx.init_params(sh, seed=5)
    tok, tgt = fx.zipf_tokens(sh.vocab, 1.1, 3, 17, seed=5)
    _check_vs_torch(sh, p, tok, tgt)
    # padded rows: zero at init, zero gradient
    o = oracle.Oracle.from_shape(sh)
    _, g = o.forward_backward(p, tok, tgt)
    wte_g = g[: sh.vocab_padded * sh.n_embd].reshape(sh.vocab_padded, sh.n_embd)
    assert np.all(wte_g[sh.vocab:] == 0)
    assert np.all(p[: sh.vocab_padded * sh.n_embd].reshape(sh.vocab_padded, -1)[sh.vocab:] == 0)


def test_shakespeare_shape_vs_torch_f64():
    wl = fx.WORKLOADS["shakespeare_char_bf16"]
    sh = fx.ModelShape(65, 65, 2, 6, 384, 256)  # the Shakespeare widths, 2 layers, short T
    p = fx.init_params(sh)
    tok, tgt = fx.zipf_tokens(65, wl.zipf_s, 2, 24)
    _check_vs_torch(sh, p, tok, tgt)


def test_f32_instantiation_close_to_f64():
    p, tok, tgt = tiny_inputs()
    o64 = oracle.Oracle.from_shape(TINY.shape)
    o32 = oracle.Oracle.from_shape(TINY.shape, dtype=np.float32)
    l64, g64 = o64.forward_backward(p, tok, tgt)
    l32, g32 = o32.forward_backward(p, tok, tgt)
    assert abs(l32 - l64) < 1e-5
    for (n, a), (_, b) in zip(per_tensor(TINY.shape, g32), per_tensor(TINY.shape, g64)):
        assert rel_max(a, b) < 1e-4, n


def test_train_step_vs_torch_adamw_two_steps():
    p, tok, tgt = tiny_inputs()
    sh = TINY.shape
    o = oracle.Oracle.from_shape(sh)
    pp = p.astype(np.float64)
    m = np.zeros_like(pp)
    v = np.zeros_like(pp)
    losses, norms = [], []
    for step in (1, 2):
        loss, g, n = o.train_step(pp, m, v, tok, tgt, TINY.lr, TINY.wd, TINY.clip, step)
        losses.append(loss)
        norms.append(n)
    tl, tg, tn, tp = tref.train_step(p, sh, tok, tgt, TINY.lr, TINY.wd, TINY.clip, steps=2)
    assert np.allclose(losses, tl, rtol=1e-11, atol=0)
    assert np.allclose(norms, tn, rtol=1e-10, atol=0)
    assert np.abs(pp - tp).max() <= 1e-12


def test_clipping_engages_like_torch():
    """A tiny clip value forces coef < 1 in both."""
    p, tok, tgt = tiny_inputs()
    o = oracle.Oracle.from_shape(TINY.shape)
    pp = p.astype(np.float64)
    m, v = np.zeros_like(pp), np.zeros_like(pp)
    _, g, n = o.train_step(pp, m, v, tok, tgt, 1e-3, 0.01, 0.05, 1)
    assert n > 0.05
    _, _, tn, tp = tref.train_step(p, TINY.shape, tok, tgt, 1e-3, 0.01, 0.05, steps=1)
    assert abs(n - tn[0]) < 1e-12 * n
    assert np.abs(pp - tp).max() <= 1e-12
    # m after one step is (1-beta1) * coef * g
    coef = 0.05 / (n + 1e-6)
    assert np.allclose(m, 0.1 * coef * g, rtol=1e-12, atol=1e-300)


# ---------------------------------------------------------------------------------------
# finite differences (double)
# ---------------------------------------------------------------------------------------

def test_finite_differences_every_tensor():
    sh = fx.ModelShape(vocab=23, vocab_padded=24, n_layer=2, n_head=2, n_embd=16, max_T=8,
                       window_left=[2, -1])
    p = fx.init_params(sh, seed=3).astype(np.float64)
    # larger weights so that every path carries signal
    p *= 10.0
    for name, off, shp, s in fx.param_layout(sh):
        if s == 0.0:
            n = int(np.prod(shp))
            p[off:off + n] = 1.0 + 0.3 * fx.normals(fx.stream_key(off, "misc"), n)
    tok, tgt = fx.zipf_tokens(sh.vocab, 1.1, 2, 7, seed=3)
    o = oracle.Oracle.from_shape(sh)
    _, g = o.forward_backward(p, tok, tgt)
    rng = np.random.default_rng(0)
    h = 1e-5
    for name, off, shp, _ in fx.param_layout(sh):
        n = int(np.prod(shp))
        gt = g[off:off + n]
        scale = max(np.abs(gt).max(), 1e-12)
        if name == "wte":
            # padded row excluded from the softmax: zero gradient
            idx = list(rng.choice(sh.vocab * sh.n_embd, 6, replace=False))
        else:
            idx = list(rng.choice(n, min(n, 6), replace=False))
        idx.append(int(np.abs(gt).argmax()))
        for i in idx:
            pp = p.copy(); pp[off + i] += h
            pm = p.copy(); pm[off + i] -= h
            fd = (o.forward(pp, tok, tgt) - o.forward(pm, tok, tgt)) / (2 * h)
            assert abs(fd - gt[i]) <= 1e-6 * scale + 1e-9, (name, i, fd, gt[i])


# ---------------------------------------------------------------------------------------
# closed forms and invariants
# ---------------------------------------------------------------------------------------

def test_initial_loss_is_about_ln_vocab():
    p, tok, tgt = tiny_inputs()
    o = oracle.Oracle.from_shape(TINY.shape)
    loss = o.forward(p, tok, tgt)
    assert abs(loss - math.log(TINY.shape.vocab)) < 0.1


def test_zero_wte_gives_exactly_ln_vocab_not_ln_padded():
    sh = fx.ModelShape(vocab=50, vocab_padded=64, n_layer=1, n_head=2, n_embd=16, max_T=8)
    p = fx.init_params(sh, seed=1).astype(np.float64)
    p[: sh.vocab_padded * sh.n_embd] = 0.0
    tok, tgt = fx.zipf_tokens(sh.vocab, 1.1, 2, 8, seed=1)
    o = oracle.Oracle.from_shape(sh)
    loss = o.forward(p, tok, tgt)
    assert abs(loss - math.log(50)) < 1e-13
    assert abs(loss - math.log(64)) > 0.1


def test_causality_bitwise():
    p, tok, tgt = tiny_inputs()
    for dt in (np.float64, np.float32):
        o = oracle.Oracle.from_shape(TINY.shape, dtype=dt)
        _, base = o.forward(p, tok, tgt, per_token=True)
        for t in (0, 5, 30):
            tok2 = tok.copy()
            tok2[:, t + 1] = (tok2[:, t + 1] + 7) % TINY.shape.vocab
            _, pert = o.forward(p, tok2, tgt, per_token=True)
            assert np.array_equal(base[:, : t + 1], pert[:, : t + 1])
            assert not np.array_equal(base[:, t + 1:], pert[:, t + 1:])


def test_adamw_step1_closed_form():
    rng = np.random.default_rng(0)
    n = 1000
    p0 = rng.standard_normal(n)
    g = rng.standard_normal(n) * 10.0 ** rng.uniform(-9, 1, n)
    o = oracle.Oracle.from_shape(TINY.shape)
    lr, wd, eps = 1e-3, 0.1, 1e-8
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    o.adamw(p, g, m, v, lr, wd, 1, coef=1.0, eps=eps)
    # t=1: mhat = g, vhat = g^2 -> dp = -lr*wd*p - lr*g/(|g|+eps)
    expect = p0 * (1 - lr * wd) - lr * g / (np.abs(g) + eps)
    assert np.allclose(p, expect, rtol=1e-14, atol=1e-18)
    assert np.allclose(m, 0.1 * g, rtol=1e-15, atol=0)
    assert np.allclose(v, 0.05 * g * g, rtol=1e-14, atol=0)
    # |step| ~ lr where |g| >> eps
    big = np.abs(g) > 1e-4
    assert np.allclose(np.abs(p - p0 * (1 - lr * wd))[big], lr, rtol=1e-4)


def test_adamw_zero_grad_is_pure_decay_and_matches_torch_later_steps():
    rng = np.random.default_rng(1)
    n = 257
    p0 = rng.standard_normal(n)
    o = oracle.Oracle.from_shape(TINY.shape)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    o.adamw(p, np.zeros(n), m, v, 1e-2, 0.1, 1)
    assert np.array_equal(p, p0 * (1 - 1e-2 * 0.1))
    # three steps with changing grads vs torch.optim.AdamW
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    tp = torch.tensor(p0, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=3e-3, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.05)
    for t in (1, 2, 3):
        g = rng.standard_normal(n)
        o.adamw(p, g, m, v, 3e-3, 0.05, t)
        tp.grad = torch.tensor(g)
        opt.step()
    assert np.abs(p - tp.detach().numpy()).max() < 1e-14


def test_grad_norm_and_clip_rules():
    rng = np.random.default_rng(2)
    g = rng.standard_normal(10000)
    o = oracle.Oracle.from_shape(TINY.shape)
    n = o.grad_norm(g)
    assert abs(n - np.linalg.norm(g)) < 1e-12 * n
    assert abs(o.grad_norm(3.0 * g) - 3.0 * n) < 1e-12 * n
    # clip >= norm -> coef 1: the step equals an unclipped AdamW step
    p, tok, tgt = tiny_inputs()
    pp = p.astype(np.float64)
    m, v = np.zeros_like(pp), np.zeros_like(pp)
    _, graw, gn = o.train_step(pp, m, v, tok, tgt, 1e-3, 0.0, 1e9, 1)
    p2, m2, v2 = p.astype(np.float64), np.zeros_like(pp), np.zeros_like(pp)
    o.adamw(p2, graw, m2, v2, 1e-3, 0.0, 1, coef=1.0)
    assert np.array_equal(pp, p2)


def test_layernorm_invariants():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((7, 48)) * 3 + 1
    gam = np.ones(48)
    o = oracle.Oracle.from_shape(TINY.shape)
    y, mu, rs = o.layernorm_fwd(x, gam)
    assert np.allclose(y.mean(1), 0, atol=1e-14)
    assert np.allclose(y.var(1), 1 / (1 + 1e-5 * rs ** 2), rtol=1e-12)  # var/(var+eps)
    tl = F.layer_norm(torch.tensor(x), (48,), eps=1e-5).numpy()
    assert np.abs(y - tl).max() < 1e-13
    g2 = rng.standard_normal(48)
    dy = rng.standard_normal((7, 48))
    dx, dg = o.layernorm_bwd(x, g2, mu, rs, dy)
    assert np.allclose(dx.sum(1), 0, atol=1e-12)
    # sum(dx * xhat) = 0 holds exactly when eps = 0 (xhat then has unit mean square)
    _, mu0, rs0 = o.layernorm_fwd(x, gam, eps=0.0)
    dx0, _ = o.layernorm_bwd(x, g2, mu0, rs0, dy)
    xhat0 = (x - mu0[:, None]) * rs0[:, None]
    assert np.allclose((dx0 * xhat0).sum(1), 0, atol=1e-12)
    xt = torch.tensor(x, requires_grad=True)
    gt = torch.tensor(g2, requires_grad=True)
    F.layer_norm(xt, (48,), weight=gt, eps=1e-5).backward(torch.tensor(dy))
    assert np.abs(dx - xt.grad.numpy()).max() < 1e-12
    assert np.abs(dg - gt.grad.numpy()).max() < 1e-12


def test_gelu_tanh_matches_torch_and_autograd():
    o = oracle.Oracle.from_shape(TINY.shape)
    xs = np.linspace(-8, 8, 401)
    t = torch.tensor(xs, requires_grad=True)
    y = F.gelu(t, approximate="tanh")
    y.sum().backward()
    got = np.array([o.gelu(x) for x in xs])
    dgot = np.array([o.gelu_grad(x) for x in xs])
    assert np.abs(got - y.detach().numpy()).max() < 1e-14
    assert np.abs(dgot - t.grad.numpy()).max() < 1e-13


def test_cross_entropy_grad_rows_sum_to_zero_and_padding():
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((9, 40)) * 4
    tg = rng.integers(0, 33, 9)
    o = oracle.Oracle.from_shape(TINY.shape)
    loss, d = o.cross_entropy(lg, tg, V=33)
    assert np.allclose(d.sum(1), 0, atol=1e-15)
    assert np.all(d[:, 33:] == 0)
    tl = F.cross_entropy(torch.tensor(lg[:, :33]), torch.tensor(tg)).item()
    assert abs(loss - tl) < 1e-13


def test_window_special_cases():
    rng = np.random.default_rng(5)
    B, T, C, H = 2, 8, 16, 2
    qkv = rng.standard_normal((B, T, 3 * C))
    o = oracle.Oracle.from_shape(TINY.shape)
    full = o.attention_fwd(qkv, H, -1)
    assert np.array_equal(o.attention_fwd(qkv, H, T), full)
    assert np.array_equal(o.attention_fwd(qkv, H, T - 1), full)
    # w = 0: each query sees only itself -> o_i = v_i exactly
    assert np.array_equal(o.attention_fwd(qkv, H, 0), qkv[:, :, 2 * C:])
    # T = 1: output = v
    assert np.array_equal(o.attention_fwd(qkv[:, :1], H, -1), qkv[:, :1, 2 * C:])
    # brute-force mask enumeration vs torch SDPA for every window 0..T
    for w in range(0, T + 1):
        mask = np.array([[(j <= i and j >= i - w) for j in range(T)] for i in range(T)])
        q, k, v = (torch.tensor(a).view(B, T, H, C // H).transpose(1, 2)
                   for a in np.split(qkv, 3, axis=-1))
        ref = F.scaled_dot_product_attention(q, k, v, attn_mask=torch.tensor(mask))
        ref = ref.transpose(1, 2).reshape(B, T, C).numpy()
        assert np.abs(o.attention_fwd(qkv, H, w) - ref).max() < 1e-13, w
        # backward vs autograd through SDPA
        qt, kt, vt = (torch.tensor(a).view(B, T, H, C // H).transpose(1, 2).requires_grad_()
                      for a in np.split(qkv, 3, axis=-1))
        dout = rng.standard_normal((B, T, C))
        y = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.tensor(mask))
        y.transpose(1, 2).reshape(B, T, C).backward(torch.tensor(dout))
        tg = np.concatenate([a.grad.transpose(1, 2).reshape(B, T, C).numpy()
                             for a in (qt, kt, vt)], -1)
        assert np.abs(o.attention_bwd(qkv, dout, H, w) - tg).max() < 1e-12, w


# ---------------------------------------------------------------------------------------
# gradient accumulation
# ---------------------------------------------------------------------------------------

def test_accumulated_step_equals_one_step_over_the_whole_batch():
    """The loss of an accumulated step is the mean over all n_micro*B*T positions, so two
    micro-batches of B=2 must give the loss, gradients and update of one B=4 step over the
    same rows (that step is pinned to the torch float64 model above)."""
    p, tok, tgt = tiny_inputs(seed=3, B=4)
    sh = TINY.shape
    o = oracle.Oracle.from_shape(sh)
    pa, pb = p.astype(np.float64), p.astype(np.float64)
    ma, va = np.zeros_like(pa), np.zeros_like(pa)
    mb, vb = np.zeros_like(pb), np.zeros_like(pb)
    la, ga, na = o.train_step_accum(pa, ma, va, tok.reshape(2, 2, -1), tgt.reshape(2, 2, -1),
                                    TINY.lr, TINY.wd, TINY.clip, 1)
    lb, gb, nb = o.train_step(pb, mb, vb, tok, tgt, TINY.lr, TINY.wd, TINY.clip, 1)
    assert abs(la - lb) <= 1e-13 * abs(lb)
    assert rel_max(ga, gb) <= 1e-12
    assert abs(na - nb) <= 1e-12 * nb
    for a, b in ((pa, pb), (ma, mb), (va, vb)):
        assert np.abs(a - b).max() <= 1e-13


def test_accumulated_step_with_one_micro_batch_is_the_plain_step():
    p, tok, tgt = tiny_inputs(seed=4)
    o = oracle.Oracle.from_shape(TINY.shape)
    pa, pb = p.astype(np.float64), p.astype(np.float64)
    za, zb = [np.zeros_like(pa) for _ in range(2)], [np.zeros_like(pb) for _ in range(2)]
    la, ga, _ = o.train_step_accum(pa, *za, tok[None], tgt[None], TINY.lr, TINY.wd, TINY.clip, 1)
    lb, gb, _ = o.train_step(pb, *zb, tok, tgt, TINY.lr, TINY.wd, TINY.clip, 1)
    assert la == lb and np.array_equal(ga, gb) and np.array_equal(pa, pb)


def test_accumulated_gradient_is_the_mean_of_micro_batch_gradients():
    """Linearity: with unequal micro-batch contents the accumulated gradient is the plain
    average of the per-micro-batch gradients (not their sum, not a token-weighted sum)."""
    p, tok, tgt = tiny_inputs(seed=5, B=6)
    o = oracle.Oracle.from_shape(TINY.shape)
    parts = [o.forward_backward(p, tok[2 * i:2 * i + 2], tgt[2 * i:2 * i + 2]) for i in range(3)]
    pa = p.astype(np.float64)
    la, ga, _ = o.train_step_accum(pa, np.zeros_like(pa), np.zeros_like(pa),
                                   tok.reshape(3, 2, -1), tgt.reshape(3, 2, -1), TINY.lr,
                                   TINY.wd, TINY.clip, 1)
    assert abs(la - sum(l for l, _ in parts) / 3) <= 1e-13 * abs(la)
    assert rel_max(ga, sum(g for _, g in parts) / 3) <= 1e-13
