"""Helpers for the GPU parity tests: run the CUDA library through its C ABI and the oracle
on the same seeded inputs, and compare with the stated tolerances."""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from gpt_transformer_step_b200 import fixtures as fx

# Tolerances (spec contract)
FP32_LOSS_ABS = 1e-4       # |loss_gpu - loss_oracle|
FP32_GRAD_REL = 1e-3       # per tensor max|dg| / max|g_oracle|
BF16_LOSS_ABS = 5e-3
BF16_GRAD_COS = 0.999      # per tensor cosine
BF16_UPDATE_ABS_PER_LR = 2e-2  # AdamW given the same grads: max|dp| <= 2e-2 * lr


def torch_dev():
    import torch
    return torch.device("cuda", 0)


@dataclass
class GpuRun:
    loss: float
    grads: np.ndarray
    params: np.ndarray
    m: np.ndarray
    v: np.ndarray
    norm: float


def to_dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(torch_dev())


def make_step(sh: fx.ModelShape, B: int, T: int, precision: int, **kw):
    from gpt_transformer_step_b200 import binding as gb
    return gb.GPTStep(sh.vocab, sh.vocab_padded, sh.n_layer, sh.n_head, sh.n_embd, sh.max_T, B,
                      sh.mlp_mult, sh.windows(), precision, **kw)


def gpu_train_step(step, params_np, tok, tgt, lr, wd, clip, m_np=None, v_np=None) -> GpuRun:
    import torch
    p = to_dev(params_np)
    g = torch.zeros_like(p)
    m = to_dev(m_np) if m_np is not None else torch.zeros_like(p)
    v = to_dev(v_np) if v_np is not None else torch.zeros_like(p)
    tk = to_dev(tok.astype(np.int32))
    tg = to_dev(tgt.astype(np.int32))
    step.use_current_torch_stream()
    loss = step.train_step(p, g, m, v, tk, tg, lr, wd, clip)
    torch.cuda.synchronize()
    return GpuRun(loss, g.cpu().numpy(), p.cpu().numpy(), m.cpu().numpy(), v.cpu().numpy(),
                  step.last_grad_norm())


def gpu_forward(step, params_np, tok, tgt):
    import torch
    p = to_dev(params_np)
    tk = to_dev(tok.astype(np.int32))
    tg = to_dev(tgt.astype(np.int32))
    ptl = torch.zeros(tok.shape, dtype=torch.float32, device=torch_dev())
    step.use_current_torch_stream()
    loss = step.forward_loss(p, tk, tg, ptl)
    torch.cuda.synchronize()
    return loss, ptl.cpu().numpy()


def per_tensor(sh, arr):
    for name, off, shp, _ in fx.param_layout(sh):
        yield name, arr[off:off + int(np.prod(shp))]


def grad_rel_err(a, b):
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-30))


def cosine(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(a @ b / (na * nb))


def oracle_adamw_on(grads, params0, m0, v0, lr, wd, clip, step, beta1=0.9, beta2=0.95, eps=1e-8):
    """The oracle's AdamW applied to the GPU's raw gradients (double)."""
    import oracle
    o = oracle.Oracle(1, 1, 1, 1, 1, 1)  # the AdamW/norm entry points take no model shape
    g = np.asarray(grads, np.float64)
    n = o.grad_norm(g)
    coef = min(1.0, clip / (n + 1e-6))
    p = np.asarray(params0, np.float64).copy()
    m = np.asarray(m0, np.float64).copy()
    v = np.asarray(v0, np.float64).copy()
    o.adamw(p, g, m, v, lr, wd, step, coef=coef, beta1=beta1, beta2=beta2, eps=eps)
    return p, m, v, n


def grad_report(sh, g_test, g_ref):
    """Per tensor (name, cosine, max|dg| / max|g_ref|) of two flat gradient vectors."""
    out = []
    for (name, a), (_, b) in zip(per_tensor(sh, g_test), per_tensor(sh, g_ref)):
        out.append((name, cosine(a, b), grad_rel_err(a, b) if np.abs(b).max() > 0 else 0.0))
    return out


def assert_bf16_grads(sh, g_test, g_ref, what=""):
    """North-star bf16 gradient bound: cosine >= 0.999 per tensor (tensors whose reference is
    exactly zero must be exactly zero). Prints the per-tensor figures."""
    rep = grad_report(sh, g_test, g_ref)
    worst = min(rep, key=lambda r: r[1])
    print(f"\n[{what}] worst cosine {worst[1]:.6f} ({worst[0]}); max rel err "
          f"{max(r[2] for r in rep):.3e}")
    for (name, a), (_, b) in zip(per_tensor(sh, g_test), per_tensor(sh, g_ref)):
        if np.abs(b).max() == 0:
            assert np.abs(a).max() == 0, name
    bad = [(n, c, r) for n, c, r in rep if c < BF16_GRAD_COS]
    assert not bad, bad
    return rep
