"""Independent float64 PyTorch-CPU model of the step, built from library routines
(F.layer_norm, F.scaled_dot_product_attention, F.gelu(approximate="tanh"),
F.cross_entropy, autograd, clip_grad_norm_, torch.optim.AdamW). It pins the oracle: the two
share no code, and a mistake in either shows up as a mismatch.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

from gpt_transformer_step_b200 import fixtures as fx


def _views(flat: torch.Tensor, sh: fx.ModelShape):
    out = {}
    for name, off, shp, _ in fx.param_layout(sh):
        n = int(np.prod(shp))
        out[name] = flat[off:off + n].view(*shp)
    return out


def forward(flat: torch.Tensor, sh: fx.ModelShape, tok, tgt, eps=1e-5, per_token=False):
    P = _views(flat, sh)
    tok = torch.as_tensor(np.asarray(tok), dtype=torch.long)
    tgt = torch.as_tensor(np.asarray(tgt), dtype=torch.long)
    B, T = tok.shape
    C, H = sh.n_embd, sh.n_head
    hd = C // H
    x = P["wte"][tok] + P["wpe"][:T].unsqueeze(0)
    i = torch.arange(T).view(T, 1)
    j = torch.arange(T).view(1, T)
    for l, w in enumerate(sh.windows()):
        a = F.layer_norm(x, (C,), weight=P[f"h{l}.ln1.g"], bias=None, eps=eps)
        qkv = a @ P[f"h{l}.w_qkv"].T
        q, k, v = qkv.split(C, dim=-1)
        q = q.view(B, T, H, hd).transpose(1, 2)
        k = k.view(B, T, H, hd).transpose(1, 2)
        v = v.view(B, T, H, hd).transpose(1, 2)
        mask = j <= i
        if w >= 0:
            mask = mask & (j >= i - w)
        y = F.scaled_dot_product_attention(q, k, v, attn_mask=mask)
        y = y.transpose(1, 2).reshape(B, T, C)
        x = x + y @ P[f"h{l}.w_attnproj"].T
        c = F.layer_norm(x, (C,), weight=P[f"h{l}.ln2.g"], bias=None, eps=eps)
        x = x + F.gelu(c @ P[f"h{l}.w_fc"].T, approximate="tanh") @ P[f"h{l}.w_mlpproj"].T
    yf = F.layer_norm(x, (C,), weight=P["lnf.g"], bias=None, eps=eps)
    logits = yf @ P["wte"][:sh.vocab].T
    if per_token:
        return F.cross_entropy(logits.reshape(-1, sh.vocab), tgt.reshape(-1),
                               reduction="none").view(B, T)
    return F.cross_entropy(logits.reshape(-1, sh.vocab), tgt.reshape(-1))


def loss_and_grad(params: np.ndarray, sh, tok, tgt, eps=1e-5):
    flat = torch.tensor(np.asarray(params, np.float64), requires_grad=True)
    loss = forward(flat, sh, tok, tgt, eps)
    loss.backward()
    return float(loss.detach()), flat.grad.numpy().copy()


def train_step(params, sh, tok, tgt, lr, wd, clip, steps=1, betas=(0.9, 0.95), eps=1e-8):
    """`steps` AdamW steps on the same batch; returns (losses, grads of the last step,
    norms, params after)."""
    flat = torch.tensor(np.asarray(params, np.float64), requires_grad=True)
    opt = torch.optim.AdamW([flat], lr=lr, betas=betas, eps=eps, weight_decay=wd)
    losses, norms, g = [], [], None
    for _ in range(steps):
        opt.zero_grad()
        loss = forward(flat, sh, tok, tgt)
        loss.backward()
        g = flat.grad.numpy().copy()
        n = torch.nn.utils.clip_grad_norm_([flat], clip)
        opt.step()
        losses.append(float(loss.detach()))
        norms.append(float(n))
    return losses, g, norms, flat.detach().numpy().copy()
