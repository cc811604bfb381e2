"""Attention kernels (tensor-core and CUDA-core paths) through the kernel-level C ABI vs
PyTorch's scaled_dot_product_attention in fp32 on the same bf16 inputs: causal and windowed
masks, ragged T (not a multiple of the 128-row tile), forward and backward. Path 2 is the
tensor-core backward as the step runs it (dK/dV writing dS^T, then dQ from the stored dS^T);
it needs T % 8 == 0."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    from gpt_transformer_step_b200 import binding as gb
    torch.backends.cuda.matmul.allow_tf32 = False
    dev = torch.device("cuda", 0)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    return torch, gb, dev, err


def _ref(torch, qkv, B, T, C, H, w, dout):
    F = torch.nn.functional
    hd = C // H
    x = qkv.float().view(B, T, 3, H, hd).permute(2, 0, 3, 1, 4)  # 3, B, H, T, hd
    q, k, v = (t.detach().clone().requires_grad_() for t in x)
    i = torch.arange(T, device=qkv.device).view(T, 1)
    j = torch.arange(T, device=qkv.device).view(1, T)
    mask = j <= i
    if w >= 0:
        mask = mask & (j >= i - w)
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask)
    s = (q @ k.transpose(-1, -2)) / math.sqrt(hd)
    s = s.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(s, dim=-1)  # B, H, T
    o.backward(dout.float().view(B, T, H, hd).transpose(1, 2))
    dqkv = torch.stack([q.grad, k.grad, v.grad]).permute(1, 3, 0, 2, 4).reshape(B * T, 3 * C)
    return o.transpose(1, 2).reshape(B * T, C), lse, dqkv


CASES = [  # B, T, H, window
    (2, 256, 2, -1),
    (1, 200, 3, -1),
    (2, 384, 2, 100),
    (1, 300, 1, 0),
    (1, 1024, 2, 512),
    (3, 77, 2, -1),
]


@pytest.mark.parametrize("path", [0, 1, 2])
@pytest.mark.parametrize("B,T,H,w", CASES)
def test_attention_vs_sdpa(env, path, B, T, H, w):
    torch, gb, dev, err = env
    if path == 2 and T % 8:
        pytest.skip("the stored-dS backward needs T % 8 == 0 (the step falls back otherwise)")
    C = 64 * H
    g = torch.Generator(device="cpu").manual_seed(B * 1000 + T + H + w)
    qkv = (torch.randn(B * T, 3 * C, generator=g) * 1.5).to(torch.bfloat16).to(dev)
    dout = torch.randn(B * T, C, generator=g).to(torch.bfloat16).to(dev)
    o = torch.zeros(B * T, C, dtype=torch.bfloat16, device=dev)
    lse = torch.zeros(B, H, T, device=dev)
    dq = torch.zeros(B * T, 3 * C, dtype=torch.bfloat16, device=dev)
    Dbuf = torch.zeros(B, H, T, device=dev)
    err.zero_()
    s = torch.cuda.current_stream().cuda_stream
    fpath = 0 if path == 2 else path
    assert gb.gptk_attention_fwd_bf16(qkv.data_ptr(), o.data_ptr(), lse.data_ptr(), B, T, C, H, w,
                                      err.data_ptr(), fpath, s) == 0
    if path == 2:
        ds = torch.full((B * H * T * T,), float("nan"), dtype=torch.bfloat16, device=dev)
        assert gb.gptk_attention_bwd_bf16_ds(qkv.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                             lse.data_ptr(), Dbuf.data_ptr(), ds.data_ptr(),
                                             dq.data_ptr(), B, T, C, H, w, err.data_ptr(), s) == 0
    else:
        assert gb.gptk_attention_bwd_bf16(qkv.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                          lse.data_ptr(), Dbuf.data_ptr(), dq.data_ptr(), B, T, C,
                                          H, w, err.data_ptr(), path, s) == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ro, rlse, rdq = _ref(torch, qkv, B, T, C, H, w, dout)
    assert (o.float() - ro).abs().max().item() <= 2e-2 * ro.abs().max().item()
    assert (lse - rlse).abs().max().item() <= 2e-3 * max(1.0, rlse.abs().max().item())
    dv_scale = rdq[:, 2 * C:].abs().max().item()
    for part in range(3):
        a = dq.float()[:, part * C:(part + 1) * C]
        r = rdq[:, part * C:(part + 1) * C]
        if r.abs().max().item() <= 1e-3 * dv_scale:
            # window 0: each query sees only itself, so dS = P(dP - D) = 0 and dq = dk = 0
            # exactly; both sides hold rounding noise only
            assert a.abs().max().item() <= 1e-2 * dv_scale, part
            continue
        cos = torch.nn.functional.cosine_similarity(a.flatten(), r.flatten(), dim=0).item()
        assert cos >= 0.999, (part, cos)
        assert (a - r).abs().max().item() <= 5e-2 * r.abs().max().item(), part
