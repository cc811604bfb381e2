"""LayerNorm kernels through the kernel-level C ABI (gptk_layernorm_fwd_bf16 / _bwd_bf16) vs
torch.nn.functional.layer_norm and its autograd gradients in fp32 on the same bf16 inputs:
C = 768 and ragged row counts, with and without an incoming residual gradient and dgamma
accumulation; the backward's invariants sum_c dx = 0 and sum_c dx * xhat = 0 per row."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,C", [(16384, 768), (1000, 768), (37, 1024), (513, 384)])
def test_layernorm_fwd_bwd_vs_torch(M, C):
    import torch
    from gpt_transformer_step_b200 import binding as gb
    dev = torch.device("cuda", 0)
    g_ = torch.Generator(device="cpu").manual_seed(M + C)
    x = (torch.randn(M, C, generator=g_) * 2 + 0.5).to(torch.bfloat16).to(dev)
    gam = (1 + 0.1 * torch.randn(C, generator=g_)).to(torch.bfloat16).to(dev)
    dy = torch.randn(M, C, generator=g_).to(torch.bfloat16).to(dev)
    dres0 = torch.randn(M, C, generator=g_).to(torch.bfloat16).to(dev)
    y = torch.empty(M, C, dtype=torch.bfloat16, device=dev)
    mean = torch.empty(M, device=dev)
    rstd = torch.empty(M, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    assert gb.gptk_layernorm_fwd_bf16(x.data_ptr(), gam.data_ptr(), y.data_ptr(), mean.data_ptr(),
                                      rstd.data_ptr(), M, C, 1e-5, s) == 0
    xr = x.float().requires_grad_()
    gr = gam.float().requires_grad_()
    yr = torch.nn.functional.layer_norm(xr, (C,), gr, None, 1e-5)
    torch.cuda.synchronize()
    assert (y.float() - yr).abs().max().item() <= 2e-2 * yr.abs().max().item()
    assert (mean - x.float().mean(1)).abs().max().item() <= 1e-5 * x.float().abs().max().item()
    yr.backward(dy.float())
    nsc = gb.gptk_layernorm_bwd_scratch_floats(M, C)
    scratch = torch.empty(nsc, device=dev)
    for dres_in, acc in ((0, 0), (1, 1)):
        dres = dres0.clone()
        dg = torch.full((C,), 0.25, device=dev)
        assert gb.gptk_layernorm_bwd_bf16(x.data_ptr(), gam.data_ptr(), mean.data_ptr(),
                                          rstd.data_ptr(), dy.data_ptr(), dres.data_ptr(), dres_in,
                                          dg.data_ptr(), acc, scratch.data_ptr(), nsc, M, C, s) == 0
        torch.cuda.synchronize()
        ref_dx = xr.grad + (dres0.float() if dres_in else 0)
        assert (dres.float() - ref_dx).abs().max().item() <= 2e-2 * ref_dx.abs().max().item()
        ref_dg = gr.grad + (0.25 if acc else 0)
        assert (dg - ref_dg).abs().max().item() <= 2e-3 * ref_dg.abs().max().item()
        if not dres_in:
            # the projections the backward removes: per row sum(dx) = 0 and sum(dx * xhat) = 0,
            # up to the bf16 rounding of dx (relative 2^-9 per element)
            xh = (x.float() - mean[:, None]) * rstd[:, None]
            d = dres.float()
            assert (d.sum(1).abs() <= 1e-2 * d.abs().sum(1)).all()
            assert ((d * xh).sum(1).abs() <= 1e-2 * (d * xh).abs().sum(1)).all()
