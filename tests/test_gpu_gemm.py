"""The tcgen05 GEMM (and the CUDA-core GEMM) through the kernel-level C ABI vs torch.matmul
in fp32 on the same bf16 operands: every operand layout, every epilogue (GELU against torch's
tanh GELU and its autograd derivative), ragged tiles, split-K."""
import ctypes

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


def _pad8(n):
    return (n + 7) // 8 * 8


def _operand(torch, dev, rows, cols, kmajor, seed):
    """Logical [rows, cols] (rows = M or N, cols = K) operand stored K-major or MN-major,
    with the leading dimension padded to a multiple of 8 elements (16 bytes)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(rows, cols, generator=g).to(torch.bfloat16)
    if kmajor:
        ld = _pad8(cols)
        stor = torch.zeros(rows, ld, dtype=torch.bfloat16)
        stor[:, :cols] = x
    else:
        ld = _pad8(rows)
        stor = torch.zeros(cols, ld, dtype=torch.bfloat16)
        stor[:, :rows] = x.t()
    return x.float().to(dev), stor.to(dev), ld


def _gelu(torch, x):
    return torch.nn.functional.gelu(x, approximate="tanh")


CASES = [
    # M, N, K, a_kmajor, b_kmajor, epi, split
    (256, 512, 256, 1, 1, "store", 1),
    (200, 300, 136, 1, 1, "store", 1),
    (128, 256, 64, 1, 1, "store", 1),
    (130, 260, 520, 0, 1, "store", 1),
    (130, 260, 520, 1, 0, "store", 1),
    (384, 768, 1024, 0, 0, "f32_store", 1),
    (300, 200, 1000, 0, 0, "f32_store", 4),
    (257, 129, 777 // 8 * 8, 1, 0, "f32_accum", 1),
    (333, 700, 192, 1, 1, "store_gelu", 1),
    (333, 700, 192, 1, 1, "resid", 1),
    (333, 700, 192, 1, 0, "dgelu", 1),
    (1024, 2304, 768, 1, 1, "store", 1),
    # large enough for 256-row tiles on CTA pairs
    (4096, 2304, 768, 1, 1, "store", 1),
    (4000, 3000, 520, 1, 0, "store", 1),
    (4100, 2600, 264, 0, 1, "dgelu", 1),
    (4096, 4096, 256, 0, 0, "f32_store", 1),
    (3900, 4000, 640, 1, 1, "store_gelu", 1),
    (4096, 3072, 512, 1, 1, "resid", 1),
    (4096, 3000, 1024, 0, 0, "f32_accum", 1),
    # split 0: the launcher picks CTA pairs plus a K split (the weight-gradient shapes)
    (768, 768, 4096, 0, 0, "f32_store", 0),
    (3072, 768, 16384, 0, 0, "f32_store", 0),
    (700, 600, 4000, 0, 0, "f32_accum", 0),
    (768, 3072, 8192, 0, 0, "f32_accum", 0),
]


@pytest.mark.parametrize("path", [0, 1])
@pytest.mark.parametrize("M,N,K,ak,bk,epi,split", CASES)
def test_gemm_vs_torch(env, path, M, N, K, ak, bk, epi, split):
    torch, gb, dev, err = env
    A, As, lda = _operand(torch, dev, M, K, ak, 1)
    B, Bs, ldb = _operand(torch, dev, N, K, bk, 2)
    ref = A @ B.t()
    ldo = _pad8(N)
    out_s = torch.zeros(M, ldo, dtype=torch.bfloat16, device=dev)
    out2_s = torch.zeros(M, ldo, dtype=torch.bfloat16, device=dev)
    aux_s = (torch.randn(M, ldo, device=dev) * 0.5).to(torch.bfloat16)
    outf_s = torch.randn(M, ldo, device=dev)
    outf0 = outf_s[:, :N].clone()
    scratch = torch.zeros(max(1, (split or 16) * M * N), device=dev)
    err.zero_()
    s = gb.gptk_gemm_bf16(M, N, K, As.data_ptr(), lda, ak, Bs.data_ptr(), ldb, bk, gb.GPTK_EPI[epi],
                          out_s.data_ptr(), ldo, out2_s.data_ptr(), ldo, aux_s.data_ptr(), ldo,
                          outf_s.data_ptr(), ldo, split, scratch.data_ptr(), scratch.numel(),
                          err.data_ptr(), path, torch.cuda.current_stream().cuda_stream)
    assert s == 0, gb.gpt_strerror(s)
    torch.cuda.synchronize()
    out, out2, aux, outf = out_s[:, :N], out2_s[:, :N], aux_s[:, :N], outf_s[:, :N]
    assert int(err.item()) == 0
    scale = ref.abs().max().item()
    if epi == "store":
        d = (out.float() - ref).abs().max().item()
        assert d <= 1e-2 * scale, d
    elif epi == "store_gelu":
        # out = gelu'(acc) (what the backward needs), out2 = gelu(acc)
        x = ref.clone().requires_grad_()
        g = _gelu(torch, x)
        g.backward(torch.ones_like(g))
        assert (out.float() - x.grad).abs().max().item() <= 1e-2 * x.grad.abs().max().item()
        assert (out2.float() - g.detach()).abs().max().item() <= 1e-2 * g.abs().max().item()
    elif epi == "resid":
        r = aux.float() + ref
        assert (out.float() - r).abs().max().item() <= 1e-2 * r.abs().max().item()
    elif epi == "dgelu":
        # aux holds gelu'(pre) as the forward stored it
        r = ref * aux.float()
        assert (out.float() - r).abs().max().item() <= 1e-2 * r.abs().max().item()
    elif epi == "f32_store":
        assert (outf - ref).abs().max().item() <= 1e-4 * scale
    elif epi == "f32_accum":
        assert (outf - (outf0 + ref)).abs().max().item() <= 1e-4 * scale
