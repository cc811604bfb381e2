"""The allocation-free attention backward (gptk_attention_bwd_bf16_noalloc).

Some callers cannot allocate device memory (an allocator hook or a memory pool that must not
re-enter the allocator); this entry point keeps its scratch in a static device array. The
test compares it, through the C ABI, with the regular entry point that takes caller scratch,
on the same inputs, on two calls in a row (the shared array keeps the previous call's
contents), and checks the size limit. It runs last so that a failure here leaves every other
test already run, and it passes alone in a fresh process as well as after the others.
"""
import pytest

pytestmark = pytest.mark.gpu


def _inputs(torch, dev, B, T, H, seed):
    C = 64 * H
    g = torch.Generator(device="cpu").manual_seed(seed)
    qkv = (torch.randn(B * T, 3 * C, generator=g) * 1.5).to(torch.bfloat16).to(dev)
    dout = torch.randn(B * T, C, generator=g).to(torch.bfloat16).to(dev)
    return C, qkv, dout


def test_noalloc_matches_regular_entry_point_twice():
    import torch
    from gpt_transformer_step_b200 import binding as gb
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream().cuda_stream
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for call, (B, T, H, w) in enumerate([(2, 300, 3, -1), (1, 520, 2, 100)]):
        C, qkv, dout = _inputs(torch, dev, B, T, H, seed=11 + call)
        o = torch.zeros(B * T, C, dtype=torch.bfloat16, device=dev)
        lse = torch.zeros(B, H, T, device=dev)
        assert gb.gptk_attention_fwd_bf16(qkv.data_ptr(), o.data_ptr(), lse.data_ptr(), B, T, C,
                                          H, w, err.data_ptr(), gb.GPTK_PATH_TCGEN05, s) == 0
        ref = torch.zeros(B * T, 3 * C, dtype=torch.bfloat16, device=dev)
        Dbuf = torch.zeros(B, H, T, device=dev)
        assert gb.gptk_attention_bwd_bf16(qkv.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                          lse.data_ptr(), Dbuf.data_ptr(), ref.data_ptr(), B, T,
                                          C, H, w, err.data_ptr(), gb.GPTK_PATH_TCGEN05, s) == 0
        got = torch.full((B * T, 3 * C), float("nan"), dtype=torch.bfloat16, device=dev)
        assert gb.gptk_attention_bwd_bf16_noalloc(qkv.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                                  lse.data_ptr(), got.data_ptr(), B, T, C, H, w,
                                                  err.data_ptr(), s) == 0
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        # same kernels, same order of every sum: bitwise equal (well inside the attention
        # tests' tolerance)
        assert torch.isfinite(got.float()).all()
        d = (got.float() - ref.float()).abs().max().item()
        assert d <= 5e-2 * ref.float().abs().max().item()
        assert torch.equal(got, ref)


def test_noalloc_rejects_rows_beyond_its_scratch():
    import torch
    from gpt_transformer_step_b200 import binding as gb
    dev = torch.device("cuda", 0)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    x = torch.zeros(16, device=dev)
    # B*H*T = 2 * 8 * 65600 > 2^20 rows: rejected before any launch
    rc = gb.gptk_attention_bwd_bf16_noalloc(x.data_ptr(), x.data_ptr(), x.data_ptr(),
                                            x.data_ptr(), x.data_ptr(), 2, 65600, 512, 8, -1,
                                            err.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == gb.GPT_ERR_SHAPE
