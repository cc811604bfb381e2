"""The tensor-core GEMM launch plan (CTA group and K split) on the CPU, through the C ABI
(gptk_gemm_plan runs no GPU code): the choices the step relies on and the plan's invariants."""
import math

import pytest


CAP_124M = 8 * 16384 * 768  # split-K scratch floats the 124M workspace provides
M, C = 16384, 768


@pytest.fixture(scope="module")
def gb():
    from gpt_transformer_step_b200 import build
    build.build()
    from gpt_transformer_step_b200 import binding
    return binding


def _plan(gb, m, n, k, epi, cap=CAP_124M, sms=148):
    s, cg, sk = gb.gemm_plan(m, n, k, epi, cap, sms)
    assert s == 0
    return cg, sk


def test_large_forward_gemms_use_pairs_without_split(gb):
    for m, n, k, epi in [(M, 3 * C, C, "store"), (M, 4 * C, C, "store_gelu"), (M, C, 4 * C, "resid"),
                         (M, 50304, C, "store")]:
        assert _plan(gb, m, n, k, epi) == (2, 1), (m, n, k)


def test_weight_gradients_split_k_on_pairs(gb):
    for m, n in [(4 * C, C), (3 * C, C), (C, C), (C, 4 * C)]:
        cg, sk = _plan(gb, m, n, M, "f32_store")
        assert cg == 2 and 2 <= sk <= 16, (m, n, cg, sk)
        # a split of s needs s*M*N floats of scratch and at least 2 k-blocks (128 wide) per range
        assert sk * m * n <= CAP_124M and M // 128 // sk >= 2


def test_no_scratch_means_no_split(gb):
    assert _plan(gb, 4 * C, C, M, "f32_store", cap=0)[1] == 1
    assert _plan(gb, C, C, M, "f32_accum", cap=0)[1] == 1


def test_split_respects_scratch_capacity(gb):
    cap = 3 * C * C  # room for at most 3 partial copies of a 768 x 768 output
    cg, sk = _plan(gb, C, C, M, "f32_store", cap=cap)
    assert sk * C * C <= cap


def test_splits_leave_no_empty_k_range(gb):
    for k in (64, 100, 520, 777 // 8 * 8, 4000, 16384, 50304):
        for m, n in [(300, 200), (768, 768), (2304, 768)]:
            _, sk = _plan(gb, m, n, k, "f32_store")
            kb = math.ceil(k / 128)
            per = math.ceil(kb / sk)
            assert 1 <= sk <= max(1, kb) and per * (sk - 1) < kb, (m, n, k, sk)


def test_machine_filling_gemm_never_splits_and_small_grid_uses_single_ctas(gb):
    # enough 256-row tiles for every SM pair: no split whatever the epilogue
    assert _plan(gb, 8192, 2048, 4096, "f32_store")[1] == 1
    # too few rows for CTA pairs and no scratch: single-CTA tiles
    assert _plan(gb, 256, 256, 256, "store", cap=0) == (1, 1)


def test_bad_arguments(gb):
    assert gb.gemm_plan(0, 10, 10, "store", 0)[0] != 0
    assert gb.gemm_plan(10, 10, 0, "store", 0)[0] != 0
    assert gb.gemm_plan(10, 10, 10, 9, 0)[0] != 0
