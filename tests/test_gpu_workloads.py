"""Full-size runs of the other workload shapes (Shakespeare-char B=64 x T=256, GPT-2 350M,
124M-width T=2048 with alternating 512-key windows) in the launch configuration the bench
uses: oracle parity on causal prefixes (positions < P depend only on tokens < P), the AdamW
update given the GPU's gradients, bitwise determinism and bitwise causality."""
import math

import numpy as np
import pytest

import oracle
from gpt_transformer_step_b200 import fixtures as fx
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


# The bf16 loss bound is about the loss, the mean over all B*T tokens, which the oracle cannot
# compute at these sizes. It is checked as a chain: the fp32 validation path matches the
# oracle token by token on causal prefixes (positions < P depend only on tokens < P), and the
# bf16 loss over the full batch matches the fp32 path. Single prefix tokens of the bf16 path
# are also bounded against the oracle directly (they spread by ~0.01, more at early positions,
# so a few dozen of them do not estimate the loss).
def _full_size_checks(name, prefix=16, rows=(0,), perturb_at=200):
    wl = fx.WORKLOADS[name]
    sh = wl.shape
    p, tok, tgt = fx.make_inputs(wl)
    o = oracle.Oracle.from_shape(sh, dtype=np.float32)
    refs = [o.forward(p, tok[b:b + 1, :prefix], tgt[b:b + 1, :prefix], per_token=True)[1][0]
            for b in rows]
    st32 = U.make_step(sh, wl.B, wl.T, 0)
    try:
        loss32, ptl32 = U.gpu_forward(st32, p, tok, tgt)
    finally:
        st32.close()
    for b, ref in zip(rows, refs):
        assert np.abs(ptl32[b, :prefix] - ref).max() <= U.FP32_LOSS_ABS
    st = U.make_step(sh, wl.B, wl.T, 1)
    try:
        loss, ptl = U.gpu_forward(st, p, tok, tgt)
        assert abs(loss - math.log(sh.vocab)) < 0.3
        assert abs(loss - loss32) <= U.BF16_LOSS_ABS, (loss, loss32)
        d = np.concatenate([ptl[b, :prefix] - ref for b, ref in zip(rows, refs)])
        assert np.abs(d).max() <= 10 * U.BF16_LOSS_ABS, np.abs(d).max()
        # causality, bitwise
        tok2 = tok.copy()
        tok2[:, perturb_at + 1] = (tok2[:, perturb_at + 1] + 7) % sh.vocab
        _, pert = U.gpu_forward(st, p, tok2, tgt)
        assert np.array_equal(ptl[:, :perturb_at + 1], pert[:, :perturb_at + 1])
        # one step twice from the same state: bitwise identical; update vs oracle AdamW
        r1 = U.gpu_train_step(st, p, tok, tgt, wl.lr, wl.wd, wl.clip)
        st.step = 0
        r2 = U.gpu_train_step(st, p, tok, tgt, wl.lr, wl.wd, wl.clip)
        assert r1.loss == r2.loss and np.array_equal(r1.grads, r2.grads)
        assert np.isfinite(r1.grads).all()
        zeros = np.zeros_like(p, dtype=np.float64)
        pe, _, _, n = U.oracle_adamw_on(r1.grads, p, zeros, zeros, wl.lr, wl.wd, wl.clip, 1)
        assert abs(r1.norm - n) <= 1e-4 * n
        assert np.abs(r1.params - pe).max() <= U.BF16_UPDATE_ABS_PER_LR * wl.lr
        V, Vp, C = sh.vocab, sh.vocab_padded, sh.n_embd
        assert np.all(r1.grads[V * C:Vp * C] == 0)
    finally:
        st.close()


def test_shakespeare_char_full_batch():
    _full_size_checks("shakespeare_char_bf16", prefix=24, rows=(0, 63), perturb_at=100)


def test_gpt2_350m_full_size():
    _full_size_checks("gpt2_350m_bf16", prefix=24, rows=(5, 6), perturb_at=300)


def test_gpt2_124m_sliding_window_full_size():
    _full_size_checks("gpt2_124m_swa_bf16", prefix=24, rows=(6, 7), perturb_at=1500)
