"""Edge cases of the step through the C ABI against the oracle: the largest padded vocabulary
the library accepts (131072 columns, 17-bit token ids sorted in two radix passes, a ragged
real vocabulary), sequences of a single token (attention over one key), and 32768 tokens in
one step."""
import numpy as np
import pytest

from gpt_transformer_step_b200 import fixtures as fx
from tests.test_gpu_parity import check_bf16, check_fp32

pytestmark = pytest.mark.gpu


def test_bf16_max_padded_vocab_ragged():
    sh = fx.ModelShape(vocab=131000, vocab_padded=131072, n_layer=1, n_head=2, n_embd=128,
                       max_T=17)
    r = check_bf16(sh, B=2, T=17, seed=11, s=1.01)
    V, C = sh.vocab, sh.n_embd
    assert np.all(r.grads[V * C:sh.vocab_padded * C] == 0)


def test_fp32_max_padded_vocab_ragged():
    sh = fx.ModelShape(vocab=131000, vocab_padded=131072, n_layer=1, n_head=2, n_embd=64,
                       max_T=9)
    check_fp32(sh, B=2, T=9, seed=12, s=1.01)


@pytest.mark.parametrize("B", [1, 3])
def test_single_token_sequences(B):
    sh = fx.ModelShape(vocab=500, vocab_padded=512, n_layer=2, n_head=2, n_embd=128, max_T=8)
    check_fp32(sh, B=B, T=1, seed=13)
    check_bf16(sh, B=B, T=1, seed=14)


def test_32768_tokens_per_step():
    """B*T = 32768 tokens in one step (twice the embedding backward's former one-CTA limit),
    with a vocabulary that takes two radix passes of the id sort: fp32 validation mode against
    the oracle at the fp32 tolerances, bf16 mode at the bf16 ones (one oracle run)."""
    import oracle
    from tests import gpu_util as U
    sh = fx.ModelShape(vocab=600, vocab_padded=640, n_layer=1, n_head=1, n_embd=64, max_T=16)
    B, T, lr, wd, clip = 2048, 16, 1e-3, 0.01, 1.0
    p = fx.init_params(sh, 15)
    tok, tgt = fx.zipf_tokens(sh.vocab, 1.1, B, T, 15)
    o = oracle.Oracle.from_shape(sh, dtype=np.float32)
    loss, g = o.forward_backward(p, tok, tgt)
    st = U.make_step(sh, B, T, 0)
    try:
        r = U.gpu_train_step(st, p, tok, tgt, lr, wd, clip)
    finally:
        st.close()
    assert abs(r.loss - loss) <= U.FP32_LOSS_ABS, (r.loss, loss)
    for (name, a), (_, b) in zip(U.per_tensor(sh, r.grads), U.per_tensor(sh, g)):
        assert U.grad_rel_err(a, b) <= U.FP32_GRAD_REL, (name, U.grad_rel_err(a, b))
    st = U.make_step(sh, B, T, 1)
    try:
        rb = U.gpu_train_step(st, p, tok, tgt, lr, wd, clip)
    finally:
        st.close()
    assert abs(rb.loss - loss) <= U.BF16_LOSS_ABS, (rb.loss, loss)
    U.assert_bf16_grads(sh, rb.grads, g, "32768 tokens bf16")
