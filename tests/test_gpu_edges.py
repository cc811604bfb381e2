"""Edge cases of the step through the C ABI against the oracle: the largest padded vocabulary
the library accepts (131072 columns, 17-bit token ids in the embedding-sort keys, a ragged
real vocabulary), and sequences of a single token (attention over one key)."""
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
