"""The C-ABI library loads and exports every symbol its header declares; argument checks
that need no GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(gptk?_\w+)\s*\(", src)
    return sorted(set(names))


@pytest.fixture(scope="module")
def gb():
    from gpt_transformer_step_b200 import build
    build.build()
    from gpt_transformer_step_b200 import binding
    return binding


def test_every_declared_symbol_is_exported(gb):
    names = declared_functions()
    assert "gpt_train_step" in names and "gpt_create" in names and "gpt_forward_loss" in names
    lib = ctypes.CDLL(gb.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(gb.EXPORTED) >= set(names)


def test_strerror_names_every_code(gb):
    for code in range(0, -9, -1):
        assert gb.gpt_strerror(code).decode() != "unknown status"
    assert gb.gpt_strerror(-99).decode() == "unknown status"


def _cfg(gb, **kw):
    base = dict(vocab=65, vocab_padded=65, n_layer=2, n_head=2, n_embd=64, max_T=32, max_B=4,
                mlp_mult=4, ln_eps=1e-5, beta1=0.9, beta2=0.95, adam_eps=1e-8,
                precision=gb.GPT_FP32, lmhead_chunk_rows=0)
    base.update(kw)
    c = gb.gpt_config()
    for k, v in base.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("bad,code", [
    (dict(vocab=0), -1), (dict(vocab_padded=10), -1), (dict(precision=7), -1),
    (dict(beta1=1.0), -1), (dict(adam_eps=0.0), -1), (dict(n_head=3), -2),
    (dict(n_embd=96, n_head=1), -2), (dict(max_B=2048, max_T=1024), -2),
    (dict(precision=1, n_embd=96, n_head=3), -2), (dict(vocab_padded=200000), -2),
])
def test_create_rejects_bad_config_without_touching_the_gpu(gb, bad, code):
    st = ctypes.c_int(0)
    h = gb.gpt_create(ctypes.byref(_cfg(gb, **bad)), ctypes.byref(st))
    assert not h
    assert st.value == code


def test_null_handle_calls_are_errors(gb):
    loss = ctypes.c_float(0)
    assert gb.gpt_train_step(None, None, None, None, None, None, None, 1, 1, 1e-3, 0.0, 1.0,
                             ctypes.byref(loss)) == gb.GPT_ERR_INVALID_ARG
    assert gb.gpt_forward_loss(None, None, None, None, 1, 1, ctypes.byref(loss), None) == \
        gb.GPT_ERR_INVALID_ARG
    assert gb.gpt_set_stream(None, None) == gb.GPT_ERR_INVALID_ARG
    assert gb.gpt_num_params(None) == 0
    assert gb.gpt_create(None, None) is None
