"""ctypes loader for the oracle -- TEST INFRASTRUCTURE ONLY.

The oracle is a plain single-threaded C++ definition of one GPT-2-style training step
(gpt_oracle.cpp). Only the tests, `__graft_entry__.smoke()` and the benchmark's CPU-baseline
leg import this package; the CUDA library and its Python binding never do.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRCS = [os.path.join(_HERE, "gpt_oracle.cpp"), os.path.join(_HERE, "muon_oracle.cpp")]
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, IEEE semantics: no fast-math)."""
    deps = _SRCS + [os.path.join(_HERE, "gpt_oracle.h")]
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(map(os.path.getmtime, deps)):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", *_SRCS, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int), ("vocab_padded", ctypes.c_int),
                ("n_layer", ctypes.c_int), ("n_head", ctypes.c_int), ("n_embd", ctypes.c_int),
                ("max_T", ctypes.c_int), ("mlp_mult", ctypes.c_int),
                ("window_left", ctypes.POINTER(ctypes.c_int)), ("ln_eps", ctypes.c_double)]


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        L = _lib
        L.oracle_num_params.restype = ctypes.c_size_t
        L.oracle_num_params.argtypes = [P]
        L.oracle_layout.restype = ctypes.c_int
        L.oracle_layout.argtypes = [P, P, P, ctypes.c_int]
        for suf, R in (("f64", ctypes.c_double), ("f32", ctypes.c_float)):
            f = getattr(L, f"oracle_forward_{suf}")
            f.restype = R
            f.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, P]
            f = getattr(L, f"oracle_forward_backward_{suf}")
            f.restype = R
            f.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, P, P]
            f = getattr(L, f"oracle_grad_norm_{suf}")
            f.restype = ctypes.c_double
            f.argtypes = [ctypes.c_size_t, P]
            f = getattr(L, f"oracle_adamw_{suf}")
            f.restype = None
            f.argtypes = [ctypes.c_size_t, P, P, P, P] + [R] * 5 + [ctypes.c_long, R]
            f = getattr(L, f"oracle_train_step_{suf}")
            f.restype = R
            f.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int] + [R] * 6 + \
                [ctypes.c_long, P]
            f = getattr(L, f"oracle_train_step_accum_{suf}")
            f.restype = R
            f.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int] + \
                [R] * 6 + [ctypes.c_long, P]
        L.oracle_layernorm_fwd_f64.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                               P, P, P]
        L.oracle_layernorm_bwd_f64.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int, P, P]
        L.oracle_attention_fwd_f64.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, P]
        L.oracle_attention_bwd_f64.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, P]
        L.oracle_gelu_f64.restype = ctypes.c_double
        L.oracle_gelu_f64.argtypes = [ctypes.c_double]
        L.oracle_gelu_grad_f64.restype = ctypes.c_double
        L.oracle_gelu_grad_f64.argtypes = [ctypes.c_double]
        L.oracle_polar_express_f64.restype = None
        L.oracle_polar_express_f64.argtypes = [P, ctypes.c_int, ctypes.c_int, P, ctypes.c_int,
                                               ctypes.c_int]
        L.oracle_muon_adamw_f64.restype = ctypes.c_double
        L.oracle_muon_adamw_f64.argtypes = [ctypes.c_size_t, P, P, P, P, ctypes.c_int, P, P, P] + \
            [ctypes.c_double] * 10 + [P, ctypes.c_int, ctypes.c_double, ctypes.c_long, ctypes.c_int]
        L.oracle_cross_entropy_f64.restype = ctypes.c_double
        L.oracle_cross_entropy_f64.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """Holds one model shape; `dtype` selects the float or double instantiation."""

    def __init__(self, vocab: int, vocab_padded: int, n_layer: int, n_head: int, n_embd: int,
                 max_T: int, mlp_mult: int = 4, window_left: Optional[Sequence[int]] = None,
                 ln_eps: float = 1e-5, dtype=np.float64):
        self.lib = _load()
        self.dtype = np.dtype(dtype)
        self.suf = "f64" if self.dtype == np.float64 else "f32"
        self._win = (ctypes.c_int * n_layer)(*(window_left if window_left else [-1] * n_layer))
        self.cfg = _Cfg(vocab, vocab_padded, n_layer, n_head, n_embd, max_T, mlp_mult,
                        ctypes.cast(self._win, ctypes.POINTER(ctypes.c_int)), ln_eps)
        self.n = int(self.lib.oracle_num_params(ctypes.byref(self.cfg)))

    @classmethod
    def from_shape(cls, sh, dtype=np.float64, ln_eps: float = 1e-5):
        return cls(sh.vocab, sh.vocab_padded, sh.n_layer, sh.n_head, sh.n_embd, sh.max_T,
                   sh.mlp_mult, sh.windows(), ln_eps, dtype)

    def layout(self) -> List[tuple]:
        cap = 16 + 6 * self.cfg.n_layer
        off = np.zeros(cap, np.int64)
        num = np.zeros(cap, np.int64)
        k = self.lib.oracle_layout(ctypes.byref(self.cfg), _ptr(off), _ptr(num), cap)
        return [(int(off[i]), int(num[i])) for i in range(k)]

    def _arr(self, a):
        return np.ascontiguousarray(a, dtype=self.dtype)

    def forward(self, params, tokens, targets, per_token=False):
        p = self._arr(params)
        tok = np.ascontiguousarray(tokens, np.int32)
        tgt = np.ascontiguousarray(targets, np.int32)
        B, T = tok.shape
        ptl = np.zeros(B * T, self.dtype) if per_token else None
        f = getattr(self.lib, f"oracle_forward_{self.suf}")
        loss = f(ctypes.byref(self.cfg), _ptr(p), _ptr(tok), _ptr(tgt), B, T, _ptr(ptl))
        return (loss, ptl.reshape(B, T)) if per_token else loss

    def forward_backward(self, params, tokens, targets, per_token=False):
        p = self._arr(params)
        tok = np.ascontiguousarray(tokens, np.int32)
        tgt = np.ascontiguousarray(targets, np.int32)
        B, T = tok.shape
        g = np.zeros(self.n, self.dtype)
        ptl = np.zeros(B * T, self.dtype) if per_token else None
        f = getattr(self.lib, f"oracle_forward_backward_{self.suf}")
        loss = f(ctypes.byref(self.cfg), _ptr(p), _ptr(tok), _ptr(tgt), B, T, _ptr(g), _ptr(ptl))
        return (loss, g, ptl.reshape(B, T)) if per_token else (loss, g)

    def grad_norm(self, g) -> float:
        g = self._arr(g)
        return getattr(self.lib, f"oracle_grad_norm_{self.suf}")(g.size, _ptr(g))

    def adamw(self, p, g, m, v, lr, wd, step, coef=1.0, beta1=0.9, beta2=0.95, eps=1e-8):
        """In place on p, m, v (arrays of this oracle's dtype)."""
        for a in (p, m, v):
            assert a.dtype == self.dtype and a.flags.c_contiguous
        g = self._arr(g)
        getattr(self.lib, f"oracle_adamw_{self.suf}")(p.size, _ptr(p), _ptr(g), _ptr(m), _ptr(v),
                                                       lr, wd, beta1, beta2, eps, step, coef)

    def train_step(self, p, m, v, tokens, targets, lr, wd, clip, step, beta1=0.9, beta2=0.95,
                   eps=1e-8):
        """In place on p, m, v. Returns (loss, raw grads, unclipped grad norm)."""
        for a in (p, m, v):
            assert a.dtype == self.dtype and a.flags.c_contiguous
        tok = np.ascontiguousarray(tokens, np.int32)
        tgt = np.ascontiguousarray(targets, np.int32)
        B, T = tok.shape
        g = np.zeros(self.n, self.dtype)
        gn = ctypes.c_double(0.0)
        f = getattr(self.lib, f"oracle_train_step_{self.suf}")
        loss = f(ctypes.byref(self.cfg), _ptr(p), _ptr(g), _ptr(m), _ptr(v), _ptr(tok), _ptr(tgt),
                 B, T, lr, wd, clip, beta1, beta2, eps, step, ctypes.byref(gn))
        return loss, g, gn.value

    def train_step_accum(self, p, m, v, tokens, targets, lr, wd, clip, step, beta1=0.9,
                         beta2=0.95, eps=1e-8):
        """Gradient accumulation: tokens/targets [n_micro, B, T]; one optimizer step over all
        micro-batches, in place on p, m, v. Returns (mean loss, raw mean grads, norm)."""
        for a in (p, m, v):
            assert a.dtype == self.dtype and a.flags.c_contiguous
        tok = np.ascontiguousarray(tokens, np.int32)
        tgt = np.ascontiguousarray(targets, np.int32)
        n_micro, B, T = tok.shape
        g = np.zeros(self.n, self.dtype)
        gn = ctypes.c_double(0.0)
        f = getattr(self.lib, f"oracle_train_step_accum_{self.suf}")
        loss = f(ctypes.byref(self.cfg), _ptr(p), _ptr(g), _ptr(m), _ptr(v), _ptr(tok), _ptr(tgt),
                 n_micro, B, T, lr, wd, clip, beta1, beta2, eps, step, ctypes.byref(gn))
        return loss, g, gn.value

    # -- single pieces (double) --
    def layernorm_fwd(self, x, g, eps=1e-5):
        x = np.ascontiguousarray(x, np.float64)
        rows, C = x.shape
        y = np.zeros_like(x)
        mu = np.zeros(rows)
        rs = np.zeros(rows)
        self.lib.oracle_layernorm_fwd_f64(_ptr(x), _ptr(np.ascontiguousarray(g, np.float64)),
                                          rows, C, eps, _ptr(y), _ptr(mu), _ptr(rs))
        return y, mu, rs

    def layernorm_bwd(self, x, g, mu, rs, dy):
        x = np.ascontiguousarray(x, np.float64)
        rows, C = x.shape
        dx = np.zeros_like(x)
        dg = np.zeros(C)
        self.lib.oracle_layernorm_bwd_f64(_ptr(x), _ptr(np.ascontiguousarray(g, np.float64)),
                                          _ptr(mu), _ptr(rs),
                                          _ptr(np.ascontiguousarray(dy, np.float64)), rows, C,
                                          _ptr(dx), _ptr(dg))
        return dx, dg

    def attention_fwd(self, qkv, H, window=-1):
        qkv = np.ascontiguousarray(qkv, np.float64)
        B, T, C3 = qkv.shape
        o = np.zeros((B, T, C3 // 3))
        self.lib.oracle_attention_fwd_f64(_ptr(qkv), B, T, C3 // 3, H, window, _ptr(o))
        return o

    def attention_bwd(self, qkv, dout, H, window=-1):
        qkv = np.ascontiguousarray(qkv, np.float64)
        B, T, C3 = qkv.shape
        d = np.zeros_like(qkv)
        self.lib.oracle_attention_bwd_f64(_ptr(qkv), _ptr(np.ascontiguousarray(dout, np.float64)),
                                          B, T, C3 // 3, H, window, _ptr(d))
        return d

    def polar_express(self, X, coeffs, ns=None, bf16=False):
        """Polar Express (normalisation, then ns iterations) of a 2-D array; returns a copy.
        bf16: every matrix the iteration stores rounded to bf16 (the page's precision)."""
        X = np.array(X, dtype=np.float64, order="C", copy=True)
        cf = np.ascontiguousarray(coeffs, np.float64).reshape(-1)
        ns = len(cf) // 3 if ns is None else ns
        self.lib.oracle_polar_express_f64(_ptr(X), X.shape[0], X.shape[1], _ptr(cf), ns, int(bf16))
        return X

    def matrices(self):
        """(offset, rows, cols) of the 2-D block matrices Muon updates: per layer w_qkv,
        w_attnproj, w_fc, w_mlpproj (the flat layout of this oracle)."""
        lay = self.layout()
        C, mC, L = self.cfg.n_embd, self.cfg.mlp_mult * self.cfg.n_embd, self.cfg.n_layer
        out = []
        for l in range(L):
            base = 2 + 6 * l  # wte, wpe, then per layer ln1, w_qkv, w_ap, ln2, w_fc, w_mp
            out += [(lay[base + 1][0], 3 * C, C), (lay[base + 2][0], C, C),
                    (lay[base + 4][0], mC, C), (lay[base + 5][0], C, mC)]
        return out

    def muon_adamw(self, p, g, m, v, lr, wd, step, clip, coeffs, matrix_lr=0.02, muon_wd=0.0,
                   mu=0.95, beta2_muon=0.95, s_eps=1e-10, beta1=0.9, beta2=0.95, eps=1e-8,
                   ns=None, bf16=False):
        """One hybrid step in place on p, m, v (double arrays); returns the grad norm. bf16:
        the Polar Express at the page's precision (oracle_polar_express_f64)."""
        for a in (p, m, v):
            assert a.dtype == np.float64 and a.flags.c_contiguous
        mats = self.matrices()
        off = np.array([x[0] for x in mats], np.int64)
        rows = np.array([x[1] for x in mats], np.int32)
        cols = np.array([x[2] for x in mats], np.int32)
        cf = np.ascontiguousarray(coeffs, np.float64).reshape(-1)
        ns = len(cf) // 3 if ns is None else ns
        g = np.ascontiguousarray(g, np.float64)
        return self.lib.oracle_muon_adamw_f64(p.size, _ptr(p), _ptr(g), _ptr(m), _ptr(v), len(mats),
                                              _ptr(off), _ptr(rows), _ptr(cols), lr, wd, beta1,
                                              beta2, eps, matrix_lr, muon_wd, mu, beta2_muon,
                                              s_eps, _ptr(cf), ns, clip, step, int(bf16))

    def gelu(self, x: float) -> float:
        return self.lib.oracle_gelu_f64(x)

    def gelu_grad(self, x: float) -> float:
        return self.lib.oracle_gelu_grad_f64(x)

    def cross_entropy(self, logits, targets, V):
        lg = np.ascontiguousarray(logits, np.float64)
        rows, Vp = lg.shape
        d = np.zeros_like(lg)
        loss = self.lib.oracle_cross_entropy_f64(_ptr(lg), _ptr(np.ascontiguousarray(targets, np.int32)),
                                                 rows, V, Vp, _ptr(d))
        return loss, d


def polar_express_coeffs(steps: int = 5, lo: float = 1e-3, npts: int = 6000) -> np.ndarray:
    """The Polar Express coefficient table (nanochat architecture page, "Polar Express
    Details", refers to it without printing it), built the way the method defines it: step t
    takes the odd quintic a x + b x^3 + c x^5 with the least max |1 - p(x)| over the interval
    the singular values are in, and the next interval is [1 - E, 1 + E], E that least error.
    Each minimax problem is solved here as a linear programme over a dense grid (HiGHS via
    scipy): minimise E subject to |1 - p(x)| <= E at every grid point. [steps, 3] float64."""
    from scipy.optimize import linprog
    out = []
    lo_t, hi_t = lo, 1.0
    for _ in range(steps):
        x = np.unique(np.concatenate([np.geomspace(lo_t, hi_t, npts // 2),
                                      np.linspace(lo_t, hi_t, npts // 2)]))
        P = np.stack([x, x ** 3, x ** 5], axis=1)
        ones = np.ones((len(x), 1))
        A_ub = np.vstack([np.hstack([-P, -ones]), np.hstack([P, -ones])])
        b_ub = np.concatenate([-np.ones(len(x)), np.ones(len(x))])
        r = linprog([0, 0, 0, 1], A_ub=A_ub, b_ub=b_ub,
                    bounds=[(None, None)] * 3 + [(0, None)], method="highs")
        a, b, c, E = r.x
        out.append((a, b, c))
        lo_t, hi_t = 1 - E, 1 + E
    return np.array(out, dtype=np.float64)
