"""Python binding of the B200 GPT-2 training-step library (libgptstep.so).

Argument marshalling only: every step of the computation runs in the library's CUDA kernels.
PyTorch supplies device memory (tensor.data_ptr()) and the current CUDA stream.
The functions carry the C names (gpt_create, gpt_forward_loss, gpt_train_step, ...); the
`GPTStep` class wraps a handle and raises `GPTError` on a non-zero status.

If libgptstep.so is missing this module raises at import time: there is no fallback path.
Build it with `python -m gpt_transformer_step_b200.build` (or `__graft_entry__.build()`).
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptstep.so")

GPT_OK = 0
GPT_ERR_INVALID_ARG = -1
GPT_ERR_SHAPE = -2
GPT_ERR_ALIGN = -3
GPT_ERR_OOM = -4
GPT_ERR_CUDA = -5
GPT_ERR_NONFINITE = -6
GPT_ERR_DEVICE_TIMEOUT = -7
GPT_ERR_BAD_TOKEN = -8
GPT_FP32 = 0
GPT_BF16 = 1
GPT_OPT_USE_GRAPHS = 1
GPT_OPT_TIME_KERNELS = 2
# kernel classes of gpt_kernel_stats: (id, name, unit of the algorithmic work)
KSTATS = [(0, "gemm", "flop"), (1, "gemm_recompute", "flop"), (2, "attn_fwd", "flop"),
          (3, "attn_bwd", "flop"), (4, "ln_fwd", "byte"), (5, "ln_bwd", "byte"),
          (6, "embed_fwd", "byte"), (7, "embed_bwd", "byte"), (8, "ce_combine", "byte"),
          (9, "grad_norm", "byte"), (10, "adamw", "byte"), (11, "muon", "flop")]

EXPORTED = [
    "gpt_create", "gpt_destroy", "gpt_num_params", "gpt_param_layout", "gpt_set_stream",
    "gpt_forward_loss", "gpt_train_step", "gpt_train_step_accum", "gpt_get_step", "gpt_set_step",
    "gpt_last_grad_norm",
    "gpt_params_changed", "gpt_set_option", "gpt_kernel_stats", "gpt_last_launch_count",
    "gpt_strerror", "gpt_last_cuda_error", "gptk_gemm_bf16", "gptk_attention_fwd_bf16",
    "gptk_attention_bwd_bf16", "gptk_attention_bwd_bf16_noalloc", "gptk_selftest_bounded_wait",
    "gptk_gemm_plan", "gpt_forward_backward", "gpt_sumsq", "gpt_adamw_ranges", "gpt_muon_update",
    "gptk_attention_bwd_bf16_ds", "gptk_layernorm_fwd_bf16", "gptk_layernorm_bwd_bf16",
    "gptk_layernorm_bwd_scratch_floats",
]


class gpt_config(ctypes.Structure):
    _fields_ = [("vocab", ctypes.c_int), ("vocab_padded", ctypes.c_int),
                ("n_layer", ctypes.c_int), ("n_head", ctypes.c_int), ("n_embd", ctypes.c_int),
                ("max_T", ctypes.c_int), ("max_B", ctypes.c_int), ("mlp_mult", ctypes.c_int),
                ("window_left", ctypes.POINTER(ctypes.c_int)), ("ln_eps", ctypes.c_float),
                ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("adam_eps", ctypes.c_float), ("precision", ctypes.c_int),
                ("lmhead_chunk_rows", ctypes.c_int), ("recompute_gelu", ctypes.c_int)]


class gpt_muon_config(ctypes.Structure):
    _fields_ = [("matrix_lr", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("momentum", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("ns_steps", ctypes.c_int), ("coeffs", ctypes.POINTER(ctypes.c_float))]


class gpt_tensor_desc(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("offset", ctypes.c_longlong),
                ("ndim", ctypes.c_int), ("shape", ctypes.c_longlong * 2)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build the CUDA library first "
                      "(python -m gpt_transformer_step_b200.build)")

_lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


gpt_create = _sig("gpt_create", _P, [ctypes.POINTER(gpt_config), ctypes.POINTER(_I)])
gpt_destroy = _sig("gpt_destroy", None, [_P])
gpt_num_params = _sig("gpt_num_params", ctypes.c_size_t, [_P])
gpt_param_layout = _sig("gpt_param_layout", _I, [_P, ctypes.POINTER(gpt_tensor_desc), _I])
gpt_set_stream = _sig("gpt_set_stream", _I, [_P, _P])
gpt_forward_loss = _sig("gpt_forward_loss", _I, [_P, _P, _P, _P, _I, _I, ctypes.POINTER(_F), _P])
gpt_train_step = _sig("gpt_train_step", _I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _F, _F, _F,
                                             ctypes.POINTER(_F)])
gpt_train_step_accum = _sig("gpt_train_step_accum", _I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I,
                                                         _F, _F, _F, ctypes.POINTER(_F)])
gpt_forward_backward = _sig("gpt_forward_backward", _I, [_P, _P, _P, _P, _P, _I, _I, _I, _F,
                                                         ctypes.POINTER(_F)])
gpt_sumsq = _sig("gpt_sumsq", _I, [_P, _P, ctypes.c_size_t, _P])
gpt_adamw_ranges = _sig("gpt_adamw_ranges", _I, [_P, _P, _P, _P, _P, _P, _P, _I, _F, _F, _F, _P,
                                                 ctypes.c_long])
gpt_muon_update = _sig("gpt_muon_update", _I, [_P, _P, _P, _P, _P, ctypes.POINTER(gpt_muon_config),
                                               _F, _F, _F])
gpt_get_step = _sig("gpt_get_step", _I, [_P, ctypes.POINTER(ctypes.c_long)])
gpt_set_step = _sig("gpt_set_step", _I, [_P, ctypes.c_long])
gpt_last_grad_norm = _sig("gpt_last_grad_norm", _F, [_P])
gpt_params_changed = _sig("gpt_params_changed", _I, [_P])
gpt_set_option = _sig("gpt_set_option", _I, [_P, _I, ctypes.c_long])
gpt_kernel_stats = _sig("gpt_kernel_stats", _I, [_P, _I, ctypes.POINTER(ctypes.c_longlong),
                                                 ctypes.POINTER(ctypes.c_double),
                                                 ctypes.POINTER(ctypes.c_double), _I])
gpt_last_launch_count = _sig("gpt_last_launch_count", _I, [_P])
gpt_strerror = _sig("gpt_strerror", ctypes.c_char_p, [_I])
gpt_last_cuda_error = _sig("gpt_last_cuda_error", ctypes.c_char_p, [_P])
_L = ctypes.c_long
gptk_gemm_bf16 = _sig("gptk_gemm_bf16", _I, [_I, _I, _I, _P, _L, _I, _P, _L, _I, _I, _P, _L, _P, _L,
                                             _P, _L, _P, _L, _I, _P, ctypes.c_size_t, _P, _I, _P])
gptk_attention_fwd_bf16 = _sig("gptk_attention_fwd_bf16", _I, [_P, _P, _P, _I, _I, _I, _I, _I, _P,
                                                               _I, _P])
gptk_attention_bwd_bf16 = _sig("gptk_attention_bwd_bf16", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I,
                                                               _I, _I, _P, _I, _P])
gptk_attention_bwd_bf16_ds = _sig("gptk_attention_bwd_bf16_ds", _I, [_P, _P, _P, _P, _P, _P, _P, _I,
                                                                     _I, _I, _I, _I, _P, _P])
gptk_layernorm_fwd_bf16 = _sig("gptk_layernorm_fwd_bf16", _I, [_P, _P, _P, _P, _P, _I, _I, _F, _P])
gptk_layernorm_bwd_scratch_floats = _sig("gptk_layernorm_bwd_scratch_floats", ctypes.c_size_t,
                                         [_I, _I])
gptk_layernorm_bwd_bf16 = _sig("gptk_layernorm_bwd_bf16", _I, [_P, _P, _P, _P, _P, _P, _I, _P, _I,
                                                               _P, ctypes.c_size_t, _I, _I, _P])
gptk_attention_bwd_bf16_noalloc = _sig("gptk_attention_bwd_bf16_noalloc", _I,
                                       [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P])
gptk_selftest_bounded_wait = _sig("gptk_selftest_bounded_wait", _I, [ctypes.c_uint, _P, _P])
gptk_gemm_plan = _sig("gptk_gemm_plan", _I, [_I, _I, _I, _I, ctypes.c_size_t, _I, ctypes.POINTER(_I),
                                             ctypes.POINTER(_I)])


def gemm_plan(M: int, N: int, K: int, epi: str, scratch_floats: int, sms: int = 148):
    """(status, cta_group, split_k) of the tensor-core launch plan for this GEMM (host only)."""
    cg, sk = _I(0), _I(0)
    s = gptk_gemm_plan(M, N, K, GPTK_EPI[epi] if isinstance(epi, str) else epi, scratch_floats,
                       sms, ctypes.byref(cg), ctypes.byref(sk))
    return s, cg.value, sk.value
GPTK_EPI = {"store": 0, "store_gelu": 1, "resid": 2, "dgelu": 3, "f32_store": 4, "f32_accum": 5}
GPTK_PATH_TCGEN05 = 0
GPTK_PATH_SIMT = 1


class GPTError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        msg = f"{where}: {gpt_strerror(status).decode()} ({status})"
        if detail:
            msg += f": {detail}"
        super().__init__(msg)
        self.status = status


def _ptr(t) -> Optional[int]:
    """Device (or host) address of a tensor / numpy array, or None."""
    if t is None:
        return None
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    return t.ctypes.data


class GPTStep:
    """One library handle on the current CUDA device."""

    def __init__(self, vocab: int, vocab_padded: int, n_layer: int, n_head: int, n_embd: int,
                 max_T: int, max_B: int, mlp_mult: int = 4,
                 window_left: Optional[Sequence[int]] = None, precision: int = GPT_BF16,
                 ln_eps: float = 1e-5, beta1: float = 0.9, beta2: float = 0.95,
                 adam_eps: float = 1e-8, lmhead_chunk_rows: int = 0, recompute_gelu: bool = False):
        self._win = (ctypes.c_int * n_layer)(*(window_left or [-1] * n_layer))
        cfg = gpt_config(vocab, vocab_padded, n_layer, n_head, n_embd, max_T, max_B, mlp_mult,
                         ctypes.cast(self._win, ctypes.POINTER(ctypes.c_int)), ln_eps, beta1,
                         beta2, adam_eps, precision, lmhead_chunk_rows, int(recompute_gelu))
        st = ctypes.c_int(0)
        self.h = gpt_create(ctypes.byref(cfg), ctypes.byref(st))
        if not self.h:
            raise GPTError(st.value, "gpt_create")
        self.n_params = int(gpt_num_params(self.h))
        self.precision = precision

    @classmethod
    def from_workload(cls, wl, max_B: Optional[int] = None, max_T: Optional[int] = None,
                      precision: Optional[int] = None, **kw):
        sh = wl.shape
        prec = precision if precision is not None else (GPT_BF16 if wl.precision == "bf16" else GPT_FP32)
        return cls(sh.vocab, sh.vocab_padded, sh.n_layer, sh.n_head, sh.n_embd,
                   sh.max_T if max_T is None else max_T, wl.B if max_B is None else max_B,
                   sh.mlp_mult, sh.windows(), prec, wl.ln_eps, wl.beta1, wl.beta2, wl.adam_eps,
                   **kw)

    def close(self):
        if getattr(self, "h", None):
            gpt_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, s: int, where: str):
        if s != GPT_OK:
            raise GPTError(s, where, gpt_last_cuda_error(self.h).decode())

    def layout(self) -> List[tuple]:
        n = gpt_param_layout(self.h, None, 0)
        arr = (gpt_tensor_desc * n)()
        gpt_param_layout(self.h, arr, n)
        return [(d.name.decode(), int(d.offset), tuple(int(d.shape[i]) for i in range(d.ndim)))
                for d in arr]

    def set_stream(self, stream_handle: int):
        self._check(gpt_set_stream(self.h, stream_handle), "gpt_set_stream")

    def use_current_torch_stream(self):
        import torch
        self.set_stream(torch.cuda.current_stream().cuda_stream)

    def forward_loss(self, params, tokens, targets, per_token_loss=None) -> float:
        B, T = tokens.shape
        loss = ctypes.c_float(0)
        s = gpt_forward_loss(self.h, _ptr(params), _ptr(tokens), _ptr(targets), B, T,
                             ctypes.byref(loss), _ptr(per_token_loss))
        self._check(s, "gpt_forward_loss")
        return loss.value

    def train_step(self, params, grads, adam_m, adam_v, tokens, targets, lr, wd, clip) -> float:
        B, T = tokens.shape
        loss = ctypes.c_float(0)
        s = gpt_train_step(self.h, _ptr(params), _ptr(grads), _ptr(adam_m), _ptr(adam_v),
                           _ptr(tokens), _ptr(targets), B, T, lr, wd, clip, ctypes.byref(loss))
        self._check(s, "gpt_train_step")
        return loss.value

    def train_step_accum(self, params, grads, adam_m, adam_v, tokens, targets, lr, wd, clip):
        """One optimizer step over micro-batches: tokens/targets [n_micro, B, T] int32."""
        n_micro, B, T = tokens.shape
        loss = ctypes.c_float(0)
        s = gpt_train_step_accum(self.h, _ptr(params), _ptr(grads), _ptr(adam_m), _ptr(adam_v),
                                 _ptr(tokens), _ptr(targets), n_micro, B, T, lr, wd, clip,
                                 ctypes.byref(loss))
        self._check(s, "gpt_train_step_accum")
        return loss.value

    def forward_backward(self, params, grads, tokens, targets, grad_scale=1.0) -> float:
        """Forward + backward only (no clip, no update): tokens/targets [B, T] or
        [n_micro, B, T]; grads = grad_scale * gradient of the mean loss. Returns the loss."""
        if len(tokens.shape) == 2:
            n_micro, (B, T) = 1, tokens.shape
        else:
            n_micro, B, T = tokens.shape
        loss = ctypes.c_float(0)
        s = gpt_forward_backward(self.h, _ptr(params), _ptr(grads), _ptr(tokens), _ptr(targets),
                                 n_micro, B, T, grad_scale, ctypes.byref(loss))
        self._check(s, "gpt_forward_backward")
        return loss.value

    def sumsq(self, x, out):
        """out (device float64 tensor, 1 element) = sum of x^2 (device fp32), enqueued."""
        self._check(gpt_sumsq(self.h, _ptr(x), x.numel(), _ptr(out)), "gpt_sumsq")

    def adamw_ranges(self, params, grads, adam_m, adam_v, ranges, lr, wd, clip, sumsq, step):
        """AdamW on params[off:off+cnt] for (off, cnt) in ranges; grads, adam_m, adam_v hold
        the ranges compactly; sumsq: device float64 global sum of squares."""
        n = len(ranges)
        offs = (ctypes.c_longlong * max(n, 1))(*[r[0] for r in ranges])
        cnts = (ctypes.c_longlong * max(n, 1))(*[r[1] for r in ranges])
        s = gpt_adamw_ranges(self.h, _ptr(params), _ptr(grads), _ptr(adam_m), _ptr(adam_v), offs,
                             cnts, n, lr, wd, clip, _ptr(sumsq), step)
        self._check(s, "gpt_adamw_ranges")

    def muon_update(self, params, grads, adam_m, adam_v, lr, wd, clip, muon=None):
        """The hybrid Muon + AdamW update on the raw gradient `grads` (gpt_muon_update);
        muon: a muon.MuonConfig (defaults: the page's matrix_lr 0.02, Polar Express x5)."""
        from gpt_transformer_step_b200.muon import MuonConfig
        mc_py = muon or MuonConfig()
        cf = (ctypes.c_float * max(1, 3 * mc_py.ns_steps))(
            *[float(x) for x in list(mc_py.coeffs.reshape(-1))[:3 * mc_py.ns_steps]])
        mc = gpt_muon_config(mc_py.matrix_lr, mc_py.weight_decay, mc_py.momentum, mc_py.beta2,
                             mc_py.eps, mc_py.ns_steps, ctypes.cast(cf, ctypes.POINTER(ctypes.c_float)))
        s = gpt_muon_update(self.h, _ptr(params), _ptr(grads), _ptr(adam_m), _ptr(adam_v),
                            ctypes.byref(mc), lr, wd, clip)
        self._check(s, "gpt_muon_update")

    def train_step_status(self, params, grads, adam_m, adam_v, tokens, targets, lr, wd, clip):
        """Like train_step, but returns (status, loss) without raising."""
        B, T = tokens.shape
        loss = ctypes.c_float(0)
        s = gpt_train_step(self.h, _ptr(params), _ptr(grads), _ptr(adam_m), _ptr(adam_v),
                           _ptr(tokens), _ptr(targets), B, T, lr, wd, clip, ctypes.byref(loss))
        return s, loss.value

    @property
    def step(self) -> int:
        v = ctypes.c_long(0)
        self._check(gpt_get_step(self.h, ctypes.byref(v)), "gpt_get_step")
        return v.value

    @step.setter
    def step(self, value: int):
        self._check(gpt_set_step(self.h, value), "gpt_set_step")

    def last_grad_norm(self) -> float:
        return float(gpt_last_grad_norm(self.h))

    def params_changed(self):
        self._check(gpt_params_changed(self.h), "gpt_params_changed")

    def set_option(self, opt: int, value: int):
        self._check(gpt_set_option(self.h, opt, value), "gpt_set_option")

    def kernel_stats(self, reset: bool = False, kind: int = 0):
        n = ctypes.c_longlong(0)
        ms = ctypes.c_double(0)
        fl = ctypes.c_double(0)
        self._check(gpt_kernel_stats(self.h, kind, ctypes.byref(n), ctypes.byref(ms),
                                     ctypes.byref(fl), int(reset)), "gpt_kernel_stats")
        return n.value, ms.value, fl.value

    def all_kernel_stats(self, reset: bool = True):
        """{name: (launches, ms, work, unit)} for every kernel class; clears them if reset."""
        out = {}
        for k, name, unit in KSTATS:
            n, ms, w = self.kernel_stats(kind=k)
            out[name] = (n, ms, w, unit)
        if reset:
            self.kernel_stats(reset=True)
        return out

    def last_launch_count(self) -> int:
        return int(gpt_last_launch_count(self.h))
