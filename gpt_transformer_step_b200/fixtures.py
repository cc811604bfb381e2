"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle's tests.

This module holds none of the model's arithmetic: it only draws random numbers and lays
them out. Both sides of a parity test receive the very same host buffers from here.

Generators (all counter-based, so any element can be drawn independently):

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
  OOPSLA 2014; Vigna's public-domain reference): the i-th output of stream key k is
  mix(k + (i + 1) * 0x9E3779B97F4A7C15) with the published 3-step xor-shift-multiply mix.
* Uniform doubles in [0, 1): the top 53 bits of a SplitMix64 output times 2^-53.
* Normals: Box-Muller on consecutive pairs of uniforms (counters 2j, 2j+1).
* Zipf token ids: inverse CDF of P(id k) proportional to (k+1)^-s over k in [0, V),
  built in float64 and searched with a binary search (numpy.searchsorted).

Stream keys: key(seed, stream) = mix(seed * GOLDEN + STREAM_ID[stream]) so that "init" and
"tokens" never share counters.

Workload presets follow the five model shapes the nanoGPT README (quick start,
"reproducing GPT-2"), the llm.c summary ("Modelo 350M") and the nanochat architecture
page (sliding window, "Modellarchitektur und FLOPs-Berechnung") describe.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
STREAM_ID = {"init": 1, "tokens": 2, "perturb": 3, "misc": 4}


def _mix(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: str) -> np.uint64:
    with np.errstate(over="ignore"):
        k = np.uint64(seed) * GOLDEN + np.uint64(STREAM_ID[stream])
    return _mix(np.array([k], dtype=np.uint64))[0]


def splitmix64(key: np.uint64, start: int, n: int) -> np.ndarray:
    """Outputs start..start+n-1 of the SplitMix64 sequence whose state starts at `key`."""
    ctr = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(np.uint64(key) + ctr * GOLDEN)


def uniform01(key: np.uint64, start: int, n: int) -> np.ndarray:
    return (splitmix64(key, start, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normals(key: np.uint64, n: int, chunk: int = 1 << 24) -> np.ndarray:
    """n standard normals from Box-Muller over pairs (u1, u2) = (U[2j], U[2j+1])."""
    out = np.empty(n, dtype=np.float64)
    npairs = (n + 1) // 2
    done = 0
    for p0 in range(0, npairs, chunk):
        p1 = min(npairs, p0 + chunk)
        u = uniform01(key, 2 * p0, 2 * (p1 - p0))
        u1, u2 = u[0::2], u[1::2]
        r = np.sqrt(-2.0 * np.log1p(-u1))  # 1-u1 in (0, 1]: log is finite
        th = 2.0 * math.pi * u2
        z = np.empty(2 * (p1 - p0), dtype=np.float64)
        z[0::2] = r * np.cos(th)
        z[1::2] = r * np.sin(th)
        take = min(len(z), n - done)
        out[done:done + take] = z[:take]
        done += take
    return out


# ---------------------------------------------------------------------------
# Model shapes and the flat parameter layout
# ---------------------------------------------------------------------------

@dataclass
class ModelShape:
    vocab: int
    vocab_padded: int
    n_layer: int
    n_head: int
    n_embd: int
    max_T: int
    mlp_mult: int = 4
    window_left: List[int] = field(default_factory=list)  # per layer; -1 = full causal

    def windows(self) -> List[int]:
        if self.window_left:
            assert len(self.window_left) == self.n_layer
            return list(self.window_left)
        return [-1] * self.n_layer


@dataclass
class Workload:
    name: str
    shape: ModelShape
    B: int
    T: int
    zipf_s: float
    lr: float
    wd: float
    clip: float
    precision: str  # "fp32" | "bf16"
    beta1: float = 0.9
    beta2: float = 0.95
    adam_eps: float = 1e-8
    ln_eps: float = 1e-5


def param_layout(sh: ModelShape) -> List[Tuple[str, int, Tuple[int, ...], float]]:
    """(name, offset, shape, init std) in flat order; std 0 means 'ones' (LayerNorm gain).

    Order: wte [Vp,C], wpe [max_T,C], per layer (ln1.g, w_qkv [3C,C], w_attnproj [C,C],
    ln2.g, w_fc [mC,C], w_mlpproj [C,mC]), lnf.g. Weights are row-major [out, in].
    """
    C, m = sh.n_embd, sh.mlp_mult
    std = 0.02
    std_res = 0.02 / math.sqrt(2.0 * sh.n_layer)
    items: List[Tuple[str, Tuple[int, ...], float]] = [
        ("wte", (sh.vocab_padded, C), std),
        ("wpe", (sh.max_T, C), std),
    ]
    for l in range(sh.n_layer):
        items += [
            (f"h{l}.ln1.g", (C,), 0.0),
            (f"h{l}.w_qkv", (3 * C, C), std),
            (f"h{l}.w_attnproj", (C, C), std_res),
            (f"h{l}.ln2.g", (C,), 0.0),
            (f"h{l}.w_fc", (m * C, C), std),
            (f"h{l}.w_mlpproj", (C, m * C), std_res),
        ]
    items.append(("lnf.g", (C,), 0.0))
    out, off = [], 0
    for name, shp, s in items:
        out.append((name, off, shp, s))
        off += int(np.prod(shp))
    return out


def num_params(sh: ModelShape) -> int:
    name, off, shp, _ = param_layout(sh)[-1]
    return off + int(np.prod(shp))


def init_params(sh: ModelShape, seed: int = 0) -> np.ndarray:
    """fp32 flat parameters: N(0, std^2) weights (Box-Muller over one stream, drawn in
    layout order, row-major), LayerNorm gains 1, padded vocab rows (>= vocab) 0."""
    lay = param_layout(sh)
    n = num_params(sh)
    p = np.zeros(n, dtype=np.float32)
    need = 0
    for name, off, shp, s in lay:
        if s == 0.0:
            continue
        cnt = int(np.prod(shp))
        if name == "wte":
            cnt = sh.vocab * sh.n_embd
        need += cnt
    z = normals(stream_key(seed, "init"), need)
    k = 0
    for name, off, shp, s in lay:
        cnt = int(np.prod(shp))
        if s == 0.0:
            p[off:off + cnt] = 1.0
            continue
        if name == "wte":
            cnt = sh.vocab * sh.n_embd
        p[off:off + cnt] = (z[k:k + cnt] * s).astype(np.float32)
        k += cnt
    return p


def zipf_cdf(V: int, s: float) -> np.ndarray:
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def zipf_tokens(V: int, s: float, B: int, T: int, seed: int = 0,
                stream: str = "tokens") -> Tuple[np.ndarray, np.ndarray]:
    """B rows of T+1 i.i.d. Zipf ids; inputs = row[:T], targets = row[1:]."""
    u = uniform01(stream_key(seed, stream), 0, B * (T + 1))
    ids = np.searchsorted(zipf_cdf(V, s), u, side="right").astype(np.int64)
    ids = np.minimum(ids, V - 1).astype(np.int32).reshape(B, T + 1)
    return np.ascontiguousarray(ids[:, :T]), np.ascontiguousarray(ids[:, 1:])


# ---------------------------------------------------------------------------
# Workload presets
# ---------------------------------------------------------------------------

def _alternating(n_layer: int, w: int) -> List[int]:
    # Layer 0 carries the window, layer 1 is full causal, and so on.
    return [w if l % 2 == 0 else -1 for l in range(n_layer)]


WORKLOADS: Dict[str, Workload] = {
    "tiny_char_fp32": Workload(
        "tiny_char_fp32", ModelShape(65, 65, 2, 2, 64, 32), B=4, T=32, zipf_s=1.1,
        lr=1e-3, wd=0.01, clip=1.0, precision="fp32"),
    "shakespeare_char_bf16": Workload(
        "shakespeare_char_bf16", ModelShape(65, 65, 6, 6, 384, 256), B=64, T=256,
        zipf_s=1.1, lr=1e-4, wd=0.01, clip=1.0, precision="bf16"),
    "gpt2_124m_bf16": Workload(
        "gpt2_124m_bf16", ModelShape(50257, 50304, 12, 12, 768, 1024), B=16, T=1024,
        zipf_s=1.05, lr=6e-4, wd=0.1, clip=1.0, precision="bf16"),
    "gpt2_350m_bf16": Workload(
        "gpt2_350m_bf16", ModelShape(50257, 50304, 24, 16, 1024, 1024), B=8, T=1024,
        zipf_s=1.05, lr=6e-4, wd=0.1, clip=1.0, precision="bf16"),
    "gpt2_124m_swa_bf16": Workload(
        "gpt2_124m_swa_bf16",
        ModelShape(50304, 50304, 12, 12, 768, 2048, window_left=_alternating(12, 512)),
        B=8, T=2048, zipf_s=1.05, lr=6e-4, wd=0.1, clip=1.0, precision="bf16"),
}


def flops_per_token(sh: ModelShape, T: int, exclude: str = "wpe") -> int:
    """Model FLOPs per token: 6*(N - excluded embedding params) + sum over layers of
    12*n_head*head_dim*effective_seq, effective_seq = min(window, T) (nanochat architecture
    page, "FLOPs-Berechnung im Detail"). exclude: "wpe" (tied head counts as a matmul) or
    "wte+wpe" (literal exclusion of both embedding tables)."""
    n = num_params(sh)
    C = sh.n_embd
    ex = sh.max_T * C
    if exclude == "wte+wpe":
        ex += sh.vocab_padded * C
    hd = C // sh.n_head
    attn = 0
    for w in sh.windows():
        eff = T if w < 0 else min(w, T)
        attn += 12 * sh.n_head * hd * eff
    return 6 * (n - ex) + attn


def make_inputs(wl: Workload, seed: int = 0, B: Optional[int] = None, T: Optional[int] = None):
    """(params fp32, tokens int32 [B,T], targets int32 [B,T]) for a workload preset."""
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    p = init_params(wl.shape, seed)
    tok, tgt = zipf_tokens(wl.shape.vocab, wl.zipf_s, B, T, seed)
    return p, tok, tgt
