"""Host-side settings of the hybrid Muon + AdamW update (gpt_muon_update in the C ABI).

nanochat architecture page, section "Optimierungsstrategien Muon und AdamW": Muon for the 2-D
matrices of the blocks, AdamW for the embeddings, the lm_head and the 0-D/1-D parameters;
the Muon update is orthogonalised by the Polar Express iteration ("Polar Express Details"),
whose coefficient table the page refers to but does not print.

`polar_express_coeffs` constructs that table the way the Polar Express method defines it:
step t uses the odd quintic p(x) = a x + b x^3 + c x^5 that minimises max |1 - p(x)| over the
interval [lo_t, hi_t] the singular values can be in, and the next interval is the image of
that one, [1 - E_t, 1 + E_t] with E_t the minimax error. Each minimax problem is solved with
the Remez exchange: the best approximation equioscillates at four points (three
coefficients), found by solving for the coefficients on a reference set and moving the
reference to the extrema of the error until they level.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Tuple

import numpy as np


def _minimax_odd_quintic(lo: float, hi: float, iters: int = 200) -> Tuple[float, float, float, float]:
    """(a, b, c, E): p(x) = a x + b x^3 + c x^5 with the least max |1 - p| on [lo, hi] and E."""
    k = np.arange(4)
    ref = lo + (hi - lo) * (1 - np.cos(np.pi * k / 3)) / 2  # Chebyshev-spaced start
    a = b = c = E = 0.0
    for _ in range(iters):
        m = np.stack([ref, ref ** 3, ref ** 5, (-1.0) ** k], axis=1)
        a, b, c, E = np.linalg.solve(m, np.ones(4))
        # extrema of the error 1 - p(x): the end points and the roots of p'(x) in (lo, hi)
        pts = [lo, hi]
        for z in np.roots([5 * c, 3 * b, a]):
            if abs(z.imag) < 1e-12 and z.real > 0:
                x = float(np.sqrt(z.real))
                if lo < x < hi:
                    pts.append(x)
        pts = np.array(sorted(pts))
        if len(pts) != 4:
            break
        err = 1 - (a * pts + b * pts ** 3 + c * pts ** 5)
        done = np.allclose(np.abs(err), abs(E), rtol=1e-13, atol=0)
        ref = pts
        if done:
            break
    return float(a), float(b), float(c), float(abs(E))


def polar_express_coeffs(steps: int = 5, lo: float = 1e-3) -> np.ndarray:
    """[steps, 3] float64 table of (a, b, c) for singular values starting in [lo, 1]."""
    out: List[Tuple[float, float, float]] = []
    l, h = lo, 1.0
    for _ in range(steps):
        a, b, c, E = _minimax_odd_quintic(l, h)
        out.append((a, b, c))
        l, h = 1 - E, 1 + E
    return np.array(out, dtype=np.float64)


@dataclass
class MuonConfig:
    """Hyper-parameters of the Muon part (the AdamW part takes those of the step)."""
    matrix_lr: float = 0.02      # the page's matrix_lr (Muon learning rate)
    weight_decay: float = 0.0    # the page's Muon weight decay (cautious)
    momentum: float = 0.95       # reading: Muon's usual momentum
    beta2: float = 0.95          # reading: the factored second moment's EMA factor
    eps: float = 1e-10           # reading: floor of the second moment
    ns_steps: int = 5            # the page: five iterations
    coeffs: np.ndarray = field(default_factory=lambda: polar_express_coeffs(5))
