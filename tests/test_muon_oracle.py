"""Pins of the oracle's hybrid Muon + AdamW update (oracle/muon_oracle.cpp) against what the
page and the mathematics fix (nanochat architecture page, "Optimierungsstrategien Muon und
AdamW"), and of the two independent constructions of the Polar Express coefficient table
(the oracle's linear programme, the library's Remez exchange)."""
import numpy as np
import pytest

import oracle
from gpt_transformer_step_b200 import fixtures as fx

SH = fx.ModelShape(vocab=65, vocab_padded=72, n_layer=2, n_head=2, n_embd=64, max_T=16)


@pytest.fixture(scope="module")
def coeffs():
    return oracle.polar_express_coeffs(5)


def _p(cf, x):
    a, b, c = cf
    return a * x + b * x ** 3 + c * x ** 5


def test_coefficients_are_minimax_and_equioscillate(coeffs):
    """Each quintic is the best uniform approximation of 1 on its interval: its error reaches
    +-E with alternating signs at four points (the end points and the critical points of p),
    and nowhere exceeds E; the next interval is [1 - E, 1 + E]."""
    lo, hi = 1e-3, 1.0
    for cf in coeffs:
        a, b, c = cf
        crit = [np.sqrt(z.real) for z in np.roots([5 * c, 3 * b, a])
                if abs(z.imag) < 1e-12 and z.real > 0 and lo < np.sqrt(z.real) < hi]
        pts = np.array(sorted([lo, hi] + crit))
        assert len(pts) == 4
        err = 1 - _p(cf, pts)
        E = np.abs(err).max()
        assert np.all(np.sign(err[1:]) == -np.sign(err[:-1]))  # alternation
        # level: the test's interval follows the continuous error, the construction's the
        # grid's, which moves the end points by ~1e-4 E
        assert np.abs(np.abs(err) - E).max() <= 2e-3 * E
        grid = np.linspace(lo, hi, 200001)
        assert np.abs(1 - _p(cf, grid)).max() <= E * (1 + 1e-6)
        lo, hi = 1 - E, 1 + E
    # five steps take every singular value in [1e-3, 1] to within 12% of 1
    x = np.geomspace(1e-3, 1.0, 10001)
    for cf in coeffs:
        x = _p(cf, x)
    assert np.abs(x - 1).max() < 0.12


def test_library_coefficients_match_the_oracle_construction(coeffs):
    """The library's Remez construction agrees with the oracle's linear programme."""
    from gpt_transformer_step_b200.muon import polar_express_coeffs
    assert np.abs(polar_express_coeffs(5) - coeffs).max() <= 1e-4 * np.abs(coeffs).max()


@pytest.mark.parametrize("r,c", [(48, 80), (96, 40), (64, 64)])
def test_polar_express_acts_on_singular_values(coeffs, r, c):
    """X = U diag(s) V^T  ->  U diag(f(s / (||s||_2 * 1.01 + 1e-6))) V^T with f the composed
    quintics: the iteration keeps the singular vectors and maps each singular value by the
    scalar polynomials (tall and wide branches, and a square matrix)."""
    rng = np.random.default_rng(r * 1000 + c)
    k = min(r, c)
    U, _ = np.linalg.qr(rng.standard_normal((r, k)))
    V, _ = np.linalg.qr(rng.standard_normal((c, k)))
    s = np.geomspace(1e-2, 3.0, k)
    X = U @ np.diag(s) @ V.T
    o = oracle.Oracle.from_shape(SH)
    Y = o.polar_express(X, coeffs)
    t = s / (np.sqrt((s ** 2).sum()) * 1.01 + 1e-6)
    for cf in coeffs:
        t = _p(cf, t)
    ref = U @ np.diag(t) @ V.T
    assert np.abs(Y - ref).max() <= 1e-9 * np.abs(ref).max()


def _step(p, g, m, v, coeffs, **kw):
    o = oracle.Oracle.from_shape(SH)
    args = dict(lr=1e-3, wd=0.1, step=1, clip=1e9, matrix_lr=0.02, muon_wd=0.0, mu=0.95,
                beta2_muon=0.95)
    args.update(kw)
    return o.muon_adamw(p, g, m, v, coeffs=coeffs, **args), o


def test_first_step_momentum_second_moment_and_update_shape(coeffs):
    """Step 1 from zero state: buf = (1 - mu) g; the update direction is the Polar Express of
    (1 - mu^2) g, rescaled per row (rows > cols) or per column so that every row (column) of
    the update has the same norm, with the Frobenius norm of that Polar Express output."""
    rng = np.random.default_rng(0)
    p0 = fx.init_params(SH, 0).astype(np.float64)
    g = rng.standard_normal(p0.size) * 1e-2
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    mu, lr = 0.95, 0.02
    _, o = _step(p, g, m, v, coeffs, matrix_lr=lr, mu=mu)
    for off, r, c in o.matrices():
        n = r * c
        assert np.allclose(m[off:off + n], (1 - mu) * g[off:off + n], rtol=1e-13, atol=0)
        X = o.polar_express((1 - mu * mu) * g[off:off + n].reshape(r, c), coeffs)
        D = (p0[off:off + n] - p[off:off + n]).reshape(r, c) / lr  # the update (wd = 0)
        assert np.all(np.sign(D) == np.sign(X))  # a positive scale per line
        ratio = D / X
        lines = ratio if r > c else ratio.T
        assert np.abs(lines - lines[:, :1]).max() <= 1e-9 * np.abs(lines).max()
        norms = np.linalg.norm(D, axis=1 if r > c else 0)
        assert np.abs(norms - norms[0]).max() <= 1e-9 * norms[0]
        assert abs(np.linalg.norm(D) - np.linalg.norm(X)) <= 1e-9 * np.linalg.norm(X)


def test_zero_gradient_is_pure_decay(coeffs):
    """g = 0: Muon's update is 0, so every matrix element gets the cautious decay
    (0 * W >= 0) and every other element AdamW's decoupled decay: p * (1 - lr * wd)."""
    p0 = fx.init_params(SH, 1).astype(np.float64)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    norm, o = _step(p, np.zeros_like(p0), m, v, coeffs, lr=1e-3, wd=0.1, matrix_lr=0.02,
                    muon_wd=0.5)
    assert norm == 0.0
    mask = np.zeros(p0.size, bool)
    for off, r, c in o.matrices():
        mask[off:off + r * c] = True
    assert np.allclose(p[mask], p0[mask] * (1 - 0.02 * 0.5), rtol=1e-15, atol=0)
    assert np.allclose(p[~mask], p0[~mask] * (1 - 1e-3 * 0.1), rtol=1e-15, atol=0)


def test_cautious_decay_only_where_update_and_weight_agree(coeffs):
    """The weight-decay term is the difference of two runs that differ only in Muon's wd: it
    is -lr * wd * W exactly where update * W >= 0 and zero elsewhere."""
    rng = np.random.default_rng(2)
    p0 = fx.init_params(SH, 2).astype(np.float64)
    g = rng.standard_normal(p0.size) * 1e-2
    runs = []
    for wd in (0.0, 0.3):
        p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
        _, o = _step(p, g, m, v, coeffs, muon_wd=wd)
        runs.append(p)
    lr = 0.02
    for off, r, c in o.matrices():
        sl = slice(off, off + r * c)
        u = (p0[sl] - runs[0][sl]) / lr           # the update direction
        decay = runs[1][sl] - runs[0][sl]
        on = u * p0[sl] >= 0
        assert on.any() and (~on).any()
        assert np.allclose(decay[on], -lr * 0.3 * p0[sl][on], rtol=1e-9, atol=1e-18)
        assert np.all(decay[~on] == 0)


def test_adamw_part_equals_the_pinned_adamw(coeffs):
    """Outside the matrices the hybrid step is the oracle's AdamW with the same clip."""
    rng = np.random.default_rng(3)
    p0 = fx.init_params(SH, 3).astype(np.float64)
    g = rng.standard_normal(p0.size) * 1e-1
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    norm, o = _step(p, g, m, v, coeffs, clip=0.5, step=3)
    coef = min(1.0, 0.5 / (np.linalg.norm(g) + 1e-6))
    assert abs(norm - np.linalg.norm(g)) <= 1e-12 * norm
    pa, ma, va = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    o.adamw(pa, g, ma, va, 1e-3, 0.1, 3, coef=coef)
    mask = np.zeros(p0.size, bool)
    for off, r, c in o.matrices():
        mask[off:off + r * c] = True
    # (the norm is summed in another order than np.linalg.norm: the clip coefficient differs in
    # the last bits)
    assert np.abs(p[~mask] - pa[~mask]).max() <= 1e-13 * np.abs(pa).max()
    assert np.abs(m[~mask] - ma[~mask]).max() <= 1e-13 * np.abs(ma).max()


def _bf16(a):
    """Round float64 values to bf16 (nearest even) through float32, with numpy bit operations."""
    u = np.asarray(a, np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return u.view(np.float32).astype(np.float64)


def test_bf16_mode_rounds_the_stored_matrices():
    """With (a, b, c) = (1, 0, 0) the iteration stores X' = 1 X + 0: at bf16 the result is the
    normalised input (scale taken in float) rounded once to bf16."""
    rng = np.random.default_rng(5)
    X = rng.standard_normal((40, 72))
    o = oracle.Oracle.from_shape(SH)
    Y = o.polar_express(X, np.array([[1.0, 0.0, 0.0]]), bf16=True)
    scale = np.float32(1.0 / (np.sqrt((X ** 2).sum()) * 1.01 + 1e-6))
    assert np.array_equal(Y, _bf16(X * np.float64(scale)))
