"""The seeded generators shared by both sides of every parity test (CPU only)."""
import math
import os

import numpy as np

from gpt_transformer_step_b200 import fixtures as fx

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_published_vector():
    vals = [int(l) for l in open(os.path.join(GOLD, "splitmix64_seed1234567.txt"))
            if l.strip() and not l.startswith("#")]
    assert [int(x) for x in fx.splitmix64(np.uint64(1234567), 0, 5)] == vals


def test_counter_based_slices_agree():
    k = fx.stream_key(7, "init")
    a = fx.splitmix64(k, 0, 100)
    assert np.array_equal(a[40:60], fx.splitmix64(k, 40, 20))


def test_normals_moments():
    z = fx.normals(fx.stream_key(0, "misc"), 400_000)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3


def test_zipf_frequencies_follow_power_law():
    V, s = 1000, 1.05
    tok, tgt = fx.zipf_tokens(V, s, 64, 1024, seed=0)
    assert tok.min() >= 0 and tok.max() < V
    # inputs/targets are one sequence shifted by one position
    assert np.array_equal(tok[:, 1:], tgt[:, :-1])
    h = np.bincount(tok.ravel(), minlength=V) / tok.size
    w = np.arange(1, V + 1) ** -s
    w /= w.sum()
    assert abs(h[0] - w[0]) < 0.01 and abs(h[1] - w[1]) < 0.01
    assert abs(h[:10].sum() - w[:10].sum()) < 0.01


def test_init_statistics_and_padding():
    sh = fx.WORKLOADS["shakespeare_char_bf16"].shape
    p = fx.init_params(sh)
    lay = {n: (o, s, sd) for n, o, s, sd in fx.param_layout(sh)}
    o, s, sd = lay["h0.w_qkv"]
    w = p[o:o + int(np.prod(s))]
    assert abs(w.std() - 0.02) < 2e-4
    o, s, sd = lay["h0.w_mlpproj"]
    w = p[o:o + int(np.prod(s))]
    assert abs(w.std() - 0.02 / math.sqrt(12)) < 1e-4
    o, s, sd = lay["h3.ln2.g"]
    assert np.all(p[o:o + s[0]] == 1.0)
    sh2 = fx.ModelShape(10, 16, 1, 1, 8, 4)
    p2 = fx.init_params(sh2)
    assert np.all(p2[10 * 8:16 * 8] == 0)


def test_flops_formula_counts():
    # 6*(N - wpe) + sum_l 12*H*hd*min(window, T)
    wl = fx.WORKLOADS["gpt2_124m_bf16"]
    n = fx.num_params(wl.shape)
    assert fx.flops_per_token(wl.shape, 1024) == 6 * (n - 1024 * 768) + 12 * 12 * 12 * 64 * 1024
    sw = fx.WORKLOADS["gpt2_124m_swa_bf16"]
    attn = sum(12 * 12 * 64 * (2048 if w < 0 else 512) for w in sw.shape.windows())
    assert fx.flops_per_token(sw.shape, 2048) == 6 * (fx.num_params(sw.shape) - 2048 * 768) + attn
