"""The hybrid Muon + AdamW update on the GPU (gpt_muon_update, tensor-core Polar Express
batched over layers) against the oracle on the same gradients and state, for two
consecutive steps.

The oracle runs the iteration at the page's precision (X = g.bfloat16(); every matrix the
iteration stores rounded to bf16 once formed, products and sums exact before that): the GPU
differs from it only by fp32 accumulation order inside the GEMMs, which flips the bf16
rounding of a small fraction of the stored elements by one unit (2^-8 relative); the first
Polar Express step (a = 8.5, b = -25, c = 19) amplifies such flips, so the matrix update is
checked at cosine >= 0.999 and relative Frobenius error <= 3e-2 per matrix, the factored
second moment at 3e-2 relative. The distance to the exact (double) iteration is printed. The
AdamW part runs in fp32 on the same inputs: the spec update bound, max |dp| <= 2e-2 * lr;
the momentum buffer is fp32 arithmetic on the same inputs: 1e-6 relative.
"""
import numpy as np
import pytest

import oracle
from gpt_transformer_step_b200 import fixtures as fx
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

SH = fx.ModelShape(vocab=1000, vocab_padded=1024, n_layer=2, n_head=2, n_embd=128, max_T=64)
LR, WD, CLIP = 6e-4, 0.1, 1.0
MATRIX_LR, MUON_WD = 0.02, 0.05


def test_muon_update_matches_oracle_two_steps():
    import torch
    from gpt_transformer_step_b200.muon import MuonConfig
    rng = np.random.default_rng(7)
    p0 = fx.init_params(SH, 7).astype(np.float64)
    o = oracle.Oracle.from_shape(SH)
    cf_oracle = oracle.polar_express_coeffs(5)
    mc = MuonConfig(matrix_lr=MATRIX_LR, weight_decay=MUON_WD)
    dev = torch.device("cuda", 0)
    st = U.make_step(SH, 2, 64, 1)
    st.use_current_torch_stream()
    P = torch.from_numpy(p0.astype(np.float32)).to(dev)
    M = torch.zeros_like(P)
    V = torch.zeros_like(P)
    po, mo, vo = p0.astype(np.float32).astype(np.float64), np.zeros_like(p0), np.zeros_like(p0)
    mats = o.matrices()
    in_mat = np.zeros(p0.size, bool)
    for off, r, c in mats:
        in_mat[off:off + r * c] = True
    for step in (1, 2):
        g = (rng.standard_normal(p0.size) * 2e-2).astype(np.float32)
        G = torch.from_numpy(g).to(dev)
        p_before = po.copy()
        st.muon_update(P, G, M, V, LR, WD, CLIP, mc)
        torch.cuda.synchronize()
        assert st.step == step
        pe, me, ve = po.copy(), mo.copy(), vo.copy()  # the exact iteration, for the report
        o.muon_adamw(pe, g.astype(np.float64), me, ve, lr=LR, wd=WD, step=step, clip=CLIP,
                     coeffs=cf_oracle, matrix_lr=MATRIX_LR, muon_wd=MUON_WD)
        o.muon_adamw(po, g.astype(np.float64), mo, vo, lr=LR, wd=WD, step=step, clip=CLIP,
                     coeffs=cf_oracle, matrix_lr=MATRIX_LR, muon_wd=MUON_WD, bf16=True)
        Pg, Mg, Vg = P.cpu().numpy().astype(np.float64), M.cpu().numpy(), V.cpu().numpy()
        # AdamW part
        assert np.abs(Pg[~in_mat] - po[~in_mat]).max() <= 2e-2 * LR
        assert np.abs(Mg[~in_mat] - mo[~in_mat]).max() <= 1e-6 * np.abs(mo[~in_mat]).max()
        # Muon part, per matrix
        for off, r, c in mats:
            sl = slice(off, off + r * c)
            assert np.abs(Mg[sl] - mo[sl]).max() <= 1e-6 * np.abs(mo[sl]).max()
            d_gpu, d_ref = Pg[sl] - p_before[sl], po[sl] - p_before[sl]
            d_ex = pe[sl] - p_before[sl]
            cos = U.cosine(d_gpu, d_ref)
            rel = np.linalg.norm(d_gpu - d_ref) / np.linalg.norm(d_ref)
            rel_ex = np.linalg.norm(d_gpu - d_ex) / np.linalg.norm(d_ex)
            print(f"step {step} matrix {r}x{c}: vs bf16 oracle cosine {cos:.6f} rel {rel:.3e}; "
                  f"vs exact iteration rel {rel_ex:.3e}")
            assert cos >= 0.999 and rel <= 3e-2, (step, r, c, cos, rel)
            nl = r if r > c else c
            s_gpu, s_ref = Vg[off:off + nl], vo[off:off + nl]
            assert np.abs(s_gpu - s_ref).max() <= 3e-2 * np.abs(s_ref).max()
        # reset to the oracle's state so the next step compares like with like
        P.copy_(torch.from_numpy(po.astype(np.float32)))
        M.copy_(torch.from_numpy(mo.astype(np.float32)))
        V.copy_(torch.from_numpy(vo.astype(np.float32)))
        po = po.astype(np.float32).astype(np.float64)
        mo = mo.astype(np.float32).astype(np.float64)
        vo = vo.astype(np.float32).astype(np.float64)
        st.params_changed()
    st.close()


def test_muon_update_deterministic_and_nonfinite_skips():
    import torch
    from gpt_transformer_step_b200.muon import MuonConfig
    dev = torch.device("cuda", 0)
    p0 = fx.init_params(SH, 8)
    g = (np.random.default_rng(8).standard_normal(p0.size) * 1e-2).astype(np.float32)
    outs = []
    for _ in range(2):
        st = U.make_step(SH, 2, 64, 1)
        st.use_current_torch_stream()
        P = torch.from_numpy(p0).to(dev)
        M, V = torch.zeros_like(P), torch.zeros_like(P)
        st.muon_update(P, torch.from_numpy(g).to(dev), M, V, LR, WD, CLIP, MuonConfig())
        torch.cuda.synchronize()
        outs.append((P.cpu(), M.cpu(), V.cpu()))
        # a non-finite gradient: nothing changes, the step counter stays
        gb = g.copy()
        gb[5] = np.inf
        P0, M0, V0 = P.clone(), M.clone(), V.clone()
        from gpt_transformer_step_b200 import binding as b
        with pytest.raises(b.GPTError) as e:
            st.muon_update(P, torch.from_numpy(gb).to(dev), M, V, LR, WD, CLIP, MuonConfig())
        assert e.value.status == b.GPT_ERR_NONFINITE
        torch.cuda.synchronize()
        assert torch.equal(P, P0) and torch.equal(M, M0) and torch.equal(V, V0)
        assert st.step == 1
        st.close()
    assert all(torch.equal(a, b) for a, b in zip(outs[0], outs[1]))


def test_muon_full_size_124m_step():
    """GPT-2 124M: forward/backward then the Muon update on the real gradients; finite, and
    the matrices' updates have the per-line structure of the factored second moment."""
    import torch
    from gpt_transformer_step_b200.muon import MuonConfig
    wl = fx.WORKLOADS["gpt2_124m_bf16"]
    p, tok, tgt = fx.make_inputs(wl)
    dev = torch.device("cuda", 0)
    st = U.make_step(wl.shape, wl.B, wl.T, 1)
    st.use_current_torch_stream()
    P = torch.from_numpy(p).to(dev)
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    loss = st.forward_backward(P, G, torch.from_numpy(tok).to(dev), torch.from_numpy(tgt).to(dev))
    assert np.isfinite(loss)
    P0 = P.clone()
    st.muon_update(P, G, M, V, wl.lr, wl.wd, wl.clip, MuonConfig())
    torch.cuda.synchronize()
    d = (P - P0).cpu().numpy()
    assert np.isfinite(d).all()
    o = oracle.Oracle.from_shape(wl.shape)
    for off, r, c in o.matrices()[:4]:
        D = d[off:off + r * c].reshape(r, c)
        norms = np.linalg.norm(D, axis=1 if r > c else 0)
        # equal line norms up to bf16 rounding of the iterate (the step-1 property)
        assert np.abs(norms - norms.mean()).max() <= 2e-2 * norms.mean(), (r, c)
    st.close()
