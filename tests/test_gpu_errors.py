"""Error paths and step properties through the C ABI on the GPU: bad ids, shape and
alignment checks, non-finite parameters (update skipped, state unchanged), resume,
CUDA-graph replay vs eager launch, host vs device token buffers, and the bounded-wait
timeout status."""
import numpy as np
import pytest

from gpt_transformer_step_b200 import fixtures as fx
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

SH = fx.ModelShape(vocab=500, vocab_padded=512, n_layer=2, n_head=2, n_embd=128, max_T=64)


def _setup(precision=1, B=2, T=64, seed=0):
    import torch
    from gpt_transformer_step_b200 import binding as gb
    st = U.make_step(SH, B, T, precision)
    st.use_current_torch_stream()
    p = fx.init_params(SH, seed)
    tok, tgt = fx.zipf_tokens(SH.vocab, 1.05, B, T, seed)
    dev = torch.device("cuda", 0)
    P = torch.from_numpy(p).to(dev)
    bufs = [torch.zeros_like(P) for _ in range(3)]
    return torch, gb, st, P, bufs, torch.from_numpy(tok).to(dev), torch.from_numpy(tgt).to(dev)


@pytest.mark.parametrize("n_micro", [1, 2])
def test_bad_token_and_target_ids(n_micro):
    """An id out of range is reported and skips the update: params, m, v and the step counter
    stay bitwise unchanged (as for a non-finite loss), for one step and an accumulated one."""
    torch, gb, st, P, (G, M, V), tk, tg = _setup()
    # non-zero optimizer state, so an update that slipped through would show
    st.train_step(P, G, M, V, tk, tg, 1e-3, 0.1, 1.0)
    torch.cuda.synchronize()
    step0 = st.step
    tkn = tk.unsqueeze(0).repeat(n_micro, 1, 1).contiguous()
    tgn = tg.unsqueeze(0).repeat(n_micro, 1, 1).contiguous()

    def call(a, b):
        if n_micro == 1:
            return st.train_step_status(P, G, M, V, a[0], b[0], 1e-3, 0.1, 1.0)[0]
        try:
            st.train_step_accum(P, G, M, V, a, b, 1e-3, 0.1, 1.0)
            return 0
        except gb.GPTError as e:
            return e.status

    for which in ("token", "target"):
        P0, M0, V0 = P.clone(), M.clone(), V.clone()
        a, b = tkn.clone(), tgn.clone()
        if which == "token":
            a[n_micro - 1, 0, 3] = SH.vocab  # == V: outside the softmax vocabulary
        else:
            b[n_micro - 1, 1, 0] = -1
        assert call(a, b) == gb.GPT_ERR_BAD_TOKEN
        torch.cuda.synchronize()
        assert torch.equal(P, P0) and torch.equal(M, M0) and torch.equal(V, V0), which
        assert st.step == step0
    # a good step still works afterwards and uses the unchanged state
    Pr, Mr, Vr = P.clone(), M.clone(), V.clone()
    assert call(tkn, tgn) == 0 and st.step == step0 + 1
    torch.cuda.synchronize()
    assert not torch.equal(P, Pr)
    # the bf16 weight copy was not touched by the failed calls: a fresh handle from the same
    # state gives the same update
    st2 = U.make_step(SH, 2, 64, 1)
    st2.use_current_torch_stream()
    st2.step = step0
    P2, M2, V2 = Pr.clone(), Mr.clone(), Vr.clone()
    if n_micro == 1:
        st2.train_step(P2, G, M2, V2, tk, tg, 1e-3, 0.1, 1.0)
    else:
        st2.train_step_accum(P2, G, M2, V2, tkn, tgn, 1e-3, 0.1, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(P2, P) and torch.equal(M2, M) and torch.equal(V2, V)
    st2.close()


def test_shape_alignment_and_argument_checks():
    torch, gb, st, P, (G, M, V), tk, tg = _setup()
    big = torch.zeros(3, 64, dtype=torch.int32, device=tk.device)  # B > max_B
    s, _ = st.train_step_status(P, G, M, V, big, big, 1e-3, 0.0, 1.0)
    assert s == gb.GPT_ERR_SHAPE
    long_ = torch.zeros(1, 65, dtype=torch.int32, device=tk.device)  # T > max_T
    s, _ = st.train_step_status(P, G, M, V, long_, long_, 1e-3, 0.0, 1.0)
    assert s == gb.GPT_ERR_SHAPE
    Pm = torch.zeros(P.numel() + 1, device=P.device)[1:]  # 4-byte, not 16-byte aligned
    s, _ = st.train_step_status(Pm, G, M, V, tk, tg, 1e-3, 0.0, 1.0)
    assert s == gb.GPT_ERR_ALIGN
    s, _ = st.train_step_status(P, G, M, V, tk, tg, 1e-3, 0.0, 0.0)  # clip must be > 0
    assert s == gb.GPT_ERR_INVALID_ARG
    s, _ = st.train_step_status(P, G, M, V, tk, tg, float("nan"), 0.0, 1.0)
    assert s == gb.GPT_ERR_INVALID_ARG


def test_nonfinite_params_skip_the_update():
    torch, gb, st, P, (G, M, V), tk, tg = _setup()
    P[123] = float("nan")
    P0, M0, V0 = P.clone(), M.clone(), V.clone()
    s, loss = st.train_step_status(P, G, M, V, tk, tg, 1e-3, 0.1, 1.0)
    assert s == gb.GPT_ERR_NONFINITE
    torch.cuda.synchronize()
    assert torch.equal(P.nan_to_num(7.0), P0.nan_to_num(7.0))
    assert torch.equal(M, M0) and torch.equal(V, V0)
    assert st.step == 0


@pytest.mark.parametrize("precision", [0, 1])
def test_resume_equals_uninterrupted(precision):
    torch, gb, st, P, (G, M, V), tk, tg = _setup(precision)
    Pa, Ma, Va = P.clone(), M.clone(), V.clone()
    for _ in range(3):
        st.train_step(Pa, G, Ma, Va, tk, tg, 1e-3, 0.1, 1.0)
    # two steps, "checkpoint" (host copies + step counter), new handle, one more step
    Pb, Mb, Vb = P.clone(), M.clone(), V.clone()
    st.step = 0
    for _ in range(2):
        st.train_step(Pb, G, Mb, Vb, tk, tg, 1e-3, 0.1, 1.0)
    ck = [t.cpu() for t in (Pb, Mb, Vb)], st.step
    st2 = U.make_step(SH, 2, 64, precision)
    st2.use_current_torch_stream()
    Pc, Mc, Vc = (t.to(P.device) for t in ck[0])
    st2.step = ck[1]
    st2.train_step(Pc, G, Mc, Vc, tk, tg, 1e-3, 0.1, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(Pc, Pa) and torch.equal(Mc, Ma) and torch.equal(Vc, Va)


def test_graph_replay_matches_eager_and_host_tokens():
    torch, gb, st, P, (G, M, V), tk, tg = _setup()
    stream = torch.cuda.Stream()
    outs = []
    for graphs, host in ((1, False), (0, False), (1, True)):
        st.set_option(gb.GPT_OPT_USE_GRAPHS, graphs)
        st.step = 0
        Pq, Mq, Vq, Gq = P.clone(), M.clone(), V.clone(), G.clone()
        a, b = (tk.cpu().pin_memory(), tg.cpu().pin_memory()) if host else (tk, tg)
        with torch.cuda.stream(stream):
            st.set_stream(stream.cuda_stream)
            losses = [st.train_step(Pq, Gq, Mq, Vq, a, b, 1e-3, 0.1, 1.0) for _ in range(2)]
        torch.cuda.synchronize()
        outs.append((losses, Pq, Gq))
    for losses, Pq, Gq in outs[1:]:
        assert losses == outs[0][0]
        assert torch.equal(Pq, outs[0][1]) and torch.equal(Gq, outs[0][2])


def test_bounded_wait_times_out_and_context_survives():
    import torch
    from gpt_transformer_step_b200 import binding as gb
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert gb.gptk_selftest_bounded_wait(20000, err.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 2  # GPT_DEVERR_TIMEOUT
    x = torch.arange(10, device="cuda").sum().item()  # the context still works
    assert x == 45

