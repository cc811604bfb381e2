"""Data parallelism with sharded optimizer state (gpt_transformer_step_b200/dp.py).

CPU: the partition's invariants, and two gloo ranks running the data-parallel step with the
oracle doing each rank's arithmetic (test-side only), against the oracle's one-process
gradient-accumulated step over the same micro-batches (rank order): the exchanged gradients
are bitwise those of the accumulated step, parameters and moments agree to rounding of the
norm's summation order. GPU (one rank, NCCL): the library's data-parallel pieces reproduce
gpt_train_step bitwise."""
import math
import os
import socket

import numpy as np
import pytest

from gpt_transformer_step_b200 import fixtures as fx
from gpt_transformer_step_b200.dp import DataParallelStep, Partition

SH = fx.WORKLOADS["tiny_char_fp32"].shape
B, T = 4, 32
LR, WD, CLIP = 1e-3, 0.01, 1.0


@pytest.mark.parametrize("n,world,bucket", [(104832, 2, 1 << 14), (104832, 8, 1 << 20),
                                            (1000, 3, 64), (124373760, 8, 1 << 24)])
def test_partition_covers_every_parameter_once(n, world, bucket):
    p = Partition(n, world, bucket)
    assert p.n_pad % (4 * world) == 0 and p.n_pad >= n and len(p.buckets) <= 64
    assert p.buckets[0][0] == 0 and p.buckets[-1][1] == p.n_pad
    owned = np.zeros(p.n_pad, np.int32)
    for r in range(world):
        sl = p.slices(r)
        assert sum(s for _, s, _ in sl) == p.shard_elems
        for (off, s, base), (b0, b1) in zip(sl, p.buckets):
            assert off % 4 == 0 and s % 4 == 0 and b0 <= off and off + s <= b1
            owned[off:off + s] += 1
        for off, cnt in p.update_ranges(r):
            assert cnt % 4 == 0 and off + cnt <= n
    assert np.all(owned == 1)


class OracleCompute:
    """Each rank's arithmetic done by the oracle (double): test infrastructure only."""

    def __init__(self, sh):
        import oracle
        self.o = oracle.Oracle.from_shape(sh)
        self.n = self.o.n

    def forward_backward(self, params, grads, tokens, targets, grad_scale):
        p = params[:self.n].numpy()
        loss, g = self.o.forward_backward(p, tokens, targets)
        grads[:self.n].copy_(__import__("torch").from_numpy(g * grad_scale))
        return loss

    def sumsq(self, x, out):
        xs = x.numpy()
        out[0] = float(np.sum(xs * xs))

    def adamw_ranges(self, params, grads, m, v, ranges, lr, wd, clip, sumsq, step):
        coef = min(1.0, clip / (math.sqrt(float(sumsq[0])) + 1e-6))
        base = 0
        for off, cnt in ranges:
            self.o.adamw(params.numpy()[off:off + cnt], grads.numpy()[base:base + cnt],
                         m.numpy()[base:base + cnt], v.numpy()[base:base + cnt], lr, wd, step,
                         coef=coef)
            base += cnt

    def params_changed(self):
        pass


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _dp_worker(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        comp = OracleCompute(SH)
        dp = DataParallelStep(comp, comp.n, world, rank, "cpu", dist, bucket_elems=1 << 14)
        P, G, GS, M, V = dp.alloc(fx.init_params(SH, 0), dtype=torch.float64)
        tok, tgt = fx.zipf_tokens(SH.vocab, 1.1, world * B, T, 0)
        losses, gs1 = [], None
        for _ in range(2):
            losses.append(dp.train_step(P, G, GS, M, V, tok[rank * B:(rank + 1) * B],
                                        tgt[rank * B:(rank + 1) * B], LR, WD, CLIP))
            if gs1 is None:
                gs1 = GS.numpy().copy()
        q.put((rank, losses, P[:comp.n].numpy().copy(), gs1, GS.numpy().copy(),
               M.numpy().copy(), V.numpy().copy(), dp.slices, dp.last_norm))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_the_accumulated_oracle_step():
    import oracle
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = q.get(timeout=300)
        res[r[0]] = r
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    # the oracle's accumulated step over the same micro-batches (rank r = micro-batch r)
    o = oracle.Oracle.from_shape(SH)
    p = fx.init_params(SH, 0).astype(np.float64)
    m, v = np.zeros_like(p), np.zeros_like(p)
    tok, tgt = fx.zipf_tokens(SH.vocab, 1.1, world * B, T, 0)
    tok, tgt = tok.reshape(world, B, T), tgt.reshape(world, B, T)
    ref_losses, ref_norm, g1 = [], None, None
    for step in (1, 2):
        loss, g, ref_norm = o.train_step_accum(p, m, v, tok, tgt, LR, WD, CLIP, step)
        ref_losses.append(loss)
        g1 = g if g1 is None else g1
    for r in range(world):
        _, losses, P, GS1, GS, M, V, slices, norm = res[r]
        assert losses[0] == ref_losses[0]
        assert losses == pytest.approx(ref_losses, rel=1e-14, abs=0)
        assert abs(norm - ref_norm) <= 1e-12 * ref_norm
        for off, s, base in slices:
            cnt = max(0, min(off + s, o.n) - off)
            # step 1's exchanged gradient slices: bitwise the accumulated mean gradient (step 2
            # starts from parameters that differ in the last bits: the norm's summation order)
            assert np.array_equal(GS1[base:base + cnt], g1[off:off + cnt])
            assert np.abs(GS[base:base + cnt] - g[off:off + cnt]).max(initial=0) <= \
                1e-10 * np.abs(g).max()
            assert np.abs(M[base:base + cnt] - m[off:off + cnt]).max(initial=0) <= \
                1e-12 * np.abs(m).max()
            assert np.abs(V[base:base + cnt] - v[off:off + cnt]).max(initial=0) <= \
                1e-12 * np.abs(v).max()
        # every rank holds the whole updated parameter vector
        assert np.abs(P - p).max() <= 1e-12 * LR


def _nccl_single_rank(fn):
    import datetime
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        return fn(dist)
    finally:
        dist.destroy_process_group()


@pytest.mark.gpu
@pytest.mark.parametrize("precision", [0, 1])
def test_one_rank_data_parallel_step_equals_train_step(precision):
    """The data-parallel pieces on one GPU (NCCL, world 1, several buckets): loss, gradients,
    norm and the updated parameters and moments are bitwise those of gpt_train_step."""
    import torch
    from tests import gpu_util as U
    sh = fx.ModelShape(vocab=500, vocab_padded=512, n_layer=2, n_head=2, n_embd=128, max_T=64)
    Bq, Tq = 2, 64
    p0 = fx.init_params(sh, 3)
    tok, tgt = fx.zipf_tokens(sh.vocab, 1.05, Bq, Tq, 3)
    dev = torch.device("cuda", 0)
    tk, tg = torch.from_numpy(tok).to(dev), torch.from_numpy(tgt).to(dev)
    ref = U.make_step(sh, Bq, Tq, precision)
    ref.use_current_torch_stream()
    Pr = torch.from_numpy(p0).to(dev)
    Gr, Mr, Vr = (torch.zeros_like(Pr) for _ in range(3))
    ref_losses = [ref.train_step(Pr, Gr, Mr, Vr, tk, tg, 6e-4, 0.1, 1.0) for _ in range(2)]
    ref_norm = ref.last_grad_norm()
    ref.close()

    def run(dist):
        st = U.make_step(sh, Bq, Tq, precision)
        st.use_current_torch_stream()
        dp = DataParallelStep(st, st.n_params, 1, 0, dev, dist, bucket_elems=1 << 16)
        P, G, GS, M, V = dp.alloc(p0)
        losses = [dp.train_step(P, G, GS, M, V, tk, tg, 6e-4, 0.1, 1.0) for _ in range(2)]
        torch.cuda.synchronize()
        out = (losses, P.clone(), G.clone(), M.clone(), V.clone(), dp.last_norm,
               len(dp.part.buckets))
        st.close()
        return out

    losses, P, G, M, V, norm, nb = _nccl_single_rank(run)
    n = Pr.numel()
    assert nb > 1
    assert losses == ref_losses
    assert torch.equal(G[:n], Gr) and torch.equal(P[:n], Pr)
    assert torch.equal(M[:n], Mr) and torch.equal(V[:n], Vr)
    assert norm == pytest.approx(ref_norm, rel=1e-6)
