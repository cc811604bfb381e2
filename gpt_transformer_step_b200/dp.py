"""Data-parallel training step with the optimizer state split across ranks (ZeRO-1).

The pages reproduce GPT-2 124M on one node of 8 GPUs with data parallelism (nanoGPT README,
"reproducing GPT-2": `torchrun` DDP over 8 A100s) and shard the optimizer state across the
ranks (llm.c summary, "Ejecución": `-z 1`, ZeRO-1). One step here, per rank r of W:

  1. forward + backward of the rank's own batch on its GPU (gpt_forward_backward, gradients
     scaled by 1/W, so that their sum over ranks is the gradient of the global mean loss);
  2. per bucket of the flat gradient vector, a reduce-scatter (sum): rank r keeps the r-th
     slice of every bucket, stored one slice after the other ("compact");
  3. the sum of squares of the rank's slices (gpt_sumsq) and an all-reduce of that one
     scalar: the global gradient norm, hence the clip coefficient, on every rank;
  4. AdamW on the rank's slices only (gpt_adamw_ranges): the first and second moments exist
     only for those slices, 1/W of the full state;
  5. per bucket, an all-gather of the updated fp32 parameter slices, after which every rank
     holds the whole updated parameter vector.

The collectives are torch.distributed calls (NCCL over NVLink on GPUs, gloo in the CPU tests);
every step of the arithmetic runs in the library's kernels (`compute` is a GPTStep). All ranks
take the same collectives in the same order, also when a step fails: the failure is agreed on
with one all-reduce before any gradient is exchanged.
"""
from __future__ import annotations

import math
from typing import List, Tuple


class Partition:
    """Buckets of the flat parameter vector and each rank's slice of every bucket.

    The vector is padded to n_pad, a multiple of 4 * world, and cut into at most `max_buckets`
    buckets whose lengths are multiples of 4 * world, so every slice is a whole number of
    16-byte vectors. Rank r owns [b0 + r * L / W, b0 + (r + 1) * L / W) of a bucket [b0, b0 + L);
    its compact shard holds those slices in bucket order (shard_elems = n_pad / W)."""

    def __init__(self, n: int, world: int, bucket_elems: int = 1 << 24, max_buckets: int = 64):
        if n <= 0 or world <= 0:
            raise ValueError("n and world must be positive")
        unit = 4 * world
        self.n, self.world = n, world
        self.n_pad = -(-n // unit) * unit
        nb = max(1, -(-self.n_pad // bucket_elems))
        nb = min(nb, max_buckets)
        size = -(-self.n_pad // (nb * unit)) * unit
        self.buckets: List[Tuple[int, int]] = []
        b0 = 0
        while b0 < self.n_pad:
            b1 = min(b0 + size, self.n_pad)
            self.buckets.append((b0, b1))
            b0 = b1
        self.shard_elems = self.n_pad // world

    def slices(self, rank: int) -> List[Tuple[int, int, int]]:
        """(param offset, length, compact offset) of the rank's slice of every bucket."""
        out, base = [], 0
        for b0, b1 in self.buckets:
            s = (b1 - b0) // self.world
            out.append((b0 + rank * s, s, base))
            base += s
        return out

    def update_ranges(self, rank: int) -> List[Tuple[int, int]]:
        """(offset, count) of the rank's slices within the real parameters [0, n): the padding
        at the end of the last bucket is not updated. Counts stay multiples of 4 when n is."""
        out = []
        for off, s, _ in self.slices(rank):
            cnt = max(0, min(off + s, self.n) - off)
            out.append((off, cnt))
        return out


class DataParallelStep:
    """One rank's side of the data-parallel step. `compute` runs the arithmetic (a GPTStep, or
    any object with forward_backward / sumsq / adamw_ranges / params_changed); `dist` is
    torch.distributed with an initialised process group of `world` ranks."""

    def __init__(self, compute, n_params: int, world: int, rank: int, device, dist,
                 bucket_elems: int = 1 << 24):
        import torch
        self.compute, self.dist = compute, dist
        self.world, self.rank, self.device = world, rank, device
        self.part = Partition(n_params, world, bucket_elems)
        self.slices = self.part.slices(rank)
        self.ranges = self.part.update_ranges(rank)
        self.step_count = 0
        self.last_norm = float("nan")
        self._sumsq = torch.zeros(1, dtype=torch.float64, device=device)
        self._flag = torch.zeros(2, dtype=torch.float64, device=device)

    # buffers a caller allocates once: full params / grads (padded), compact shards
    def alloc(self, params_init, dtype=None):
        """(params [n_pad], grads [n_pad], grad_shard, m_shard, v_shard), zero padded; fp32
        unless `dtype` says otherwise."""
        import torch
        dtype = dtype or torch.float32
        n, n_pad, s = self.part.n, self.part.n_pad, self.part.shard_elems
        p = torch.zeros(n_pad, dtype=dtype, device=self.device)
        p[:n].copy_(torch.as_tensor(params_init, dtype=dtype))
        z = lambda k: torch.zeros(k, dtype=dtype, device=self.device)  # noqa: E731
        return p, z(n_pad), z(s), z(s), z(s)

    def train_step(self, params, grads, grad_shard, m_shard, v_shard, tokens, targets,
                   lr: float, wd: float, clip: float) -> float:
        """One optimizer step over the union of all ranks' batches; returns the global mean
        loss. Raises RuntimeError on every rank when any rank's step failed (bad ids, a
        non-finite loss or norm); parameters and moments are then unchanged."""
        dist, W = self.dist, self.world
        status, loss = 0, float("nan")
        try:
            loss = self.compute.forward_backward(params, grads, tokens, targets, 1.0 / W)
        except Exception as e:  # the library's error: agreed on below, raised after
            status = int(getattr(e, "status", -1)) or -1
        # one all-reduce: [sum of losses, number of failed ranks]
        self._flag[0] = loss if status == 0 else 0.0
        self._flag[1] = 1.0 if (status != 0 or not math.isfinite(loss)) else 0.0
        dist.all_reduce(self._flag, op=dist.ReduceOp.SUM)
        loss_sum, failed = self._flag.tolist()
        if failed > 0:
            raise RuntimeError(f"data-parallel step skipped: {int(failed)} rank(s) failed "
                               f"(this rank's status {status})")
        # gradient exchange: rank r keeps the sum over ranks of its slices
        for (b0, b1), (off, s, base) in zip(self.part.buckets, self.slices):
            dist.reduce_scatter_tensor(grad_shard[base:base + s], grads[b0:b1],
                                       op=dist.ReduceOp.SUM)
        self.compute.sumsq(grad_shard, self._sumsq)
        dist.all_reduce(self._sumsq, op=dist.ReduceOp.SUM)
        sumsq = float(self._sumsq.item())
        self.last_norm = math.sqrt(sumsq) if sumsq >= 0 else float("nan")
        if not math.isfinite(sumsq):
            raise RuntimeError("data-parallel step skipped: non-finite gradient norm")
        t = self.step_count + 1
        self.compute.adamw_ranges(params, grad_shard, m_shard, v_shard, self.ranges, lr, wd,
                                  clip, self._sumsq, t)
        # every rank gets every updated slice
        for (b0, b1), (off, s, _) in zip(self.part.buckets, self.slices):
            dist.all_gather_into_tensor(params[b0:b1], params[off:off + s].clone())
        self.compute.params_changed()
        self.step_count = t
        return loss_sum / W
