#!/usr/bin/env python
"""Benchmark: one GPT-2 training step (forward, backward, grad-norm clip, AdamW) per
iteration through the library's C ABI, on synthetic Zipf tokens and random-init weights.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--parallel dp|replicas] [--micro-batches n]

Prints one JSON line (rank 0). With N > 1 (launched by torch.distributed.run) each rank takes
its own batch of the workload's size (weak scaling). --parallel dp (the default) runs one
data-parallel optimizer step over all ranks' batches: gradients reduce-scattered over NCCL,
the optimizer state split across the ranks (ZeRO-1), parameters all-gathered;
--parallel replicas runs N independent copies of the single-GPU step. The timed region is
bracketed by barriers and the slowest rank's time is used.

--impl reference times the oracle (plain single-threaded C++ CPU definition of the step) on
the host cores, each step a bounded sample (B=1, a short causal prefix) of the workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

METRIC = "train tokens/s (GPT-2 step, MFU from 6N+attn FLOPs)"

# DRAM bytes (read + write) per tcgen05 GEMM launch: ncu dram__bytes_read.sum +
# dram__bytes_write.sum of one launch of each block GEMM shape and of the lm_head dX / dwte
# chunks (kernel_bench cases, profiles/gemm_shapes_gpt2_124m_ncu.md), averaged with the launch
# counts of one step (148 launches; 148.7 MB algorithmic per launch on the same basis). The
# split-K reduce kernels and the lm_head statistics / recompute launches are not in the mean.
# In the step, the attention-projection dgrad GEMM also reads the attention output (25 MB) for
# the D epilogue; its capture is the plain-store form, so the step's mean is ~2 MB higher.
GEMM_DRAM_BYTES_PER_LAUNCH: dict = {"gpt2_124m_bf16": 136.6e6}
GEMM_ALG_BYTES_PER_LAUNCH: dict = {"gpt2_124m_bf16": 148.7e6}

def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK, "fallback"


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, path: str | None = None):
        self.index = index
        self.proc = None
        self.keep = path is not None
        if path is None:
            import tempfile
            fd, path = tempfile.mkstemp(prefix=f"clocks_gpu{index}_", suffix=".csv")
            os.close(fd)
        self.path = path

    def start(self):
        try:
            d = os.path.dirname(self.path)
            if d:
                os.makedirs(d, exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.index)], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not self.keep:
            try:
                os.remove(self.path)
            except OSError:
                pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest value over all ranks (the slowest replica's time); identity for world 1."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def oracle_sample_step(wl, T_sample: int, seed: int = 0, B_sample: int = 1):
    """One oracle training step (float instantiation, one thread) on B_sample x T_sample tokens
    of the workload's model. Returns (seconds, tokens)."""
    import numpy as np
    import oracle
    from gpt_transformer_step_b200 import fixtures as fx
    o = oracle.Oracle.from_shape(wl.shape, dtype=np.float32)
    p = fx.init_params(wl.shape, seed)
    tok, tgt = fx.zipf_tokens(wl.shape.vocab, wl.zipf_s, B_sample, T_sample, seed)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    t0 = time.perf_counter()
    o.train_step(p, m, v, tok, tgt, wl.lr, wl.wd, wl.clip, 1)
    return time.perf_counter() - t0, B_sample * T_sample


def host_cpu():
    """(logical cores, CPU model) of this host."""
    model = "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return os.cpu_count(), model


def cpu_baseline(wl, T_sample=20):  # ~10 s of one host core for the 124M model
    """The oracle timed on one host thread: the headline sample (B=1 x T_sample of the bench
    workload's full model) plus full oracle steps of the two small workload shapes."""
    from gpt_transformer_step_b200 import fixtures as fx
    sec, ntok = oracle_sample_step(wl, T_sample)
    nproc, model = host_cpu()
    out = {"value": ntok / sec, "unit": "tokens/s", "cores": 1, "kind": "oracle",
           "sample": f"one oracle train step (fp32, 1 thread) on B=1 x T={T_sample} tokens of "
                     f"the {wl.name} model (full width/depth/vocab); {sec:.1f} s",
           "host_nproc": nproc, "host_cpu": model, "other_workloads": []}
    tiny = fx.WORKLOADS["tiny_char_fp32"]
    sec_t, n_t = oracle_sample_step(tiny, tiny.T, B_sample=tiny.B)
    out["other_workloads"].append({"workload": tiny.name, "tokens_per_s": n_t / sec_t,
                                   "sample": f"full step B={tiny.B} x T={tiny.T}",
                                   "seconds": sec_t})
    sh = fx.WORKLOADS["shakespeare_char_bf16"]
    sec_s, n_s = oracle_sample_step(sh, sh.T, B_sample=1)
    out["other_workloads"].append({"workload": sh.name, "tokens_per_s": n_s / sec_s,
                                   "sample": f"one step at B=1 x T={sh.T} (full T; the workload's "
                                             f"B={sh.B} is {sh.B}x this)",
                                   "seconds": sec_s})
    return out


def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    T_sample = 8
    secs = []
    for i in range(args.warmup + args.steps):
        s, _ = oracle_sample_step(wl, T_sample, seed=i)
        if i >= args.warmup:
            secs.append(s)
    ms = 1000 * sum(secs) / len(secs)
    val = T_sample / (ms / 1000)
    from gpt_transformer_step_b200 import fixtures as fx
    fpt = fx.flops_per_token(wl.shape, wl.T)
    line = {
        "impl": "reference", "metric": METRIC, "value": val,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": world * wl.B, "seq_len": wl.T,
                   "parallelism": f"replicas{world}" if world > 1 else "single",
                   "sample": f"each step: the oracle on B=1 x T={T_sample} tokens"},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"oracle train step on B=1 x T={T_sample} tokens per step"},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "mfu_nominal": val * fpt / (NOMINAL_BF16_TFLOPS * 1e12),
    }
    print(json.dumps(line), flush=True)


def kernel_table(kst, n_steps, pk, pk_kind):
    """Per kernel class: launches and ms per step, achieved rate on algorithmic work, and the
    fraction of the measured copy bandwidth (bytes) or bf16 burst peak (FLOPs)."""
    out = {}
    for name, (n, ms, work, unit) in kst.items():
        if n == 0 or ms <= 0:
            continue
        rec = {"launches_per_step": n / n_steps, "ms_per_step": ms / n_steps}
        if unit == "byte":
            gbs = work / (ms / 1000) / 1e9
            rec.update({"achieved": gbs, "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                        "bound": "hbm", "work_per_launch": work / n})
        else:
            tf = work / (ms / 1000) / 1e12
            rec.update({"achieved": tf, "unit": "TFLOP/s", "frac": tf / pk["bf16_tflops"],
                        "bound": "tensor", "work_per_launch": work / n})
        out[name] = rec
    out["_peaks"] = f"{pk_kind}: {pk['hbm_gbs']} GB/s copy, {pk['bf16_tflops']} TFLOP/s bf16 burst"
    return out


def use_dp(args, world: int) -> bool:
    """The data-parallel step runs for --parallel dp under torch.distributed.run (any world
    size, so one GPU can run it too); a plain single-process run takes the one-GPU step."""
    return args.parallel == "dp" and (world > 1 or "WORLD_SIZE" in os.environ)


def run_ours(args, wl, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from gpt_transformer_step_b200 import binding as gb
    from gpt_transformer_step_b200 import fixtures as fx

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    sh = wl.shape
    B, T = wl.B, wl.T
    p, tok, tgt = fx.make_inputs(wl, seed=0)
    nm = max(1, args.micro_batches)  # micro-batches per optimizer step (gradient accumulation)
    tok, tgt = fx.zipf_tokens(sh.vocab, wl.zipf_s, nm * B, T, seed=rank)  # own batch per replica
    if nm > 1:
        tok, tgt = tok.reshape(nm, B, T), tgt.reshape(nm, B, T)
    st = gb.GPTStep.from_workload(wl, lmhead_chunk_rows=args.lmhead_chunk_rows,
                                  recompute_gelu=args.recompute)
    stream = torch.cuda.Stream(device=dev)
    dp = None
    if use_dp(args, world):
        # data parallelism with the optimizer state split across the ranks (ZeRO-1)
        from gpt_transformer_step_b200.dp import DataParallelStep
        dp = DataParallelStep(st, st.n_params, world, rank, dev, dist)
        P, G, GS, Mm, Vv = dp.alloc(p)
    else:
        P = torch.from_numpy(p).to(dev)
        G = torch.zeros_like(P)
        Mm = torch.zeros_like(P)
        Vv = torch.zeros_like(P)
    tk = torch.from_numpy(tok).to(dev)
    tg = torch.from_numpy(tgt).to(dev)
    tk_h = torch.from_numpy(tok).pin_memory()
    tg_h = torch.from_numpy(tgt).pin_memory()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()

    muon_cfg = None
    if args.optimizer == "muon":
        from gpt_transformer_step_b200.muon import MuonConfig
        muon_cfg = MuonConfig()

    def step(a, b):
        if muon_cfg is not None:  # hybrid Muon + AdamW: forward/backward, then the update
            loss = st.forward_backward(P, G, a, b)
            st.muon_update(P, G, Mm, Vv, wl.lr, wl.wd, wl.clip, muon_cfg)
            return loss
        if dp is not None:
            return dp.train_step(P, G, GS, Mm, Vv, a, b, wl.lr, wl.wd, wl.clip)
        if nm > 1:
            return st.train_step_accum(P, G, Mm, Vv, a, b, wl.lr, wl.wd, wl.clip)
        return st.train_step(P, G, Mm, Vv, a, b, wl.lr, wl.wd, wl.clip)

    def timed(n, host_inputs=False):
        """Device time of n steps (CUDA events on the launching stream), max over ranks, and
        the median of the per-step event intervals."""
        a, b = (tk_h, tg_h) if host_inputs else (tk, tg)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        barrier()
        torch.cuda.synchronize()
        losses = []
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            for i in range(n):
                losses.append(step(a, b))
                ev[i + 1].record(stream)
        torch.cuda.synchronize()
        barrier()
        ms = max_over_ranks(ev[0].elapsed_time(ev[n]) / n, world, dev)
        med = statistics.median(ev[i].elapsed_time(ev[i + 1]) for i in range(n))
        return ms, losses, med

    st.set_stream(stream.cuda_stream)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step(tk, tg)
    torch.cuda.synchronize()
    launches = st.last_launch_count() + (2 if dp is not None else 0)  # + sumsq, ranged AdamW
    if muon_cfg is not None:  # the update's launches (the last call was the update)
        st.forward_backward(P, G, tk, tg)
        launches = st.last_launch_count()
        st.muon_update(P, G, Mm, Vv, wl.lr, wl.wd, wl.clip, muon_cfg)
        launches += st.last_launch_count()

    clk = Clocks(local_rank, args.clock_log)
    clk.start()
    ms, losses, ms_med = timed(args.steps)
    clocks = clk.stop()

    # end to end through the same C ABI call with host (pinned) token buffers
    ms_e2e, _, ms_e2e_med = timed(args.steps, host_inputs=True)

    # every kernel class, CUDA events around each launch on the step's stream (separate
    # instrumented steps: graphs are off while timing)
    n_inst = max(2, args.steps // 4)
    st.set_option(gb.GPT_OPT_TIME_KERNELS, 1)
    st.kernel_stats(reset=True)
    timed(n_inst)
    kst = st.all_kernel_stats(reset=True)
    st.set_option(gb.GPT_OPT_TIME_KERNELS, 0)
    n_rc, rc_ms, rc_flops, _ = kst["gemm_recompute"]
    n_l, gemm_ms, gemm_flops, _ = kst["gemm"]

    if rank != 0:
        return
    pk, pk_kind = peaks()
    tokens = world * nm * B * T
    value = tokens / (ms / 1000)
    fpt = fx.flops_per_token(sh, T)
    fpt_lit = fx.flops_per_token(sh, T, exclude="wte+wpe")
    # algorithmic FLOPs (the method's own contractions) over the time of every GEMM launch,
    # the logits recompute of the cross-entropy backward included in the time
    achieved = (gemm_flops / (gemm_ms / 1000)) / 1e12 if gemm_ms > 0 else None
    peak_b = pk["bf16_tflops"]
    peak_s = pk["bf16_tflops_sustained"]
    line = {
        "metric": METRIC,
        "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_median": ms_med,
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (Zipf tokens, N(0,0.02) init)",
        "config": {"workload": wl.name, "global_batch": world * nm * B, "seq_len": T,
                   "micro_batches": nm, "recompute_gelu": bool(args.recompute),
                   "optimizer": args.optimizer,
                   "parallelism": f"dp{world}-zero1" if dp is not None
                   else (f"replicas{world}" if world > 1 else "single"),
                   "l2": "working set ~6 GB >> 126 MB L2 (no flush needed)"},
        "mfu": {"nominal_2250": value / world * fpt / 2.25e15,
                "measured_burst": value / world * fpt / (peak_b * 1e12),
                "measured_sustained": value / world * fpt / (peak_s * 1e12),
                "flops_per_token": fpt, "flops_per_token_literal_excl_wte": fpt_lit},
        "loss_first_timed": losses[0] if losses else None,
        "e2e": {"value": tokens / (ms_e2e / 1000), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * nm * B * T * 4, "d2h_bytes_per_step": 128,
                "ms_per_step_median": ms_e2e_med},
        "roofline": {"bound": "tensor", "kernel": "tcgen05 GEMMs (all launches, flop-weighted)",
                     "achieved": achieved, "peak": peak_b, "unit": "TFLOP/s",
                     "frac": (achieved / peak_b) if achieved else None,
                     "frac_vs_sustained": (achieved / peak_s) if achieved else None,
                     "traffic": GEMM_DRAM_BYTES_PER_LAUNCH.get(wl.name),
                     "traffic_algorithmic": GEMM_ALG_BYTES_PER_LAUNCH.get(wl.name),
                     "traffic_unit": "bytes per GEMM launch (ncu dram__bytes_read.sum + "
                                     "dram__bytes_write.sum)",
                     "flops": "algorithmic: 2MNK of the block GEMMs and the lm_head forward, "
                              "dX and dwte; the logits recompute is timed but not counted",
                     "peak_kind": f"{pk_kind} burst bf16 (the step is ~17 ms, not a seconds-long "
                                  f"loop); sustained {peak_s} beside it",
                     "launches_timed": n_l,
                     "gemm_ms_per_step": gemm_ms / n_inst,
                     "gemm_tflop_per_step": gemm_flops / n_inst / 1e12,
                     "recompute": {"launches": n_rc, "ms_per_step": rc_ms / n_inst,
                                   "tflop_per_step": rc_flops / n_inst / 1e12}},
        "kernels": kernel_table(kst, n_inst, pk, pk_kind),
        "clocks": clocks,
        "gpu_launches": launches * args.steps,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)
    st.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="gpt2_124m_bf16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clock-log", default=None,
                    help="keep the nvidia-smi clock samples of the timed region in this file")
    ap.add_argument("--parallel", default="dp", choices=["dp", "replicas"],
                    help="with --gpus N > 1: data parallelism with ZeRO-1 optimizer sharding "
                         "(gradients exchanged over NCCL) or N independent replicas")
    ap.add_argument("--micro-batches", type=int, default=1,
                    help="micro-batches of B x T per optimizer step (gradient accumulation)")
    ap.add_argument("--optimizer", default="adamw", choices=["adamw", "muon"],
                    help="muon: the hybrid Muon (block matrices) + AdamW update")
    ap.add_argument("--recompute", action="store_true",
                    help="activation recompute: GELU recomputed in the backward (llm.c -r)")
    ap.add_argument("--lmhead-chunk-rows", type=int, default=0,
                    help="rows per lm_head backward chunk (0 = the library default)")
    args = ap.parse_args()
    from gpt_transformer_step_b200 import fixtures as fx
    wl = fx.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    pg = world > 1 or use_dp(args, world)
    if pg:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, wl, rank, world, local_rank)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
