"""Per-kernel timing of the step's GEMM and attention kernels at the GPT-2 124M shapes
(B=16, T=1024, C=768, H=12), through the kernel-level C ABI (include/gpt_kernels.h).

    python -m gpt_transformer_step_b200.kernel_bench [--case NAME ...] [--reps N] [--path tc|simt]
                                                     [--torch] [--gemm M,N,K[,EPI] ...]

Each case runs `warmup` untimed launches, then `reps` launches timed with CUDA events on the
launching stream; prints one JSON line per case with ms per launch and TFLOP/s (algorithmic
FLOPs: 2*M*N*K per GEMM; 4*hd per admitted score forward, 8*hd backward). attn_bwd is the
two-pass backward (dQ with D, then dK/dV); attn_bwd_ds the one the step runs (D, dK/dV writing
dS^T, dQ from it).
Also the workload for small ncu captures of a single kernel (few hundred MB on the device).
"""
from __future__ import annotations

import argparse
import json

B, T, C, H = 16, 1024, 768, 12
M = B * T

# name: (M, N, K, a_kmajor, b_kmajor, epilogue, split); split 0 = the launcher's choice
GEMMS = {
    "gemm_qkv": (M, 3 * C, C, 1, 1, "store", 1),
    "gemm_attnproj": (M, C, C, 1, 1, "resid", 1),
    "gemm_fc": (M, 4 * C, C, 1, 1, "store_gelu", 1),
    "gemm_mlpproj": (M, C, 4 * C, 1, 1, "resid", 1),
    "gemm_dgrad_mlpproj": (M, 4 * C, C, 1, 0, "dgelu", 1),
    "gemm_dgrad_fc": (M, C, 4 * C, 1, 0, "store", 1),
    "gemm_wgrad_fc": (4 * C, C, M, 0, 0, "f32_store", 0),
    "gemm_wgrad_qkv": (3 * C, C, M, 0, 0, "f32_store", 0),
    "gemm_wgrad_attnproj": (C, C, M, 0, 0, "f32_store", 0),
    "gemm_wgrad_mlpproj": (C, 4 * C, M, 0, 0, "f32_store", 0),
    "gemm_dgrad_attnproj": (M, C, C, 1, 0, "store", 1),
    "gemm_dgrad_qkv": (M, C, 3 * C, 1, 0, "store", 1),
    "gemm_lmhead": (M, 50304, C, 1, 1, "store", 1),
    # the lm_head backward's two products on one 8192-row chunk (dS is A in both)
    "gemm_lmhead_dx": (8192, C, 50304, 1, 0, "store", 0),
    "gemm_lmhead_dwte": (50304, C, 8192, 0, 0, "f32_store", 1),
    # the second chunk's dwte, accumulated into the fp32 gradient
    "gemm_lmhead_dwte_acc": (50304, C, 8192, 0, 0, "f32_accum", 1),
}
# launches of each shape in one 124M step (the lm_head forward statistics and dS recompute
# run the gemm_lmhead shape with cross-entropy epilogues: two of them per chunk pair)
STEP_LAUNCHES = {"gemm_qkv": 12, "gemm_attnproj": 12, "gemm_fc": 12, "gemm_mlpproj": 12,
                 "gemm_dgrad_mlpproj": 12, "gemm_dgrad_fc": 12, "gemm_dgrad_attnproj": 12,
                 "gemm_dgrad_qkv": 12, "gemm_wgrad_fc": 12, "gemm_wgrad_qkv": 12,
                 "gemm_wgrad_attnproj": 12, "gemm_wgrad_mlpproj": 12, "gemm_lmhead_dx": 2,
                 "gemm_lmhead_dwte": 2}
ATTN = ("attn_fwd", "attn_bwd", "attn_bwd_ds")
LN = ("ln_fwd", "ln_bwd")


def causal_scores(Bn, Tn, Hn, w=-1):
    s = 0
    for i in range(Tn):
        lo = 0 if w < 0 else max(0, i - w)
        s += i - lo + 1
    return s * Bn * Hn


def main():
    import torch

    from gpt_transformer_step_b200 import binding as gb
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", nargs="*", default=list(GEMMS) + list(ATTN) + list(LN))
    ap.add_argument("--reps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--path", default="tc", choices=["tc", "simt"])
    ap.add_argument("--torch", action="store_true",
                    help="also time torch.matmul (cuBLAS, bf16 output, no epilogue) on each "
                         "GEMM case's shapes and layouts, for comparison")
    ap.add_argument("--gemm", nargs="*", default=[], metavar="M,N,K[,EPI]",
                    help="extra K-major x K-major GEMM cases (epilogue store by default)")
    args = ap.parse_args()
    for spec in args.gemm:
        f = spec.split(",")
        GEMMS[f"gemm_{spec}"] = (int(f[0]), int(f[1]), int(f[2]), 1, 1,
                                 f[3] if len(f) > 3 else "store", 1)
        args.case.append(f"gemm_{spec}")
    path = gb.GPTK_PATH_TCGEN05 if args.path == "tc" else gb.GPTK_PATH_SIMT
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for name in args.case:
        with torch.cuda.stream(stream):
            s = stream.cuda_stream
            if name in LN:
                x = torch.randn(M, C, device=dev).to(torch.bfloat16)
                gam = torch.ones(C, device=dev).to(torch.bfloat16)
                y = torch.empty(M, C, dtype=torch.bfloat16, device=dev)
                mean = torch.empty(M, device=dev)
                rstd = torch.empty(M, device=dev)
                gb.gptk_layernorm_fwd_bf16(x.data_ptr(), gam.data_ptr(), y.data_ptr(),
                                           mean.data_ptr(), rstd.data_ptr(), M, C, 1e-5, s)
                dres = torch.randn(M, C, device=dev).to(torch.bfloat16)
                dg = torch.zeros(C, device=dev)
                nsc = gb.gptk_layernorm_bwd_scratch_floats(M, C)
                scr = torch.empty(nsc, device=dev)
                if name == "ln_fwd":
                    def run():
                        rc = gb.gptk_layernorm_fwd_bf16(x.data_ptr(), gam.data_ptr(), y.data_ptr(),
                                                        mean.data_ptr(), rstd.data_ptr(), M, C,
                                                        1e-5, s)
                        assert rc == 0, rc
                    nbytes = M * (4.0 * C + 8)
                else:
                    def run():
                        rc = gb.gptk_layernorm_bwd_bf16(x.data_ptr(), gam.data_ptr(),
                                                        mean.data_ptr(), rstd.data_ptr(),
                                                        y.data_ptr(), dres.data_ptr(), 1,
                                                        dg.data_ptr(), 0, scr.data_ptr(), nsc, M,
                                                        C, s)
                        assert rc == 0, rc
                    nbytes = M * (8.0 * C + 8)
                flops = None
            elif name in GEMMS:
                m, n, k, ak, bk, epi, split = GEMMS[name]
                A = torch.randn(m * k, device=dev).to(torch.bfloat16)
                Bm = torch.randn(n * k, device=dev).to(torch.bfloat16)
                lda = k if ak else m
                ldb = k if bk else n
                f32 = epi.startswith("f32")
                out = torch.empty(1 if f32 else m * n, dtype=torch.bfloat16, device=dev)
                out2 = torch.empty(m * n if epi == "store_gelu" else 1, dtype=torch.bfloat16, device=dev)
                aux = torch.randn(m * n if epi in ("resid", "dgelu") else 1, device=dev).to(torch.bfloat16)
                outf = torch.empty(m * n if f32 else 1, device=dev)
                scratch = torch.empty(16 * m * n if split == 0 else (split * m * n if split > 1 else 1),
                                      device=dev)

                def run():
                    rc = gb.gptk_gemm_bf16(m, n, k, A.data_ptr(), lda, ak, Bm.data_ptr(), ldb, bk,
                                           gb.GPTK_EPI[epi], out.data_ptr(), n, out2.data_ptr(), n,
                                           aux.data_ptr(), n, outf.data_ptr(), n, split,
                                           scratch.data_ptr(), scratch.numel(), err.data_ptr(),
                                           path, s)
                    assert rc == 0, rc
                flops = 2.0 * m * n * k
                if args.torch:
                    At = A.view(m, k) if ak else A.view(k, m).t()
                    Bt = Bm.view(n, k).t() if bk else Bm.view(k, n)
                    for _ in range(args.warmup):
                        torch.matmul(At, Bt)
                    t0 = torch.cuda.Event(enable_timing=True)
                    t1 = torch.cuda.Event(enable_timing=True)
                    t0.record(stream)
                    for _ in range(args.reps):
                        torch.matmul(At, Bt)
                    t1.record(stream)
                    torch.cuda.synchronize()
                    torch_ms = t0.elapsed_time(t1) / args.reps
            else:
                qkv = torch.randn(M, 3 * C, device=dev).to(torch.bfloat16)
                o = torch.empty(M, C, dtype=torch.bfloat16, device=dev)
                lse = torch.empty(B, H, T, device=dev)
                dout = torch.randn(M, C, device=dev).to(torch.bfloat16)
                D = torch.empty(B, H, T, device=dev)
                dq = torch.empty(M, 3 * C, dtype=torch.bfloat16, device=dev)
                gb.gptk_attention_fwd_bf16(qkv.data_ptr(), o.data_ptr(), lse.data_ptr(), B, T, C,
                                           H, -1, err.data_ptr(), path, s)
                hd = C // H
                sc = causal_scores(B, T, H)
                if name == "attn_fwd":
                    def run():
                        rc = gb.gptk_attention_fwd_bf16(qkv.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                                        B, T, C, H, -1, err.data_ptr(), path, s)
                        assert rc == 0, rc
                    flops = 4.0 * hd * sc
                elif name == "attn_bwd":
                    def run():
                        rc = gb.gptk_attention_bwd_bf16(qkv.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                                        lse.data_ptr(), D.data_ptr(), dq.data_ptr(),
                                                        B, T, C, H, -1, err.data_ptr(), path, s)
                        assert rc == 0, rc
                    flops = 8.0 * hd * sc
                else:
                    ds = torch.zeros(B * H * T * T, dtype=torch.bfloat16, device=dev)

                    def run():
                        rc = gb.gptk_attention_bwd_bf16_ds(qkv.data_ptr(), o.data_ptr(),
                                                           dout.data_ptr(), lse.data_ptr(),
                                                           D.data_ptr(), ds.data_ptr(), dq.data_ptr(),
                                                           B, T, C, H, -1, err.data_ptr(), s)
                        assert rc == 0, rc
                    flops = 8.0 * hd * sc
            for _ in range(args.warmup):
                run()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.reps):
                run()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.reps
        rec = {"case": name, "ms": ms, "err": int(err.item())}
        if flops is None:
            rec["gbs"] = nbytes / (ms * 1e-3) / 1e9
        else:
            rec["tflops"] = flops / (ms * 1e-3) / 1e12
            if args.torch and name in GEMMS:
                rec["torch_ms"] = torch_ms
                rec["torch_tflops"] = flops / (torch_ms * 1e-3) / 1e12
        print(json.dumps(rec), flush=True)


if __name__ == "__main__":
    main()
