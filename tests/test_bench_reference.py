"""bench.py's reference arm (the oracle on the host cores) on the CPU: one JSON line with the
contract's keys, the same metric as the library's arm, and under torchrun only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline",
        "e2e"}


def _lines(out):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                          "--warmup", "1", "--workload", "tiny_char_fp32"], cwd=ROOT,
                         capture_output=True, text=True, timeout=300, check=True).stdout
    lines = _lines(out)
    assert len(lines) == 1
    d = lines[0]
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    import bench  # the same metric and unit as the library's arm
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_under_torchrun_prints_on_rank_0_only():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    out = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                          "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                          "--master-port", "29531", "bench.py", "--impl", "reference",
                          "--gpus", "2", "--steps", "1", "--warmup", "0",
                          "--workload", "tiny_char_fp32"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=300, check=True).stdout
    lines = _lines(out)
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2
