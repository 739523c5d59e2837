"""bench.py's host-only arm: the reference (the oracle on the host cores) prints the contract's JSON
line, once, also when launched as two ranks with torchrun (rank 0 alone does the work)."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REQUIRED = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _json_lines(out: str):
    return [json.loads(x) for x in out.splitlines() if x.startswith("{")]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_prints_one_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "3",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert REQUIRED <= set(d), REQUIRED - set(d)
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_two_ranks_rank0_only():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl",
                        "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3", "--gpus", "2"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference"


def test_workload_shapes_and_flop_counts():
    """The synthetic workloads carry the configured shapes: bench's algorithmic FLOPs per layer
    (2MNK for the FP4 product, 2Mr(K+N) for the branch) reproduce the per-config GFLOP figures
    derived from the configuration list (to the 0.1 GFLOP they are quoted at)."""
    sys.path.insert(0, ROOT)
    import bench
    from bit_diffusion_transformer_svdquant_b200 import synth
    want = {"tiny": [(0.134, 0.01)], "qkv_1024": [(260.9, 3.6)], "mlp_1024": [(695.8, 8.2), (347.9, 4.5)],
            "qkv_2048": [(956.7, 13.3)], "edit_2048": [(1884.4, 26.2), (628.1, 13.1)]}
    for name, layers in want.items():
        specs = synth.WORKLOADS[name].layers
        assert len(specs) == len(layers), name
        for spec, (fp4, lr) in zip(specs, layers):
            f, l = bench.layer_flops(spec)
            digits = 3 if fp4 < 1 else 1
            assert round(f / 1e9, digits) == fp4, (name, f / 1e9)
            assert abs(l / 1e9 - lr) <= 0.051, (name, l / 1e9)


def test_fp8r_side_measurement_never_raises():
    """The row-wise FP8 side measurement runs in a child process; without a usable GPU (or on any
    failure) it comes back as an error entry and the main line is unaffected."""
    import argparse
    import torch
    if torch.cuda.is_available():
        import pytest
        pytest.skip("a GPU is present")
    sys.path.insert(0, ROOT)
    import bench
    r = bench.fp8r_side(argparse.Namespace(workload="tiny", steps=3))
    assert set(r) == {"error"} and r["error"].startswith("exit ")
