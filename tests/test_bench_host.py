"""Host logic of bench.py that needs no GPU: argument defaults, workload naming, the
GEMM traffic record's source check, and the reference arm (the oracle timed on the
host cores) printing its JSON line."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _args(*argv):
    old = sys.argv
    sys.argv = ["bench.py", *argv]
    try:
        return bench.parse()
    finally:
        sys.argv = old


def test_defaults_follow_the_contract():
    a = _args()
    assert a.gpus == 1 and a.steps >= 1 and a.warmup >= 3 and a.impl == "fp4"
    assert a.format == "mxfp4" and a.hadamard == 16 and a.side_stream == 1
    assert _args("--warmup", "1").warmup == 3  # at least three warm-up steps


def test_library_compare_shapes():
    """--library-compare times the step's own GEMMs: per projection Fprop (M = tokens),
    Dgrad (N and K swapped) and Wgrad (contraction over the tokens)."""
    a = _args("--library-compare", "--format", "nvfp4")
    assert a.library_compare and a.format == "nvfp4"
    layers, tokens, _ = bench.layer_table(a)
    shapes = bench.gemm_shapes(layers, tokens)
    assert len(shapes) == 3 * len(layers) == 15
    by = {lab: (m, n, k) for lab, m, n, k in shapes}
    assert by["down.fprop"] == (8192, 4096, 14336)
    assert by["down.dgrad"] == (8192, 14336, 4096)
    assert by["down.wgrad"] == (4096, 14336, 8192)
    flops = sum(2 * m * n * k for _, m, n, k in shapes)
    assert abs(flops / 15 / 1e9 - 714.68) < 0.01  # 714.7 GFLOP per GEMM on average


def test_workload_names():
    assert bench.workload_name(_args()) == bench.WORKLOAD
    assert "NVFP4 + H32" in bench.workload_name(_args("--format", "nvfp4", "--hadamard", "32"))
    assert "sr quantiser variant" in bench.workload_name(_args("--variant", "sr"))
    g = bench.workload_name(_args("--workload", "gpt3", "--hadamard", "0"))
    assert g.startswith("gpt3-175b") and "no rotation" in g
    with pytest.raises(SystemExit):
        _args("--variant", "amax")  # a supplied amax is NVFP4 only
    assert "next layer (fused)" in bench.workload_name(_args("--next-layer-quant", "fused"))
    assert _args().next_layer_quant == "none"
    with pytest.raises(SystemExit):
        _args("--next-layer-quant", "fused", "--format", "nvfp4")  # Y is quantised as MXFP4


def test_layer_tables():
    from fp4_block_scaled_deterministic_b200 import synthetic
    layers, tokens, mult = bench.layer_table(_args("--workload", "gpt3"))
    assert layers == synthetic.GPT3_LAYERS and tokens == 4096 and mult == 100.0
    layers, tokens, mult = bench.layer_table(_args())
    assert layers == synthetic.LLAMA_LAYERS and tokens == 8192 and mult == 50.0


def test_traffic_record_is_tied_to_the_gemm_sources():
    rec = json.load(open(os.path.join(ROOT, "profiles", "gemm_llama_traffic.json")))
    assert bench.kernel_source_hash() == bench.kernel_source_hash()
    got = bench.recorded_traffic("mxfp4_group")  # one grouped launch per projection
    if rec["source_sha1"] == bench.kernel_source_hash():
        assert got == rec["per_launch_bytes"]["mxfp4_group"] and got > 0
    else:
        assert got is None  # the kernel changed since the counters were taken
    assert bench.recorded_traffic("no-such-kernel") is None


def test_reference_arm_prints_one_json_line():
    a = _args("--impl", "reference", "--steps", "1", "--warmup", "3", "--cpu-budget", "0.1")
    out = io.StringIO()
    with redirect_stdout(out):
        bench.run_reference(a)
    lines = [ln for ln in out.getvalue().splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["extrapolated"] is True and d["cpu_baseline"]["extrapolated"] is True
    host = d["cpu_baseline"]["host"]
    assert host["cpu_count"] >= 1 and host["affinity_cpus"] >= 1 and "cpu_model" in host
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == bench.WORKLOAD


def test_host_facts_and_threads():
    h = bench.host_facts()
    assert h["cpu_count"] == os.cpu_count() and h["affinity_cpus"] == bench.host_threads()
    assert h["affinity"]  # e.g. "0-7"


def test_gpus_n_spawns_ranks_or_fails_loudly():
    """`bench.py --gpus 2` as a plain process re-launches itself as two ranks; without
    two visible GPUs it stops with a clear error and exit status 2 instead of running
    one rank and calling it two."""
    import subprocess
    import torch
    if torch.cuda.device_count() >= 2:
        pytest.skip("host has two GPUs: the spawn would run the real benchmark")
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--steps", "1"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 2
    assert "needs 2 visible CUDA devices" in r.stderr
