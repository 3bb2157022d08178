"""bench.py's reference arm (the CPU oracle on a bounded sample) runs without
a GPU: its JSON line carries every field of the bench contract, for the
forward and the input-gradient measurement."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"]


@pytest.mark.parametrize("extra,unit", [([], "TOPS"), (["--op", "backward"], "TFLOP/s")])
def test_reference_arm_json_line(extra, unit):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0", *extra],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in KEYS:
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == unit and d["value"] > 0
    assert d["higher_is_better"] is True and d["data"] == "synthetic" and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["unit"] == unit and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_algorithmic_bytes_by_hand():
    """The bytes each stage must move at least once, counted by hand for
    LLaMA-2-7B q_proj at 16 tokens with 41 outlier channels."""
    sys.path.insert(0, ROOT)
    import bench
    # GEMM: INT4 weights 8 MiB, c 16 KiB, W_O 41 x 4096 fp16, Xq 64 KiB,
    # a 64 B, XqO 656 B, Y 16 x 4096 fp16
    assert bench.algorithmic_bytes(16, 4096, 4096, 41, 0) == (
        8388608 + 16384 + 335872 + 65536 + 64 + 656 + 131072,
        # quantization: read X (128 KiB), write Xq, a and XqO
        131072 + 65536 + 64 + 656)
    # g128 adds the fp16 ratios (32 groups x 4096); INT8 weights are 16 MiB
    g, _ = bench.algorithmic_bytes(16, 4096, 4096, 41, 1)
    assert g == 8388608 + 16384 + 262144 + 335872 + 65536 + 64 + 656 + 131072
    g, _ = bench.algorithmic_bytes(16, 4096, 4096, 41, 2)
    assert g == 16777216 + 16384 + 335872 + 65536 + 64 + 656 + 131072


def test_layer_bytes_by_hand():
    """The fused layer's algorithmic bytes (no INT8 round trip between the
    two kernels): X, packed weights with their scales and outlier rows, Y."""
    sys.path.insert(0, ROOT)
    import bench
    # 70B up_proj at one token, g128, 82 outliers
    K, N, nO = 8192, 28672, 82
    want = 2 * K + K * N // 2 + 4 * N + 2 * (K // 128) * N + 2 * nO * N + 16 * nO + 2 * N
    assert bench.layer_bytes(1, K, N, nO, 1) == want


def test_offq_bytes_by_hand():
    """OffQ: the quantization reads X and writes one code byte per value and
    an fp32 scale and offset per (token, group); the GEMM reads those, the
    packed INT4 weights, the channel scales and per-group column sums, and
    writes Y.  Llama-3-8B k_proj at 4096 tokens."""
    sys.path.insert(0, ROOT)
    import bench
    M, K, N = 4096, 4096, 1024
    G = K // 128
    assert bench.offq_bytes(M, K, N) == (2 * M * K + M * K + 8 * M * G,
                                         M * K + 8 * M * G + K * N // 2 + 4 * N + 4 * G * N + 2 * M * N)


def test_roofline_bound_follows_arithmetic_intensity():
    """Decode buckets are bound by HBM, prefill buckets by the INT8 tensor
    peak (twice the measured bf16 figure); the fraction is the roofline time
    over the measured time."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"hbm": 6551.0, "bf16": 1666.8, "bf16_sus": 1391.0, "kind": "measured"}
    K, N, nO = 8192, 28672, 82
    for M, bound in [(1, "hbm"), (16, "hbm"), (1024, "tensor"), (8192, "tensor")]:
        ops, nb = 2 * M * K * N, bench.layer_bytes(M, K, N, nO, 1)
        t_roof = max(nb / 6551e9, ops / (2 * 1666.8e12))
        r = bench.roofline_of(ops, nb, 2 * t_roof, peaks)
        assert r["bound"] == bound, M
        assert abs(r["frac"] - 0.5) < 1e-9
        assert r["peak"] == (6551.0 if bound == "hbm" else 2 * 1666.8)
