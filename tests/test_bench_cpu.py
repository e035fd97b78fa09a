"""bench.py on the CPU: the reference arm end to end and the host-side bookkeeping.

The reference arm times the float64 oracle on the host cores and must print one
JSON line with the contract's keys; the algorithmic byte and FLOP counts that
the roofline fractions divide by are checked against a hand count.
"""

import json
import os
import subprocess
import sys
import types

import pytest

import bench
from lsh_attention_hash_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run_reference(*extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "1", "--warmup", "3", *extra]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, check=True).stdout
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out
    return json.loads(lines[0])


@pytest.mark.parametrize("extra,mask", [((), None), (("--causal", "--union"), "causal+bucket+union")])
def test_reference_arm_prints_one_contract_line(extra, mask):
    line = _run_reference(*extra)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "gpu_launches"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["gpu_launches"] == 0
    assert line["config"].get("mask") == mask
    assert line["config"]["seq_len"] == synth.WORKLOADS["tiny"].L


def test_mask_options_and_config():
    ns = types.SimpleNamespace
    assert bench.mask_config(ns(causal=False, bucket_mask=False, union=False)) == {}
    assert bench.mask_config(ns(causal=True, bucket_mask=False, union=False)) == {"mask": "causal"}
    assert bench.mask_config(ns(causal=False, bucket_mask=False, union=True)) == {"mask": "bucket+union"}
    assert bench.mask_options(ns(causal=False, bucket_mask=False, union=True)) == {
        "causal": False, "bucket_mask": True, "union": True}


def test_algorithmic_counts_of_the_64k_step():
    """Hand count for B 8, H 8, L 65536, D 128, bf16, 8 rounds, chunk 64, 1024 buckets."""
    w = synth.WORKLOADS["64k"]
    a = bench.algorithmic(w)
    T, TR, row = 8 * 8 * 65536, 8 * 8 * 65536 * 8, 128 * 2
    assert a["hash"]["bytes"] == T * row + TR * 4                 # read x, write the buckets
    assert a["sort"]["bytes"] == TR * 8                           # read the buckets, write perm
    assert a["attend"]["bytes"] == TR * (4 + 2 * row + row + 4)   # perm, gather QK and V, write o_r and lse
    assert a["combine"]["bytes"] == TR * (row + 4) + T * row       # read o_r and lse, write out
    assert a["total_bytes"] == sum(a[s]["bytes"] for s in bench.STAGES)
    assert abs(a["total_bytes"] / 1e9 - 37.31) < 0.01
    # a 64 x 128 window per query: QK^T and PV, 2 flops per multiply-add
    assert a["attn_flops"] == 2 * 2 * TR * (2 * w.chunk) * w.D
    assert a["hash"]["flops"] == 2 * T * w.D * 512 * 8


def test_peaks_come_from_the_measured_file_when_present():
    peaks, src = bench.load_peaks()
    assert set(peaks) == set(bench.FALLBACK_PEAKS)
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert src.startswith("measured")
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            assert peaks["hbm_gbs"] == float(json.load(f)["hbm_gbs"])


def test_backward_flop_count_and_alu_peak():
    w = synth.small_workload("bwd_count", 1, 1, 256, 64, "f32", 8, 64, 2)
    # chunk 0: 64 queries x 64 keys; chunks 1..3: 64 queries x 128 keys; per round
    pairs = 2 * (64 * 64 + 3 * 64 * 128)
    assert bench.backward_flops(w) == 10 * 64 * pairs
    assert abs(bench.alu_peak_tflops(148, 1965.0) - 74.45) < 0.01


def test_reference_arm_under_torchrun_prints_once():
    """Launched as two ranks (as the driver launches N > 1), rank 0 alone prints the line."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", "--master-port=29533", os.path.join(ROOT, "bench.py"), "--impl",
           "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3", "--gpus", "2"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, check=True).stdout
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
