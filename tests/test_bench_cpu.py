"""Host logic of bench.py that runs without a GPU: the roofline byte count, the recorded
DRAM traffic lookup and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import numpy as np

import bench
from sparse_windowed_atom_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _tensor_bytes(spec):
    """The same algorithmic byte count, taken from the tensors a launch touches."""
    w = workloads.make_inputs(spec, seed=1)
    s = 2 if spec.dtype == "bfloat16" else 4
    rows = spec.B * spec.A
    hd = spec.H * spec.D
    n = w["structure"]["key_index"].nbytes + w["masks"]["window_mask"].nbytes
    if spec.style == "af3":
        n += w["activations"]["pair"].size * s
    n += rows                                  # usable flags
    n += 4 * rows * hd * s + rows * hd * s     # Q, K, V, G read; gated output written
    n += spec.B * spec.H * spec.A * spec.K * s  # attention weights written
    return n


def test_attention_bytes_match_the_tensors():
    for name in ("af3_encoder_fp32_a256", "esm_encoder_fp32_a4096"):
        spec = workloads.WORKLOADS[name]
        assert bench.attention_bytes(spec) == _tensor_bytes(spec)
    spec = workloads.tiny_spec("af3", "encoder", "bfloat16")
    assert bench.attention_bytes(spec) == _tensor_bytes(spec)


def test_attention_bytes_of_the_headline_workload():
    """The algorithmic bytes of one attention launch at the ESMFold2 bf16 workload (B=2,
    A=32768, H=8, K=128), counted by hand: 75.5 MB of key_index + window_mask, 134.2 MB of
    weights, 84.0 MB of Q/K/V/G/O and usable flags."""
    spec = workloads.WORKLOADS["esm_encoder_bf16_b2_a32768"]
    assert bench.attention_bytes(spec) == 75_497_472 + 134_217_728 + 83_951_616


def test_dense_flops_per_atom():
    spec = workloads.WORKLOADS["esm_encoder_bf16_b2_a32768"]
    assert bench.dense_flops(spec) == 851_968 * spec.B * spec.A
    dec = workloads.WORKLOADS["af3_decoder_fp32_a24576"]
    per_atom = 2 * 128 * 8 * 128 + 2 * 128 * 512 + 2 * 128 * 128 + 2 * 128 * 512 + 2 * 256 * 128 + 2 * 128 * 3
    assert bench.dense_flops(dec) == per_atom * dec.A + 2 * 384 * 128 * dec.T


def test_default_workload_is_the_largest():
    assert bench.DEFAULT_WORKLOAD == max(workloads.WORKLOADS.values(), key=lambda w: w.entries).name


def test_recorded_traffic_is_keyed_by_workload_and_source():
    v = bench.recorded_traffic(bench.DEFAULT_WORKLOAD, "k_attn_rows")
    # the committed record is taken on the current kernel source; it may only be absent
    # while a kernel change awaits its capture
    assert v is None or v > 0
    assert bench.recorded_traffic("no_such_workload") is None


def test_attention_kernel_choice():
    # every workload of the benchmark list has H*D = 128 and K <= 128: the row-gather
    # kernel for bf16 storage and small float32 problems, the per-(query, head) kernel
    # for larger float32 ones
    for w in workloads.WORKLOADS.values():
        want = "k_attn_rows" if w.dtype == "bfloat16" or w.B * w.A <= 1024 else "k_slot_attention"
        assert bench.attention_kernel(w) == want, w.name
    import dataclasses
    w = workloads.WORKLOADS["esm_encoder_bf16_b2_a32768"]
    assert bench.attention_kernel(dataclasses.replace(w, K=160)) == "k_slot_attention"
    assert bench.attention_kernel(dataclasses.replace(w, H=2, D=32)) == "k_slot_attention"
    assert bench.attention_kernel(dataclasses.replace(w, H=16, D=8)) == "k_slot_attention"


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "af3_encoder_fp32_a256", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300,
                         env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"))
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "atoms/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"] == "af3_encoder_fp32_a256"
    assert np.isfinite(d["ms_per_step"])
