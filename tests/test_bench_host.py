"""Host-side arithmetic of bench.py, without a GPU: the algorithmic byte and
FLOP counts that every roofline fraction divides by, summed here tensor by
tensor from the definition of each entry point, the band's key count against
brute force, and the two files the bench reads (measured peaks, committed
ncu traffic) with their fallbacks."""
import json
import os

import pytest

import bench
import workloads

BF16, F32 = 2, 4


def row(heads, D=128, elt=BF16):
    """Bytes of one token's rows for `heads` heads."""
    return heads * D * elt


def test_forward_bytes_are_q_g_o_and_k_v():
    c = workloads.LAYER
    per_token = row(32) + row(32) + row(32) + row(8) + row(8)  # q, g in; o out; k, v in
    assert bench.FWD_BYTES_PER_TOKEN(c) == per_token == 28_672
    assert per_token * c.B * c.T == 469_762_048              # one layer-shape launch
    assert per_token * workloads.LONG.T == 7_516_192_768      # the 1 x 262144 step


def test_backward_and_training_step_bytes():
    c = workloads.TRAIN
    reads = row(32) * 3 + row(8) * 2 + 32 * F32   # q, g, dO; k, v; lse
    writes = row(32) * 2 + row(8) * 2             # dq, dg; dk, dv
    assert bench.BWD_BYTES_PER_TOKEN(c) == reads + writes == 49_280
    # forward with its lse write, then the backward
    step = bench.FWD_BYTES_PER_TOKEN(c) + 32 * F32 + bench.BWD_BYTES_PER_TOKEN(c)
    assert step == 78_080
    assert step * c.T == 1_279_262_720


def test_decode_bytes_per_sequence_and_layer():
    c = workloads.DECODE
    older_slots = (128 - 1) * row(8) * 2   # K and V of the 127 older ring slots
    new_kv_in = row(8) * 2
    slot_writes = row(8) * 2
    q_g_o = row(32) * 3
    assert bench.DECODE_BYTES_PER_SEQ_LAYER(c) == older_slots + new_kv_in + slot_writes + q_g_o
    assert bench.DECODE_BYTES_PER_SEQ_LAYER(c) == 552_960
    assert bench.DECODE_BYTES_PER_SEQ_LAYER(c) * c.N * c.layers == 3_822_059_520


@pytest.mark.parametrize("T,W", [(1, 128), (5, 3), (127, 128), (128, 128), (129, 128),
                                 (4096, 128), (300, 1), (50, 64)])
def test_band_keys_brute_force(T, W):
    assert bench.band_keys(T, W) == sum(min(i + 1, W) for i in range(T))


def test_forward_flops_count_two_contractions_over_the_band():
    c = workloads.LAYER
    keys = sum(min(i + 1, c.W) for i in range(c.T))
    # QK^T and PV: 2 FLOPs per multiply-add, D per key, per query head and batch row
    assert bench.fwd_flops(c) == 2 * 2 * c.D * keys * c.Hq * c.B


def test_peaks_fall_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"].startswith("fallback") and p["hbm_gbs"] == 6650.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6544.0,
                                                               "bf16_tflops": 1657.0}))
    p = bench.load_peaks()
    assert p["source"].startswith("measured") and p["hbm_gbs"] == 6544.0
    assert p["bf16_tflops_sustained"] == 1657.0  # burst figure when no sustained one


def test_committed_traffic_is_dropped_when_the_kernel_changes(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    csrc = tmp_path / "hybrid_sliding_window_gated_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1\n")
    (tmp_path / "profiles").mkdir()
    digest = bench.kernel_source_digest(["k.cu"])
    (tmp_path / "profiles" / "k.txt").write_text(
        f"# header\nkernel_sources_sha256_16 = {digest}\ndram_bytes_per_launch = 1234\n")
    assert bench.committed_traffic("k.txt", ["k.cu"]) == 1234.0
    (csrc / "k.cu").write_text("kernel v2\n")
    assert bench.committed_traffic("k.txt", ["k.cu"]) is None
    assert bench.committed_traffic("missing.txt", ["k.cu"]) is None
    assert os.path.exists(tmp_path / "profiles" / "k.txt")


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` runs the oracle on the host cores (no GPU)
    and prints one JSON line with the same metric and workload as the GPU
    arm, plus its cpu_baseline and e2e blocks."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], cwd=root, env=env, capture_output=True, text=True,
                         timeout=600, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 1 and rec["steps"] == 1
    assert rec["metric"] == "gated-SWA forward tokens/s (layer-shape prefill)"
    assert rec["unit"] == "tokens/s" and rec["higher_is_better"] is True
    assert rec["config"]["workload"] == workloads.LAYER.name
    assert rec["value"] > 0 and rec["cpu_baseline"]["value"] == rec["value"]
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"] == {"value": rec["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
