"""The roofline arithmetic of bench.py, on the host: the per-launch algorithmic work of each
step kernel, the choice of the binding floor, the achieved / peak fraction, and the rule
that DRAM traffic from a committed ncu summary is reported only while the kernel source
it was measured on is unchanged.

The work counts are checked against an independent enumeration: the bytes of every
tensor a launch must read or write at least once (features, neighbour table, weights,
bias, gradients) and the multiply-adds of the 9-tap sum over the kept tokens, summed
tensor by tensor from their shapes."""
import hashlib
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PEAKS = {"hbm_gbs": 6549.4, "bf16_tflops": 1586.2, "source": "measured"}


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def tensor_bytes(shapes_and_sizes):
    total = 0
    for shape, elem in shapes_and_sizes:
        count = 1
        for d in shape:
            count *= d
        total += count * elem
    return total


@pytest.mark.parametrize("n,T,Cin,Cout,elem,elem_out,bias", [
    (49477, 384, 256, 256, 2, 2, True),   # the large-channel step
    (29568, 384, 64, 64, 2, 2, True),     # the small-channel step
    (49152, 384, 256, 256, 1, 2, True),   # e4m3 inputs, bf16 output
    (128, 2, 16, 16, 4, 4, False),        # fp32, no bias
])
def test_conv_work_counts_each_tensor_once(bench, n, T, Cin, Cout, elem, elem_out, bias):
    w = bench.conv_work(n, T, Cin, Cout, elem, bias, elem_out)
    table = ((n, 9), 4)                   # N: 9 int32 per token
    weights = ((Cout, 9, Cin), elem)      # W
    fwd = tensor_bytes([((n, Cin), elem), ((n, Cout), elem_out), table, weights] + ([((Cout,), 4)] if bias else []))
    bwd_data = tensor_bytes([((n, Cout), elem), ((n, Cin), elem), table, weights])
    bwd_weight = tensor_bytes([((n, Cout), elem), ((n, Cin), elem), table, ((Cout, 9, Cin), 4), ((Cout,), 4)])
    index = tensor_bytes([((n, 3), 4), ((T + 1,), 4), table])  # (t, y, x) per token, frame offsets, N written
    assert w["fwd"]["bytes"] == fwd
    assert w["bwd_data"]["bytes"] == bwd_data
    assert w["bwd_weight"]["bytes"] == bwd_weight
    assert w["build_index"]["bytes"] == index and w["build_index"]["flops"] == 0
    # one multiply-add (2 flops) per (token, tap, input channel, output channel), for each pass
    taps = 9
    macs = n * taps * Cin * Cout
    for k in ("fwd", "bwd_data", "bwd_weight"):
        assert w[k]["flops"] == 2 * macs


def test_headline_work_matches_the_stated_figures(bench):
    w = bench.conv_work(49477, 384, 256, 256, 2, True)
    assert w["fwd"]["flops"] == 58365444096
    assert abs(w["fwd"]["bytes"] / 1e6 - 53.63) < 0.01       # 28.3 MB read + 25.3 MB of Y
    assert abs(w["bwd_weight"]["bytes"] / 1e6 - 54.80) < 0.01  # 52.4 MB read + 2.4 MB of dW, db


def test_roofline_takes_the_larger_floor(bench):
    big = bench.conv_work(49477, 384, 256, 256, 2, True)["bwd_weight"]
    r = bench.roofline_entry(big, 0.0702, PEAKS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(big["flops"] / 70.2e-6 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops"])
    assert r["frac"] == pytest.approx(0.524, abs=0.001)
    # C = 64: 250 flop/B against a measured ridge of 1586.2e12 / 6549.4e9 = 242 flop/B
    small = bench.conv_work(29568, 384, 64, 64, 2, True)["fwd"]
    assert small["flops"] / small["bytes"] > PEAKS["bf16_tflops"] * 1e12 / (PEAKS["hbm_gbs"] * 1e9)
    assert bench.roofline_entry(small, 0.015, PEAKS)["bound"] == "tensor"
    # a pure byte mover is HBM-bound, reported in GB/s
    r = bench.roofline_entry({"bytes": 6549.4e6, "flops": 0}, 1.0, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["frac"] == pytest.approx(1.0)


def test_e4m3_and_fp32_peaks(bench):
    assert bench.flop_peak(PEAKS, fp8=True) == pytest.approx(2 * PEAKS["bf16_tflops"])
    assert bench.flop_peak(PEAKS, alu=True) == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)
    work = bench.conv_work(49152, 384, 256, 256, 1, True, 2)["fwd"]
    r = bench.roofline_entry(work, 0.039, PEAKS, fp8=True)
    assert r["peak"] == pytest.approx(2 * PEAKS["bf16_tflops"]) and r["bound"] == "tensor"
    assert bench.floor_seconds(work, PEAKS, fp8=True) == pytest.approx(work["flops"] / (2 * PEAKS["bf16_tflops"] * 1e12))


def test_traffic_is_reported_only_for_the_source_it_was_measured_on(bench, tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"w/k": {"source": "kernel.cu", "source_sha": sha, "dram_bytes_per_launch": 12345}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("w", "k") == 12345
    assert bench.kernel_traffic("w", "other") is None
    src.write_text("// kernel v2\n")  # the kernel changed after the counters were taken
    assert bench.kernel_traffic("w", "k") is None


def test_committed_traffic_entries_name_their_source(bench):
    """Every committed entry names an existing kernel source and the sha256 prefix it was
    measured on (bench.py reports null for an entry whose source has changed since)."""
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    entries = {k: v for k, v in d.items() if not k.startswith("_")}
    assert entries
    for key, ent in entries.items():
        assert os.path.exists(os.path.join(ROOT, ent["source"])), key
        assert len(ent["source_sha"]) == 16 and int(ent["source_sha"], 16) >= 0, key
        assert ent["dram_bytes_per_launch"] > 0, key
