"""The bench's roofline arithmetic on the host: the per-kernel FLOP table, the choice between the
burst and the sustained GEMM peak, and the DRAM-traffic lookup that is only trusted while the
kernel's source is unchanged since the capture."""
import hashlib
import json
import os

import bench
from workloads import get_config


def test_expert_gemm_flops_sum_to_eighteen_ndh():
    # Forward: X W1, X W3 (2 N d 2h) and A W2 (2 N h d); backward: dA (2 N d h), dX (2 N 2h d),
    # dW1 / dW3 (2 N d 2h), dW2 (2 N h d): 18 N d h in all, the figure the bench's GEMM rate uses.
    for name in ("dsv3_bf16", "dsmoe16b_bf16", "finegrained_bf16", "small_ragged_bf16"):
        cfg = get_config(name)
        total = 0.0
        for k in bench.gemm_names():
            kind, flops = bench.kernel_work(cfg, k)
            assert kind == "tensor", k
            total += flops
        assert total == 18.0 * cfg.N * cfg.d * cfg.h
        assert bench.gemm_summary(cfg, {}, 1, 1.0)["flops_per_step"] == total


def test_gate_and_row_kernels_are_counted():
    cfg = get_config("dsv3_bf16")
    T, d, E, k = cfg.T, cfg.d, cfg.E, cfg.k
    N = T * k
    assert bench.kernel_work(cfg, "gate_logits") == ("tensor", 2.0 * T * d * E)
    # the gather-sum reads each of the N PFT rows once and writes T rows (BF16), plus 8 bytes per slot
    assert bench.kernel_work(cfg, "combine") == ("hbm", float(N * d * 2 + T * d * 2 + 8 * N))
    assert bench.kernel_work(cfg, "no_such_kernel") == (None, None)


def test_tensor_peak_burst_for_short_passes_sustained_for_long():
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1350.0}
    pk, src = bench.tensor_peak(peaks, "measured", 400.0)
    assert pk == 1600.0 and "burst" in src
    pk, src = bench.tensor_peak(peaks, "measured", 9000.0)
    assert pk == 1350.0 and "sustained" in src
    pk, _ = bench.tensor_peak({}, "fallback", 10.0)
    assert pk == bench.PEAKS_FALLBACK["bf16_tflops"]


def test_traffic_is_used_only_while_the_source_is_unchanged(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_bytes(b"// kernel v1\n")
    os.makedirs(tmp_path / "profiles")
    entry = {"dram_bytes_per_launch": 12345, "source": "kernel.cu",
             "source_sha256": hashlib.sha256(b"// kernel v1\n").hexdigest()}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"wl": {"kern": entry}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("kern", "wl") == 12345
    assert bench.traffic_for("kern", "other_workload") is None
    assert bench.traffic_for("other_kernel", "wl") is None
    src.write_bytes(b"// kernel v2\n")
    assert bench.traffic_for("kern", "wl") is None


def test_committed_traffic_entries_name_existing_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    entries = [e for wl, ks in t.items() if not wl.startswith("_") for e in ks.values()]
    assert entries
    for e in entries:
        assert os.path.exists(os.path.join(bench.ROOT, e["source"]))
        assert os.path.exists(os.path.join(bench.ROOT, e["capture"]))
        assert e["dram_bytes_per_launch"] > 0
