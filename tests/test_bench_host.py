"""Host-side pieces of bench.py (no GPU): the algorithmic work model, the
per-shape table of multi-linear workloads, and the DRAM-traffic record that
must match the current kernel sources."""
import importlib.util
import os
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_algorithmic_work_of_the_prefill_linear(bench):
    w = bench.algorithmic_work_mnk(2048, 4096, 4096, 2, 2, 8)
    assert w["calib_absmax"]["bytes"] == 2 * 2048 * 4096 + 4 * 4096            # X once + absmax
    assert w["w8a8_gemm_dequant"]["ops"] == 2 * 2048 * 4096 * 4096
    assert w["w8a8_gemm_dequant"]["bytes"] == 2048 * 4096 + 4096 * 4096 + 4 * 2048 + 4 * 4096 + 2 * 2048 * 4096
    assert w["sq_pack_int4"]["bytes"] == 0
    w4 = bench.algorithmic_work_mnk(16, 8192, 28672, 2, 2, 4)
    # int4: the codes are packed (read N K, write N K / 2) and read packed by the GEMM
    assert w4["sq_pack_int4"]["bytes"] == 28672 * 8192 * 3 // 2
    assert w4["w8a8_gemm_dequant"]["bytes"] - 16 * 8192 - 4 * 16 - 4 * 28672 - 2 * 16 * 28672 == 28672 * 8192 // 2


def test_per_shape_table_groups_linears_by_shape(bench):
    probs = [SimpleNamespace(M=8192, K=1024, N=3072), SimpleNamespace(M=8192, K=1024, N=1024),
             SimpleNamespace(M=8192, K=1024, N=3072)]
    # ms per kernel (NAMES order: calib, smooth, ssz, pack, act quant, gemm) per linear
    assert bench.NAMES == ["calib_absmax", "smooth_fold", "ssz_quant_weight", "sq_pack_int4", "quant_act_per_token",
                           "w8a8_gemm_dequant"]
    lin = [[0.01, 0.01, 0.05, 0.0, 0.01, 0.030], [0.01, 0.01, 0.04, 0.0, 0.01, 0.020],
           [0.03, 0.01, 0.07, 0.0, 0.01, 0.030]]
    t = bench.per_shape_table(probs, lin, {"bf16_tflops": 1000.0})
    assert set(t) == {"8192x1024->3072", "8192x1024->1024"}
    qkv = t["8192x1024->3072"]
    assert qkv["linears"] == 2
    assert qkv["us"]["calib_absmax"] == pytest.approx(20.0)
    tops = 2 * 8192 * 1024 * 3072 / 30e-6 / 1e12
    assert qkv["gemm_tops"] == pytest.approx(round(tops, 1))
    assert qkv["gemm_frac"] == pytest.approx(round(tops / (1000.0 * bench.INT8_OVER_BF16), 4))
    assert qkv["linear_tops"] == pytest.approx(round(2 * 8192 * 1024 * 3072 / 40e-6 / 1e12, 1))


def test_per_shape_linear_time_comes_from_the_group_timing(bench):
    """With the shape groups timed back to back (shape_ms: ms a linear), the
    linear's TOPS uses that time, not the per-kernel sum (which carries the
    event nodes' latency)."""
    probs = [SimpleNamespace(M=8192, K=1024, N=1024)] * 2
    lin = [[0.0, 0.0, 0.0, 0.0, 0.012, 0.018]] * 2
    t = bench.per_shape_table(probs, lin, {"bf16_tflops": 1000.0}, {"8192x1024->1024": 0.020})
    row = t["8192x1024->1024"]
    assert row["linear_tops"] == pytest.approx(round(2 * 8192 * 1024 * 1024 / 20e-6 / 1e12, 1))
    assert row["gemm_tops"] == pytest.approx(round(2 * 8192 * 1024 * 1024 / 18e-6 / 1e12, 1))


def test_e2e_chunks(bench):
    """The end-to-end chunks: about four a linear, 256 to 2048 rows each."""
    assert bench.e2e_chunk_rows(8192) == 2048 and bench.e2e_chunk_rows(2048) == 512
    assert bench.e2e_chunk_rows(16) == 256 and bench.e2e_chunk_rows(1000) == 256
    assert bench.e2e_chunk_rows(1 << 20) == 2048
    assert bench.E2E_SLOTS >= 2


def test_default_workload_is_the_mlp_up_projection(bench):
    assert bench.DEFAULT_WORKLOAD == "mlp_up_8192x4096x11008"


def test_oracle_arm_reports_the_linear_metric(bench):
    """The oracle arm times the whole path on a small linear and reports
    2 M N K over its activation quantization + GEMM time, like our arm."""
    ops, t, sample, spent = bench.oracle_workload("single_linear_16x256x128", frac=1.0)
    assert ops == 2 * 16 * 256 * 128
    assert set(t) == {"calib_absmax", "smooth_fold", "ssz_quant_weight", "quant_act_per_token", "w8a8_gemm_dequant"}
    lin, path = bench.oracle_metric(ops, t)
    assert lin == pytest.approx(ops / (t["quant_act_per_token"] + t["w8a8_gemm_dequant"]) / 1e12)
    assert path < lin
    ops2, t2, sample2, _ = bench.oracle_workload("single_linear_16x256x128", frac=0.5)
    assert "8 of 16 tokens" in sample2 and "64 of 128 channels" in sample2


def test_recorded_traffic_matches_the_current_sources(bench):
    """profiles/dram_traffic.json is keyed by a hash of every source a step's
    kernels are built from; a recorded entry is used only while it matches,
    and each file named in the key exists."""
    for step, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(ROOT, "w8a8_linear_layers_b200", "csrc", f)), f
        got = bench.dram_traffic(step, "prefill_2048x4096x4096")
        assert got is None or got > 0
    assert bench.dram_traffic("ssz_quant_weight", "no_such_workload") is None


def test_partial_traffic_capture_keeps_other_records(bench, tmp_path, monkeypatch):
    """A capture of one kernel updates that step's record and leaves the
    workload's other records as they were."""
    import csv
    import json
    (tmp_path / "profiles").mkdir()
    path = tmp_path / "profiles" / "dram_traffic.json"
    old = {"w": {"ssz_quant_weight": {"bytes_per_launch": 7, "launches": 1, "src_sha": "a"},
                 "w8a8_gemm_dequant": {"bytes_per_launch": 5, "launches": 1, "src_sha": "old"}}}
    path.write_text(json.dumps(old))
    rows = [["ID", "Kernel Name", "Metric Name", "Metric Unit", "Metric Value"]]
    name = "void w8a8_gemm_pair_kernel<__nv_bfloat16, 0>(...)"
    rows += [["0", name, "dram__bytes_read.sum", "Mbyte", "98.5"], ["0", name, "dram__bytes_write.sum", "byte", "1,500"],
             ["0", name, "gpu__time_duration.sum", "usecond", "240"]]
    cap = tmp_path / "cap.csv"
    with open(cap, "w", newline="") as f:
        csv.writer(f, quoting=csv.QUOTE_ALL).writerows(rows)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_sha", lambda files: "new")
    bench.record_traffic(str(cap), "w")
    got = json.loads(path.read_text())["w"]
    assert got["ssz_quant_weight"] == old["w"]["ssz_quant_weight"]
    assert got["w8a8_gemm_dequant"] == {"bytes_per_launch": 98501500, "launches": 1, "src_sha": "new"}
