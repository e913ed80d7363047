"""Host-side accounting of bench.py: the recorded DRAM traffic table and the
algorithmic work per kernel (no GPU)."""
import bench
from train_alignment_b200 import workloads as W


def test_traffic_rows_match_kernel_names():
    cfg = W.CONFIGS["moe_t2048_h1024_e8k2_f2048"]
    names = set(bench.kernel_work(cfg, 5120))
    for src, kernels in bench.KERNEL_SOURCES.items():
        assert set(kernels) <= names, src
    assert names <= {k for ks in bench.KERNEL_SOURCES.values() for k in ks}


def test_recorded_traffic_is_positive_or_stale():
    for k in bench.kernel_work(W.CONFIGS["moe_t2048_h1024_e8k2_f2048"], 5120):
        t = bench.recorded_traffic("moe_t2048_h1024_e8k2_f2048", k)
        assert t is None or t > 0
    assert bench.recorded_traffic("no_such_workload", "gemm_gate_up") is None


def test_stale_hash_gives_null(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    good = bench.source_hash("gemm_gate_up")
    (prof / "traffic.md").write_text(
        "| workload | kernel | r | w | us | source |\n|---|---|---|---|---|---|\n"
        f"| wl | gemm_gate_up | 100 | 20 | 1.0 | `{good}` |\n"
        "| wl | gemm_down | 100 | 20 | 1.0 | `000000000000` |\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_hash", lambda k: good)
    assert bench.recorded_traffic("wl", "gemm_gate_up") == 120.0
    assert bench.recorded_traffic("wl", "gemm_down") is None


def test_whole_job_aggregate():
    assert bench.whole_job_tflops(2e12, 4, 1000.0) == 8.0
