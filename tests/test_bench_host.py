"""Host-side accounting of bench.py: the recorded DRAM traffic table, the
algorithmic work per kernel and the reference arm's oracle sample (no GPU)."""
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


def test_oracle_sample_slices_stay_small_and_consistent():
    """The reference arm's sample: the ffn slice is a whole number of
    16-column blocks, tokens times width track the fraction, and the
    smallest sample runs in well under a second per step."""
    import time
    cfg = W.CONFIGS["moe_t2048_h1024_e8k2_f2048"]
    s = bench.OracleSample(cfg, seed=0, frac=1e-6)
    assert (s.F_s, s.T_s, s.rows_gu, s.rows_d) == (16, 1, 16, 16)
    t0 = time.perf_counter()
    s.run()
    assert time.perf_counter() - t0 < 5.0
    for f in (1.0 / 1024, 1.0 / 64):
        s.set_fraction(f)
        assert s.F_s % 16 == 0 and 16 <= s.F_s <= cfg.F
        got = s.T_s * s.F_s / (cfg.T * cfg.F)
        assert 0.5 * f <= got <= 2.0 * f, (f, got)
        assert s.flops > 0 and int((s.chan_h_s >= 0).sum()) <= s.F_s // 2


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    import argparse
    args = argparse.Namespace(impl="reference", gpus=2, steps=1, warmup=0, workload="moe_t2048_h1024_e8k2_f2048")
    assert bench.run_reference(args) == 0
