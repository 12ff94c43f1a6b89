"""Host arithmetic of bench.py, on CPU: the roofline's algorithmic bytes
and flops, the measured-peak lookup and its fallback, and the rule that a
recorded DRAM traffic figure is used only for the kernel source it was
captured on."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


# Per-workload totals worked out independently of bench.py (A and B read
# once, one E8M0 byte per 32 elements of each row, BF16 C written once).
@pytest.mark.parametrize("fmt,M,N,K,alg_bytes", [
    (0, 32, 256, 512, 168_448),
    (1, 32, 14336, 4096, 32_182_272),
    (0, 64, 4096, 4096, 18_096_128),
    (1, 64, 4096, 4096, 9_576_448),
    (0, 2048, 28672, 8192, 376_963_072),
    (1, 2048, 28672, 8192, 251_133_952),
    (0, 8192, 8192, 8192, 272_629_760),
    (1, 8192, 8192, 8192, 205_520_896),
    (0, 4096, 4096, 14336, 154_664_960),
    (1, 4096, 4096, 14336, 95_944_704),
])
def test_algorithmic_bytes_of_the_workloads(fmt, M, N, K, alg_bytes):
    assert bench.algorithmic_bytes(fmt, M, N, K) == alg_bytes
    assert bench.flops(M, N, K) == 2.0 * M * N * K


def test_every_named_workload_resolves():
    from microscaling_block_scaled_b200 import synth
    for name in synth.WORKLOADS:
        fmt_name, M, N, K, seed, kind = bench.workload(name)
        assert fmt_name in ("mxfp8", "mxfp4") and K % 128 == 0 and kind in ("normal", "heavy")
    assert bench.DEFAULT_WORKLOAD in synth.WORKLOADS
    with pytest.raises(SystemExit):
        bench.workload("no_such_workload")


def test_measured_peaks_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, how = bench.measured_peaks()
    assert how == "fallback" and peaks["hbm_gbs"] == 6650.0 and peaks["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7000.0, "bf16_tflops": 1700.0}))
    peaks, how = bench.measured_peaks()
    assert how == "measured" and peaks["hbm_gbs"] == 7000.0


def test_recorded_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("mxfp4_32x14336x4096", "one_cta") is None        # no file
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(
        {"mxfp4_32x14336x4096": {"kernel_hash": "aaaa", "dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "kernel_hash", lambda kind: "aaaa" if kind == "one_cta" else "cccc")
    assert bench.recorded_traffic("mxfp4_32x14336x4096", "one_cta") == 123
    assert bench.recorded_traffic("mxfp4_32x14336x4096", "pair") is None            # another kernel
    assert bench.recorded_traffic("mxfp8_32x256x512", "one_cta") is None           # not captured
    monkeypatch.setattr(bench, "kernel_hash", lambda kind: "bbbb")
    assert bench.recorded_traffic("mxfp4_32x14336x4096", "one_cta") is None        # kernel changed since


def test_kernel_hash_covers_each_kernels_sources():
    for kind, main in (("one_cta", "gemm_kernel.cuh"), ("pair", "gemm_pair_kernel.cuh")):
        h = bench.kernel_hash(kind)
        assert len(h) == 16 and int(h, 16) >= 0
        assert any(p.endswith(main) for p in bench.KERNEL_SOURCES[kind])
        assert any(p.endswith("gemm_common.cuh") for p in bench.KERNEL_SOURCES[kind])
    assert bench.kernel_hash("one_cta") != bench.kernel_hash("pair")


def test_schedule_overrides_parse_and_key_the_traffic():
    from microscaling_block_scaled_b200 import mxgemm
    assert bench.parse_schedule("auto") == (mxgemm.SCHED_AUTO, 1, 0)
    assert bench.parse_schedule("dp") == (mxgemm.SCHED_DP, 1, 0)
    assert bench.parse_schedule("splitk:3") == (mxgemm.SCHED_SPLITK, 3, 0)
    assert bench.parse_schedule("streamk:148") == (mxgemm.SCHED_STREAMK, 1, 148)
    assert bench.parse_schedule("ksplit:4") == (mxgemm.SCHED_KSPLIT, 4, 0)
    for bad in ("splitk", "splitk:0", "streamk:x", "dp:2", "fast", "ksplit:3", "ksplit"):
        with pytest.raises(SystemExit):
            bench.parse_schedule(bad)

    class A:
        workload = "mxfp4_32x14336x4096"
        schedule = "auto"
        kchunks = 0

    a = A()
    assert bench.traffic_key(a) == "mxfp4_32x14336x4096" and bench.override_config(a) == {}
    a.schedule, a.kchunks = "splitk:2", 1
    assert bench.traffic_key(a) == "mxfp4_32x14336x4096@splitk2_kc1"
    assert bench.override_config(a) == {"planner_override": "splitk2_kc1"}


def test_committed_traffic_matches_the_kernel_sources():
    """Every recorded DRAM-traffic figure under profiles/ was captured on the
    current source of its kernel (and planner), so the default workload's
    roofline.traffic is filled in."""
    with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
        d = json.load(f)
    for name, e in d.items():
        if name == "_about":
            continue
        kind = "pair" if "pair" in e["kernel"] else "one_cta"
        assert bench.recorded_traffic(name, kind) == e["dram_bytes_per_launch"], name
    assert bench.recorded_traffic(bench.DEFAULT_WORKLOAD, "pair") is not None
