"""Host-side logic of bench.py (CPU): the reference arm's per-step sample and its thread count,
the roofline's peak source and the traffic record's source check."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_sample_whole_units():
    # one unit takes 0.1 s, a step may take 1 s: 10 passes of 16 parallel units, capped at B
    units, n, cores = bench.reference_sample(B=32, N=3136, threads=16, unit_s=0.1, budget=1.0)
    assert (units, n, cores) == (32, 3136, 16)
    units, n, cores = bench.reference_sample(B=32, N=3136, threads=16, unit_s=0.4, budget=1.0)
    assert (units, n, cores) == (32, 3136, 16)
    units, n, cores = bench.reference_sample(B=32, N=3136, threads=16, unit_s=0.9, budget=1.0)
    assert (units, n, cores) == (16, 3136, 16)


def test_reference_sample_token_prefix_keeps_every_thread_busy():
    """When one whole unit overruns the budget, every thread still gets a unit (cut to its
    first n tokens), and the reported cores equal the threads actually used."""
    units, n, cores = bench.reference_sample(B=32, N=3136, threads=16, unit_s=0.12, budget=0.006)
    assert units == 16 and cores == 16
    assert n == int(3136 * 0.006 / 0.12)
    # fewer units than threads: the oracle caps its threads at the unit count
    units, n, cores = bench.reference_sample(B=4, N=3136, threads=16, unit_s=0.12, budget=0.006)
    assert units == 4 and cores == 4
    units, n, cores = bench.reference_sample(B=32, N=3136, threads=1, unit_s=0.12, budget=0.006)
    assert units == 1 and cores == 1


def test_cores_never_exceed_units():
    for B in (1, 3, 32):
        for threads in (1, 8, 64):
            for unit_s, budget in ((0.1, 5.0), (0.1, 0.01), (2.0, 0.5)):
                units, n, cores = bench.reference_sample(B, 3136, threads, unit_s, budget)
                assert 1 <= units <= B and 16 <= n <= 3136
                assert cores == min(threads, units)


def test_peaks_fall_back_and_say_so(tmp_path, monkeypatch):
    """Without MEASURED_PEAKS.json the roofline divides by the fallback and labels it; with the
    file it uses the measured figures (burst and sustained)."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    hbm, burst, sust, src = bench.peaks()
    assert (hbm, src) == (bench.FALLBACK_HBM_GBS, "fallback") and burst > sust > 0
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 6538.3, "bf16_tflops": 1674.7, "bf16_tflops_sustained": 1364.0}')
    assert bench.peaks() == (6538.3, 1674.7, 1364.0, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6538.3}')  # incomplete: fallback
    assert bench.peaks()[3] == "fallback"


def test_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    """The DRAM traffic of a committed ncu summary is reported only while the kernel source
    hashes to the summary's kernel_source_sha; after any edit it becomes null."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cuh"
    src.write_text("__global__ void k() {}\n")
    _, sha = bench.kernel_traffic(["k.cuh"], "k.md")
    (tmp_path / "profiles" / "k.md").write_text(
        f"# k\n\nkernel_source_sha: {sha}\ntraffic_bytes_per_launch: 12345\n")
    assert bench.kernel_traffic(["k.cuh"], "k.md") == (12345.0, sha)
    src.write_text("__global__ void k() { }\n")
    traffic, sha2 = bench.kernel_traffic(["k.cuh"], "k.md")
    assert traffic is None and sha2 != sha
    assert bench.kernel_traffic(["k.cuh"], "missing.md")[0] is None
