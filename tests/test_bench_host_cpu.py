"""bench.py host logic on the CPU: the hash-gated DRAM traffic lookup from the committed
ncu summaries, and the clock summary built from sampled SM clocks and throttle reasons."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _summary(tmp_path, workload, digest, nbytes):
    prof = tmp_path / "profiles"
    prof.mkdir(exist_ok=True)
    (prof / f"{workload}.md").write_text(
        f"# summary\n\nworkload: {workload}\ndram_bytes_per_full_launch: {nbytes}\n"
        f"kernel_source_sha256_16: {digest}\n")


def test_traffic_only_from_a_summary_of_the_current_sources(tmp_path, monkeypatch):
    bench = _bench()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "00112233aabbccdd")
    assert bench.ncu_traffic("vit_l14_336px_b256") == (None, None)  # no summary at all
    _summary(tmp_path, "vit_l14_336px_b256", "ffffffffffffffff", 123)
    assert bench.ncu_traffic("vit_l14_336px_b256") == (None, None)  # stale sources
    _summary(tmp_path, "other_workload", "00112233aabbccdd", 456)
    assert bench.ncu_traffic("vit_l14_336px_b256") == (None, None)  # another workload
    _summary(tmp_path, "vit_l14_336px_b256", "00112233aabbccdd", 789)
    traffic, src = bench.ncu_traffic("vit_l14_336px_b256")
    assert traffic == 789.0 and src == os.path.join("profiles", "vit_l14_336px_b256.md")


def test_source_hash_covers_the_kernel_sources():
    bench = _bench()
    for rel in bench.KERNEL_SOURCES:
        assert os.path.exists(os.path.join(ROOT, rel)), rel
    h = bench.kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0


def test_clock_summary_reasons_and_median():
    bench = _bench()
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs._ok, cs.max_mhz = True, 1965
    cs._t0, cs._t1 = 10.0, 11.0
    # (host time, MHz, reasons): samples before and after the timed region are dropped.
    cs.samples = [(9.0, 1200, 0x20), (10.1, 1965, 0x1), (10.2, 1965, 0x4),
                  (10.5, 1845, 0x4 | 0x8), (10.9, 1965, 0), (11.5, 900, 0x40)]
    s = cs.summary()
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965 and s["sm_mhz_min"] == 1845
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]  # idle is not a throttle reason
    assert s["samples"] == 4
    # A region shorter than one query: the last sample before it stands in.
    cs._t0, cs._t1 = 9.5, 9.6
    s = cs.summary()
    assert s["samples"] == 1 and s["sm_mhz"] == 1200.0
    cs.samples = []
    assert cs.summary() is None
    cs._ok = False
    cs.samples = [(10.5, 1965, 0)]
    assert cs.summary() is None
