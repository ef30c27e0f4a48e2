"""The bench's JSON record, assembled on the CPU from fake timings: both branches of the committed
ncu record (matching the kernel sources, and stale), so that the line the bench prints is built
here before it is built on a GPU."""
import json

import pytest

import bench


def _fake_record(monkeypatch, rec):
    monkeypatch.setattr(bench, "profile_record", lambda: rec)


def _line(R=73, steps=20, B=1, world=1, per_launch=23.4e-6, e2e_factor=1.5):
    secs = steps * R * per_launch
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 12}
    return bench.build_line(steps, 5, R, B, world, secs, secs * e2e_factor, clk, 148, "NVIDIA B200")


REQUIRED = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"]


def test_line_with_matching_ncu_record(monkeypatch):
    _fake_record(monkeypatch, {"traffic_bytes_per_launch": 8_000_000, "warp_instructions_per_launch": 1_000_000})
    line = _line()
    json.dumps(line)
    for k in REQUIRED:
        assert k in line, k
    alg = bench.algorithmic_bytes()
    assert line["value"] == pytest.approx(alg / 23.4e-6 / 1e9)
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["traffic"] == 8_000_000
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    ir = line["issue_roofline"]
    assert ir["achieved"] == pytest.approx(1_000_000 * 32 / 23.4e-6)
    assert ir["peak"] == pytest.approx(148 * 4 * 32 * 1965e6)
    assert line["e2e"]["value"] == pytest.approx(line["value"] / 1.5)
    assert line["e2e"]["h2d_bytes_per_step"] == 73 * bench.NB * 24 * 2
    assert line["e2e"]["d2h_bytes_per_step"] == 73 * bench.ROWS * 4
    assert line["gpu_launches"] == 20 * 73
    assert line["ms_per_step"] == pytest.approx(73 * 23.4e-3)


def test_line_with_stale_ncu_record(monkeypatch):
    _fake_record(monkeypatch, None)
    line = _line()
    json.dumps(line)
    assert line["roofline"]["traffic"] is None
    assert line["issue_roofline"] is None


def test_line_batch_and_ranks(monkeypatch):
    _fake_record(monkeypatch, None)
    line = _line(B=4, world=2)
    json.dumps(line)
    assert "issue_roofline" not in line
    assert line["n_gpus"] == 2
    # whole job: both ranks' bytes over the max time
    assert line["value"] == pytest.approx(2 * bench.algorithmic_bytes(batch=4) / 23.4e-6 / 1e9)
    assert line["roofline"]["achieved"] == pytest.approx(bench.algorithmic_bytes(batch=4) / 23.4e-6 / 1e9)


def test_committed_record_is_read_when_sources_match(monkeypatch, tmp_path):
    rec = {"kernel_sources_sha256": bench.kernel_sources_hash(), "traffic_bytes_per_launch": 123,
           "warp_instructions_per_launch": 456}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda: rec["kernel_sources_sha256"])
    assert bench.profile_record() == rec
    assert bench.measured_traffic() == 123
    line = _line()
    assert line["issue_roofline"]["achieved"] == pytest.approx(456 * 32 / 23.4e-6)


def test_search_roofline_line(monkeypatch):
    """The search line's fp64 roofline: algorithmic FMAs (class-codeword pairs x (groups + 1)) x 2
    per launch over the launch time, against SMs x 64 FMA lanes x 2 x the clock; the DRAM traffic
    only from a record of the same launch size."""
    r = {"n": bench.SEARCH_N, "max_shell": 13, "ms_per_launch": 102.0}
    monkeypatch.setattr(bench, "search_record", lambda: {"n": bench.SEARCH_N, "traffic_bytes_per_launch": 13_379_840})
    ro = bench.search_roofline(r, 1965.0, 148)
    json.dumps(ro)
    assert ro["bound"] == "alu" and ro["unit"] == "TFLOP/s"
    assert ro["achieved"] == pytest.approx(2 * 3_805_180 * bench.SEARCH_N / 0.102 / 1e12)
    assert ro["peak"] == pytest.approx(148 * 64 * 2 * 1965e6 / 1e12)
    assert ro["frac"] == pytest.approx(ro["achieved"] / ro["peak"]) and 0.2 < ro["frac"] < 0.3
    assert ro["traffic"] == 13_379_840
    monkeypatch.setattr(bench, "search_record", lambda: {"n": 1024, "traffic_bytes_per_launch": 1})
    assert bench.search_roofline(r, 1965.0, 148)["traffic"] is None
    monkeypatch.setattr(bench, "search_record", lambda: None)
    assert bench.search_roofline(r, 1965.0, 148)["traffic"] is None


def test_search_fma_counts_match_the_class_list():
    """SEARCH_FMAS (the roofline's algorithmic work) recounted from the oracle's class list: for each
    class of shells 2..M, its codewords (4096 odd; those of weight k even) x (nonzero groups + 1)."""
    import oracle
    words = {0: 1, 8: 759, 12: 2576, 16: 759, 24: 1}
    o = oracle.Codec(48)
    for M, fmas in bench.SEARCH_FMAS.items():
        n = 0
        for c in o.classes():
            if c.m <= M:
                n += (4096 if c.odd else words[c.k]) * (sum(1 for v in c.vals if v) + 1)
        assert n == fmas, M
