"""Host logic of bench.py on CPU: the figures it takes from a committed ncu
summary, and the oracle baseline's bounded sample.

A summary's figures (DRAM bytes per launch, pipe shares) describe one kernel
source. The bench must report them only while the attention sources still
hash to the value the summary records, and null otherwise.
"""
import bench
import workloads


def _write_summary(root, name, digest, extra=""):
    d = root / "profiles"
    d.mkdir(parents=True, exist_ok=True)
    (d / f"attn_fwd_{name}.md").write_text(
        "# capture\n\n| metric | value |\n|---|---|\n\n"
        "dram_bytes_per_launch: 1288714752\n"
        "tensor_pipe_pct_active: 49.9\n"
        "mufu_pipe_pct_active: 37.8\n"
        f"kernel_source_sha256_16: {digest}\n" + extra)


def test_profile_figures_follow_the_source_hash(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "attn_source_hash", lambda: "00112233aabbccdd")
    _write_summary(tmp_path, "w", "00112233aabbccdd")
    assert bench.profile_figures("w") == {"traffic": 1288714752.0, "tensor_pipe_pct": 49.9,
                                          "mufu_pipe_pct": 37.8}
    # the kernel source changed since the capture: every figure is withdrawn
    monkeypatch.setattr(bench, "attn_source_hash", lambda: "ffffffffffffffff")
    assert bench.profile_figures("w") == {"traffic": None, "tensor_pipe_pct": None, "mufu_pipe_pct": None}


def test_profile_figures_missing_summary_or_lines(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "attn_source_hash", lambda: "0123456789abcdef")
    assert bench.profile_figures("absent") == {"traffic": None, "tensor_pipe_pct": None, "mufu_pipe_pct": None}
    d = tmp_path / "profiles"
    d.mkdir()
    (d / "attn_fwd_partial.md").write_text("dram_bytes_per_launch: 5\nkernel_source_sha256_16: 0123456789abcdef\n")
    assert bench.profile_figures("partial") == {"traffic": 5.0, "tensor_pipe_pct": None, "mufu_pipe_pct": None}


def test_cpu_baseline_counts_kept_tiles_and_times_the_block_mask():
    w = workloads.get(1)
    data = workloads.make(w)
    r = bench.cpu_baseline(w, data)
    # causal over 2 x 2 tiles keeps 3 (one full, two partial)
    assert "3 kept tiles" in r["sample"]
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
    bm = r["block_mask"]
    assert bm["unit"] == "GB/s" and bm["value"] > 0 and "2 x 2 tiles" in bm["sample"]
    # with the tile classes given (the reference arm), no block-mask timing
    from oracle import block_mask as obm
    cls = obm.tile_classes(data["mask"], 0, w.M, w.N)
    r2 = bench.cpu_baseline(w, data, cls=cls)
    assert "3 kept tiles" in r2["sample"] and "block_mask" not in r2


def test_clock_sampler_keeps_the_timed_window():
    """The summary keeps the samples read inside the timed region (and one
    interval after it); with none there it falls back to all samples and
    says so."""
    s = bench.ClockSampler(0)
    row = "0, {mhz}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {cap}"
    s.lines = [(1.000, row.format(mhz=1000, cap="Not Active")),   # before the region
               (2.005, row.format(mhz=1965, cap="Active")),       # inside
               (2.030, row.format(mhz=1950, cap="Not Active")),   # inside
               (2.070, row.format(mhz=1900, cap="Not Active")),   # within one interval after the end
               (3.000, row.format(mhz=500, cap="Not Active"))]    # after
    s.t0, s.t1 = 2.0, 2.05
    c = s.summary()
    assert c["in_window"] and c["samples"] == 3 and c["sm_mhz"] == 1950.0
    assert c["reasons"] == ["sw_power_cap"] and c["sm_max_mhz"] == 1965.0
    assert c["window_ms"] == 50.0
    s.t0, s.t1 = 2.5, 2.51  # no sample inside: every sample is used
    c = s.summary()
    assert not c["in_window"] and c["samples"] == 5
