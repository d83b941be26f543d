"""Host logic of bench.py that needs no GPU: the algorithmic FLOP and byte
counts behind the roofline, the clock-sample parsing that decides whether a
run is kept, the frames a recache recomputes, and the DRAM figure taken from
a committed ncu summary, and what the reference arm (the oracle on the host
cores) reports."""
import types

import bench
import swa_workloads as W
import sink_window_attention_b200 as swa
from oracle import window


def test_algorithmic_flops_and_bytes():
    # softmax(Q K^T) V per head: 2*Nq*Nk*D for Q K^T and as many for P V
    assert bench.attention_flops(W.WAN) == 4 * 1560 * 18720 * 128 * 12          # 179.4 GFLOP per layer-step
    assert round(bench.attention_flops(W.WAN) / 1e9, 1) == 179.4
    assert bench.attention_flops(W.CHUNK) == 4 * 3 * 1560 * 18720 * 128 * 12    # 3-frame chunk: 538.3 GFLOP
    n = 1560 * 12 * 128
    # append: read K, V (bf16), write them to the cache; FP8 adds one fp32 scale per (token, head)
    assert bench.append_bytes(W.WAN, 2) == 8 * n                                 # 19.2 MB
    assert bench.append_bytes(W.WAN, 1) == 4 * n + 2 * n + 2 * 1560 * 12 * 4
    # in-place RoPE of Q: every bf16 element read once and written once
    assert bench.rope_bytes(W.WAN, 1) == 4 * n                                   # 9.58 MB
    assert bench.rope_bytes(W.CHUNK, 3) == 12 * n                                # 28.75 MB
    assert round(bench.rope_bytes(W.WAN, 1) / 1e6, 2) == 9.58
    # the recache: one GEMM of X [18720, 1536] by [Wk | Wv] [1536, 2 * 1536]
    assert bench.recache_flops(W.STREAM) == 2 * 18720 * 1536 * 3072
    assert round(bench.recache_flops(W.STREAM) / 1e9, 1) == 176.7


def _sampler_with(lines):
    s = bench.ClockSampler("0")
    s.proc = types.SimpleNamespace(terminate=lambda: None, wait=lambda timeout=None: 0, kill=lambda: None)
    s.thread = types.SimpleNamespace(join=lambda timeout=None: None)
    s.lines = lines
    return s


def test_clock_samples_give_median_and_active_reasons():
    row = "0, {sm}, 1965, 900.5, 0x{a:x}, {hw}, Not Active, Not Active, {cap}"
    lines = [row.format(sm=sm, a=4, hw="Not Active", cap="Active") for sm in (1700, 1710, 1720)]
    lines.append("garbage line")
    got = _sampler_with(lines).stop()
    assert got["sm_mhz"] == 1710 and got["sm_max_mhz"] == 1965 and got["samples"] == 3
    assert got["reasons"] == ["sw_power_cap"]
    lines.append(row.format(sm=1200, a=8, hw="Active", cap="Not Active"))
    assert _sampler_with(lines).stop()["reasons"] == ["hw_slowdown", "sw_power_cap"]
    none = bench.ClockSampler("0").stop()                  # nvidia-smi never started
    assert none["sm_mhz"] is None and none["reasons"] == ["nvidia-smi unavailable"]


def test_recache_recomputes_exactly_the_cached_frames():
    """At a prompt switch before frame F the recache rebuilds the frames the
    cache holds after frame F-1 (LongLive review, 'KV Recache'), in slot order."""
    fake = types.SimpleNamespace(w=W.STREAM, swa=swa)
    for last in (0, 1, 2, 5, 11, 12, 39, 40, 79, 919):
        held = bench.Stream.held_frames(fake, last)
        assert sorted(held) == window.attended_frames(last, 3, 9)
        assert held == [f for f in window.slot_frames(last, 3, 9) if f >= 0]


def test_traffic_figure_only_for_the_captured_kernel(tmp_path, monkeypatch):
    """The bench line's roofline.traffic comes from the committed capture file
    profiles/traffic.json only while the attention sources hash to the version
    that capture names; otherwise it is null (a stale DRAM figure is never
    reported)."""
    import json
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(
        {"k": {"kernel_source_sha256_16": "0123456789abcdef", "dram_bytes_per_launch": 230756864}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0123456789abcdef")
    assert bench.load_traffic("k") == 230756864
    assert bench.load_traffic("missing") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "fedcba9876543210")
    assert bench.load_traffic("k") is None


def test_fp8mma_cache_only_in_attention_mode(monkeypatch, capsys):
    """--cache fp8mma times the FP8 tensor-core attention alone; the stream
    line carries it as fp8_mma_stream, so the stream mode rejects it before
    touching a GPU."""
    import pytest
    monkeypatch.setattr("sys.argv", ["bench.py", "--cache", "fp8mma"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert e.value.code == 2
    assert "fp8_mma_stream" in capsys.readouterr().err


def test_stream_attention_launch_counts():
    """Launches per attention call as the bench counts them: one for a bf16
    cache, two for an E4M3 cache (the staging pass or the V-scale pass, then
    the attention kernel)."""
    st = bench.Stream.__new__(bench.Stream)
    st.caches = [types.SimpleNamespace(dtype="bf16"), types.SimpleNamespace(dtype="fp8")]
    assert st.attention_launches(0) == 1
    assert st.attention_launches(1) == 2


def test_reference_arm_reports_what_it_timed(monkeypatch):
    """The reference arm (the oracle on the host cores) on a small stream:
    rank 0 alone prints; ms_per_step is the mean of the timed samples, value
    is the latent frames those samples amount to per second, and the
    whole-frame figure is kept apart as an extrapolation."""
    small = W.replace(W.STREAM, grid_h=4, grid_w=6, H=2, D=64, pairs=(12, 10, 10), layers=3)
    monkeypatch.setattr(bench.W, "STREAM", small)
    monkeypatch.setattr(bench, "STEP_TARGET_S", 0.01)
    timed = []
    orig = bench.OracleStep.time

    def record(self, rows):
        t = orig(self, rows)
        timed.append((rows, t))
        return t

    monkeypatch.setattr(bench.OracleStep, "time", record)
    args = types.SimpleNamespace(steps=3, warmup=2)
    assert bench.run_reference(args, 1, 2) is None
    assert timed == []
    line = bench.run_reference(args, 0, 1)
    rows = timed[-1][0]
    assert rows == small.N == 24                         # a frame of fewer than 64 rows: all of them
    samples = [t for _, t in timed[-3:]]
    assert len(timed) == 2 + 2 + 3                       # two probes, warm-up, timed steps
    assert abs(line["ms_per_step"] - sum(samples) / 3 * 1e3) <= 1e-3
    frames = rows / small.N / small.layers
    assert abs(line["value"] - frames / (sum(samples) / 3)) <= 1e-6 * max(1.0, line["value"])
    assert line["impl"] == "reference" and line["higher_is_better"] is True and line["dtype"] == "f64"
    assert line["steps"] == 3 and line["warmup"] == 2 and line["n_gpus"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert "not a measurement" in line["extrapolated"]["note"]


def test_cpu_baseline_repeats_the_sample_to_its_time_budget(monkeypatch):
    """Our arm's cpu_baseline repeats the oracle sample until the budget is
    spent and reports the frames of all samples over their summed time."""
    small = W.replace(W.STREAM, grid_h=4, grid_w=6, H=2, D=64, pairs=(12, 10, 10), layers=3)
    monkeypatch.setattr(bench, "STEP_TARGET_S", 0.01)
    monkeypatch.setattr(bench, "BASELINE_TARGET_S", 0.05)
    timed = []
    orig = bench.OracleStep.time

    def record(self, rows):
        t = orig(self, rows)
        timed.append(t)
        return t

    monkeypatch.setattr(bench.OracleStep, "time", record)
    cb = bench.cpu_baseline(small)
    samples = timed[2:]                                   # after the two probes
    assert 1 <= len(samples) <= bench.BASELINE_MAX_SAMPLES
    assert sum(samples) >= 0.05 or len(samples) == bench.BASELINE_MAX_SAMPLES
    frames = len(samples) * small.N / small.N / small.layers
    assert abs(cb["value"] - frames / sum(samples)) <= 1e-6 + 1e-6 * cb["value"]
    assert cb["kind"] == "oracle" and cb["sample"].startswith(f"{len(samples)} consecutive samples")
