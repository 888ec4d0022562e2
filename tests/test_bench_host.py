"""Host-side arithmetic of the benchmark (no GPU): the algorithmic bytes of
the whole pass, the roofline of the dominant stage, and the ncu traffic
record, which is reported only while its kernel source is unchanged."""
import dataclasses
import hashlib
import importlib.util
import os

import pytest

from frame_wise_delta_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_whole_pass_bytes_at_h3(bench):
    w = synth.WORKLOADS["h3"]
    qkvo = 4 * 24 * 102 * 1008 * 128 * 2  # Q, K, V read and O written, bf16
    text = 2 * 24 * 512 * 128 * 2
    gates = 24 * (102 * (128 + 1) + 1) * 4  # alpha per channel, beta per frame, beta_x
    assert bench.alg_bytes(w) == qkvo + text + gates
    assert abs(bench.alg_bytes(w) / 1e9 - 2.53) < 0.01
    # the gated epilogue adds the gate logits (input dtype) and the RMSNorm weights
    assert bench.alg_bytes(w, gated=True) - bench.alg_bytes(w) == 24 * 102 * 1008 * 128 * 2 + 24 * 128 * 4


def test_roofline_of_the_dominant_stage(bench):
    w = synth.WORKLOADS["h3"]
    stage_ms = {"text_state": 0.15, "frame_grams": 0.25, "frame_factor": 0.14, "chunk_compose": 0.12,
                "scan_bidir": 0.05, "chunk_readout": 0.22}
    r = bench.roofline(w, stage_ms, 6531.9, "measured")
    assert r["kernel"] == "frame_grams" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    frames = 24 * 102
    # algorithmic bytes of the Gram stage: K and V read once (bf16), nothing else
    kv = frames * 2 * 1008 * 128 * 2
    assert r["algorithmic_bytes"] == kv
    assert r["achieved"] == pytest.approx(kv / 0.25e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6531.9)
    # what the kernel writes beyond that is reported beside it, not counted in it
    assert r["intermediate_bytes"] == frames * (128 * 128 * 4 + 3 * 64 * 64 * 4 + 36 * 64 * 4)
    # the traffic record is reported while its kernel source is the one it was taken on
    rec = bench.NCU_TRAFFIC["frame_grams"]
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        same = hashlib.sha256(f.read()).hexdigest()[:16] == rec["sha256_16"]
    assert r["traffic"] == (rec["bytes"] if same else None)
    if same:
        assert r["traffic_over_algorithmic"] == pytest.approx(rec["bytes"] / kv)
    # another workload name: no recorded traffic
    w2 = dataclasses.replace(w, name="h3_other")
    assert bench.roofline(w2, stage_ms, 6531.9, "measured")["traffic"] is None


def test_readout_roofline_counts_q_and_o(bench):
    w = synth.WORKLOADS["h3"]
    stage_ms = {"frame_grams": 0.20, "frame_factor": 0.14, "chunk_compose": 0.12, "scan_bidir": 0.05,
                "chunk_readout": 0.22}
    r = bench.roofline(w, stage_ms, 6531.9, "measured")
    assert r["kernel"] == "chunk_readout"
    qo = 24 * 102 * 2 * 1008 * 128 * 2
    assert r["algorithmic_bytes"] == qo
    assert r["achieved"] == pytest.approx(qo / 0.22e-3 / 1e9)
    # the boundary states it reads are intermediate bytes
    assert r["intermediate_bytes"] == 24 * 21 * 2 * 128 * 128 * 4


def test_whole_pass_roofline(bench):
    w = synth.WORKLOADS["h3"]
    r = bench.whole_pass_roofline(w, 0.8, 1, 6531.9, "measured")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(bench.alg_bytes(w) / 0.8e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6531.9)
    # two ranks, each with its own problem: the same fraction per GPU, twice the job's bytes
    r2 = bench.whole_pass_roofline(w, 0.8, 2, 6531.9, "measured")
    assert r2["frac"] == pytest.approx(r["frac"]) and r2["job_bytes"] == 2 * r["algorithmic_bytes"]


def test_reference_arm_times_only_the_oracle(bench, monkeypatch):
    """The reference arm draws its inputs before the warm-up: no input is
    generated between the start and the end of its timed steps."""
    import oracle

    w = dataclasses.replace(synth.WORKLOADS["tiny"], H=6)
    events = []
    real_gen = synth.generate_head
    monkeypatch.setattr(synth, "generate_head", lambda *a, **k: (events.append("gen"), real_gen(*a, **k))[1])
    real_head = oracle.vda_head
    monkeypatch.setattr(oracle, "vda_head", lambda *a, **k: (events.append("oracle"), real_head(*a, **k))[1])
    real_pc = bench.time.perf_counter
    monkeypatch.setattr(bench.time, "perf_counter", lambda: (events.append("clock"), real_pc())[1])
    args = type("A", (), {"warmup": 2, "steps": 5, "gpus": 1})()
    monkeypatch.setenv("RANK", "0")
    bench.run_reference(args, w)
    timed = events[events.index("clock"):len(events) - events[::-1].index("clock")]
    assert "gen" not in timed
    assert timed.count("oracle") == 5


def test_traffic_records_name_existing_sources(bench):
    for rec in bench.NCU_TRAFFIC.values():
        assert os.path.exists(os.path.join(ROOT, rec["source"]))
        assert len(rec["sha256_16"]) == 16


def test_clock_summary_keeps_the_timed_window(bench):
    import datetime

    clk = bench.ClockSampler(0)
    base = datetime.datetime(2026, 12, 2, 10, 0, 0).timestamp()

    def line(dt, mhz, cap="Not Active"):
        ts = datetime.datetime.fromtimestamp(base + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, 0, {mhz}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {cap}"

    # idle samples before and after the window are ignored; the window's median is reported
    clk.lines = [line(0.0, 300), line(0.10, 1965), line(0.15, 1950), line(0.20, 1965, "Active"), line(0.40, 300)]
    clk.t0, clk.t1 = base + 0.05, base + 0.25
    s = clk.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]
    # a window shorter than the period: the sample nearest its middle
    clk.t0, clk.t1 = base + 0.39, base + 0.395
    s = clk.summary()
    assert s["samples"] == 1 and s["sm_mhz"] == 300
