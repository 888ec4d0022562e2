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
    per_frame = 2 * 1008 * 128 * 2 + 128 * 128 * 4 // 2 + 128 * 128 * 4 + 16384
    assert r["achieved"] == pytest.approx(frames * per_frame / 0.25e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6531.9)
    # the traffic record is reported while its kernel source is the one it was taken on
    rec = bench.NCU_TRAFFIC["frame_grams"]
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        same = hashlib.sha256(f.read()).hexdigest()[:16] == rec["sha256_16"]
    assert r["traffic"] == (rec["bytes"] if same else None)
    # another workload name: no recorded traffic
    w2 = dataclasses.replace(w, name="h3_other")
    assert bench.roofline(w2, stage_ms, 6531.9, "measured")["traffic"] is None


def test_traffic_records_name_existing_sources(bench):
    for rec in bench.NCU_TRAFFIC.values():
        assert os.path.exists(os.path.join(ROOT, rec["source"]))
        assert len(rec["sha256_16"]) == 16
