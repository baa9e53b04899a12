"""Host arithmetic of bench.py on CPU: the algorithmic work behind every fraction it
reports, the roofline's choice of bound and its fractions, and the DRAM-traffic
lookup that must go null when a captured kernel source changes."""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_mixture_experts_12_b200 import synth  # noqa: E402

PEAKS = dict(bench.FALLBACK_PEAKS)


def _rs(rows, touched, tokens_read=None):
    rs = {"rows_kept": rows, "touched_experts": touched, "dropped": 0, "max_expert_load": 0,
          "min_expert_load": 0}
    if tokens_read is not None:
        rs["tokens_read"] = tokens_read
    return rs


def test_stage_work_mixtral_by_hand():
    wl = synth.WORKLOADS["mixtral_prefill"]
    T, d, E, k, F = wl.T, wl.d_model, wl.n_experts, wl.top_k, wl.d_ff
    R = T * k
    w = bench.stage_work(wl, _rs(R, E), want_aux=False)
    # SwiGLU: three matrices, 2 flop per multiply-add
    assert w["expert_ffn"]["flops"] == 2.0 * R * 3 * d * F
    assert w["expert_ffn"]["bytes"] == E * 3 * d * F * 2 + 2.0 * R * d * 2
    # router: x and W_r read once, (index, gate) pairs written
    assert w["route"]["bytes"] == T * d * 2 + E * d * 2 + T * k * 8
    # permute: every token read once, every kept row written, 12 B of maps per pair
    assert w["permute"]["bytes"] == T * d * 2 + R * d * 2 + T * k * 12
    # combine: kept rows read, y written, the (row, gate) pairs read
    assert w["combine"]["bytes"] == R * d * 2 + T * d * 2 + T * k * 8
    assert w["shared_ffn"]["flops"] == 0.0


def test_stage_work_switch_statistics_and_drops():
    wl = synth.WORKLOADS["switch"]
    T, d, E, F = wl.T, wl.d_model, wl.n_experts, wl.d_ff
    w = bench.stage_work(wl, _rs(1721, 26, tokens_read=1721), want_aux=True)
    # GELU MLP: two matrices; only the 26 touched experts' weights are read
    assert w["expert_ffn"]["flops"] == 2.0 * 1721 * 2 * d * F
    assert w["expert_ffn"]["bytes"] == 26 * 2 * d * F * 2 + 2.0 * 1721 * d * 2
    # the statistics need the logits as well
    assert w["route"]["bytes"] == T * d * 2 + E * d * 2 + T * 1 * 8 + T * E * 4
    # only tokens with a kept slot are read by the permute
    assert w["permute"]["bytes"] == 1721 * d * 2 + 1721 * d * 2 + T * 12


def test_stage_work_shared_experts():
    wl = synth.WORKLOADS["deepseek"]
    T, d = wl.T, wl.d_model
    Fs = wl.n_shared * wl.d_ff_shared
    w = bench.stage_work(wl, _rs(T * wl.top_k, wl.n_experts), want_aux=False)
    assert w["shared_ffn"]["flops"] == 2.0 * T * 3 * d * Fs
    assert w["combine"]["bytes"] == (T * wl.top_k * d * 2 + T * d * 2 + T * wl.top_k * 8
                                     + T * d * 4)


def test_roofline_bound_and_fractions():
    wl = synth.WORKLOADS["mixtral_prefill"]
    R = wl.T * wl.top_k
    work = bench.stage_work(wl, _rs(R, wl.n_experts), want_aux=False)
    flops = work["expert_ffn"]["flops"]
    roof = bench.ffn_roofline(wl, work, 2.0, PEAKS, "fallback")
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["achieved"] == pytest.approx(flops / 2.0e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / PEAKS["bf16_tflops"])
    assert roof["frac_of_nominal"] == pytest.approx(
        roof["achieved"] / bench.NOMINAL_PEAKS["bf16_tflops"])
    assert roof["frac_of_sustained"] == pytest.approx(
        roof["achieved"] / PEAKS["bf16_tflops_sustained"])
    # decode: arithmetic intensity far below the ridge, so the bound is HBM
    dwl = synth.WORKLOADS["decode1"]
    dwork = bench.stage_work(dwl, _rs(2, 2), want_aux=False)
    droof = bench.ffn_roofline(dwl, dwork, 0.13, PEAKS, "fallback")
    byts = dwork["expert_ffn"]["bytes"]
    assert droof["bound"] == "hbm" and droof["unit"] == "GB/s"
    assert droof["achieved"] == pytest.approx(byts / 0.13e-3 / 1e9)
    assert droof["frac"] == pytest.approx(droof["achieved"] / PEAKS["hbm_gbs"])
    assert droof["frac_of_nominal"] == pytest.approx(
        droof["achieved"] / bench.NOMINAL_PEAKS["hbm_gbs"])


def test_tokens_per_second():
    # 8 ranks, 10 steps of 4096 tokens each in 25 ms of the slowest rank
    assert bench.tokens_per_second(4096, 8, 10, 25.0) == pytest.approx(4096 * 8 * 10 / 0.025)


def test_traffic_goes_null_when_a_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// version 1\n")
    (tmp_path / "profiles").mkdir()
    entry = {"dram_bytes_per_call": 12345,
             "sources": {"kernel.cu": hashlib.sha256(src.read_bytes()).hexdigest()}}
    (tmp_path / "profiles" / "ffn_traffic.json").write_text(json.dumps({"wl": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic("wl") == 12345
    assert bench._traffic("other") is None
    src.write_text("// version 2\n")
    assert bench._traffic("wl") is None


def test_committed_traffic_lists_existing_sources():
    with open(os.path.join(ROOT, "profiles", "ffn_traffic.json")) as f:
        d = json.load(f)
    for name, ent in d.items():
        if name.startswith("_"):
            continue
        assert ent["dram_bytes_per_call"] > 0
        for rel in ent["sources"]:
            assert os.path.exists(os.path.join(ROOT, rel)), rel
