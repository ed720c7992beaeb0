"""Host-side arithmetic of bench.py on the CPU: the algorithmic bytes and FLOPs
behind the roofline fractions, the roofline record, and the digest check that
keeps a stale ncu traffic figure out of the JSON line."""

import json
import os
import shutil

import numpy as np
import pytest

import bench

# Gemma-4-26B-A4B (model card / TransformerConfig): embed 2816, expert width
# 704, shared MLP width 2112, 128 experts, top-8.
D, F, S, E, K = 2816, 704, 2112, 128, 8


def test_model_dims():
    assert (bench.D, bench.F, bench.S, bench.E, bench.K_TOP) == (D, F, S, E, K)


def test_decode_gateup_bytes_are_the_touched_weights_plus_activations():
    """T=64 with 126 touched experts: the gate and up matrices of those experts
    (bf16), the shared MLP's two, the routed and token rows in, h and hs out."""
    T, touched = 64, 126
    byts, flops = bench.algorithmic("grouped_gemm_gateup", T, touched, None)
    weights = touched * 2 * (D * F * 2) + 2 * (D * S * 2)
    acts = (T * K) * D * 2 + T * D * 2 + (T * K) * F * 2 + T * S * 2
    assert byts == weights + acts == 1_027_186_688
    # two projections, one multiply-add (2 FLOP) per weight per routed row / token
    assert flops == 2 * (T * K) * (2 * D * F) + 2 * T * (2 * D * S)


def test_down_bytes_and_flops():
    T, touched = 4096, 128
    byts, flops = bench.algorithmic("grouped_gemm_down", T, touched, None)
    assert byts == touched * F * D * 2 + S * D * 2 + T * K * F * 2 + T * S * 2 + T * K * D * 2 + T * D * 4
    assert flops == 2 * T * K * F * D + 2 * T * S * D


def test_flop_per_token_matches_the_three_projections():
    # gate, up and down of 8 experts and of the shared MLP, plus the router
    assert bench.FLOP_PER_TOKEN_GEMM == K * 3 * 2 * D * F + 3 * 2 * D * S
    assert bench.FLOP_PER_TOKEN == bench.FLOP_PER_TOKEN_GEMM + 2 * D * E


def _fake_result(kernel, dom_ms, step_ms, T, touched):
    return {"dominant": kernel, "dom_ms": dom_ms, "touched": touched, "cnt": None,
            "agg": {"ms_per_step": step_ms}}


PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0, "source": "test"}


def test_roofline_hbm_fraction():
    res = _fake_result("grouped_gemm_gateup", 0.2, 0.3, 64, 126)
    roof, block = bench.roofline_of(res, 64, "hbm", PEAKS, ms_total=0.3 * 20)
    byts, _ = bench.algorithmic("grouped_gemm_gateup", 64, 126, None)
    assert roof["achieved"] == pytest.approx(byts / 0.2e-3 / 1e9)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6000.0)
    assert roof["unit"] == "GB/s" and roof["traffic"] is None
    w = 126 * bench.BYTES_PER_EXPERT + bench.SHARED_BYTES + bench.ROUTER_BYTES
    assert block["hbm_frac"] == pytest.approx(w / 0.3e-3 / 1e9 / 6000.0)


def test_roofline_tensor_peak_burst_or_sustained():
    res = _fake_result("grouped_gemm_gateup", 0.35, 0.7, 4096, 128)
    short, _ = bench.roofline_of(res, 4096, "tensor", PEAKS, ms_total=0.7 * 100)
    long_, _ = bench.roofline_of(res, 4096, "tensor", PEAKS, ms_total=0.7 * 5000)
    assert short["peak"] == 1500.0 and long_["peak"] == 1400.0  # a timed region over 2 s: sustained
    _, flops = bench.algorithmic("grouped_gemm_gateup", 4096, 128, None)
    assert short["achieved"] == pytest.approx(flops / 0.35e-3 / 1e12)


def test_traffic_entries_are_well_formed():
    with open(os.path.join(bench.ROOT, "profiles", "dram_traffic.json")) as f:
        table = json.load(f)
    csrc = os.path.join(bench.ROOT, "mixture_experts_transformer_b200", "csrc")
    for key, ent in table.items():
        kernel, _, workload = key.partition("@")
        assert kernel and workload, key
        assert ent["bytes_per_launch"] > 0, key
        assert os.path.exists(os.path.join(bench.ROOT, ent["source"])), key
        for f in ent["files"]:
            assert os.path.exists(os.path.join(csrc, f)), (key, f)
        assert len(ent["digest"]) == 16


def test_stale_traffic_is_dropped(tmp_path, monkeypatch):
    """A traffic figure whose kernel sources changed since its capture is not
    reported."""
    root = tmp_path / "repo"
    csrc = root / "mixture_experts_transformer_b200" / "csrc"
    csrc.mkdir(parents=True)
    (root / "profiles").mkdir()
    (csrc / "k.cuh").write_text("kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    ent = {"bytes_per_launch": 123.0, "source": "profiles/x.md", "files": ["k.cuh"],
           "digest": bench.source_digest(["k.cuh"])}
    (root / "profiles" / "dram_traffic.json").write_text(json.dumps({"kern@wl": ent}))
    assert bench.ncu_traffic("kern", "wl") == 123.0
    assert bench.ncu_traffic("kern", "other") is None
    (csrc / "k.cuh").write_text("kernel v2\n")
    assert bench.ncu_traffic("kern", "wl") is None
