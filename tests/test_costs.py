"""Closed forms the pages print, checked against the byte/FLOP counters the roofline uses (CPU only)."""
import json
import os

import pytest

from latent_kv_attention_b200 import costs

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def test_glossary_cached_values_per_token():
    gd = golden("gqa_glossary_example.json")
    assert costs.cache_elems_per_token("gqa", kv_heads=2, d=64) == gd["printed_cached_values_per_token_gqa"]
    assert costs.cache_elems_per_token("mha", kv_heads=8, d=64) == gd["printed_cached_values_per_token_mha"]


def test_llama31_8b_kv_cache_sizes():
    gd = golden("kv_cache_sizes.json")
    per_layer = costs.cache_elems_per_token("gqa", kv_heads=gd["kv_heads"], d=gd["head_dim"])
    per_token = gd["layers"] * per_layer * gd["bytes_per_value"]
    assert per_token == gd["per_token_bytes_gqa"] == 128 * 1024
    assert per_token * gd["context_tokens"] == gd["full_context_bytes_gqa"] == 16 * 2**30
    mha = gd["layers"] * costs.cache_elems_per_token("mha", kv_heads=gd["query_heads"], d=gd["head_dim"]) * 2
    assert mha == gd["per_token_bytes_mha"] and mha * gd["context_tokens"] == gd["full_context_bytes_mha"]


def test_gqla_cache_and_intensity_closed_forms():
    gd = golden("gqla_closed_forms.json")
    c = gd["config"]
    lat = costs.cache_elems_per_token("latent", r_kv=c["r_kv"], d_r=c["d_r"])
    exp = costs.cache_elems_per_token("expanded", g=c["g"], d_h=c["d_h"], d_r=c["d_r"])
    assert lat == gd["absorbed_cache_elems_per_token"] and exp == gd["gqa_path_cache_elems_per_token"]
    assert lat / gd["llama3_8b_gqa_cache_elems_per_token"] == gd["absorbed_vs_llama3_8b_gqa_fraction"]
    ai = costs.arithmetic_intensity_per_token(c["h_q"], c["r_kv"] + c["d_r"], c["r_kv"], lat, s_q=1)
    assert ai == pytest.approx(gd["absorbed_sq1_intensity_flops_per_byte_approx"], abs=0.5)
    assert ai < gd["h100_bf16_ridge_flops_per_byte"]  # "just below the H100 ridge"
    ai2 = costs.arithmetic_intensity_per_token(c["h_q"], c["d_h"] + c["d_r"], c["d_h"], exp, s_q=2)
    assert ai2 == pytest.approx(gd["h20_ridge_flops_per_byte_approx"], rel=0.06)
    assert c["h_q"] // c["g"] == gd["recommended_heads_per_group"]


def test_counters_match_per_token_forms():
    lens = [5, 9]
    assert costs.latent_core_flops(lens, 128, 512, 64, 1, True) == 14 * 128 * (2 * 576 + 2 * 512)
    assert costs.gqa_flops([4], 8, 64, 4, True) == (1 + 2 + 3 + 4) * 8 * 4 * 64
    assert costs.gta_flops([3], 3, 12, 64, 64, 3, True) == 6 * (3 * 128 + 12 * 128)
    assert costs.gqa_bytes([10], 32, 8, 128, 1) == 10 * 8 * 256 * 2 + 32 * 128 * 2 * 2


def test_long_context_sweep_points():
    # batch 64, s_q 1, equal cache lengths 1K ... 64K: GQA (32 / 8 heads, d_h 128) reads 64 * L * 4096 cache
    # bytes, the latent layout 64 * L * 1152 bytes and does 64 * L * 128 * (2 * 576 + 2 * 512) FLOPs
    import synthetic

    assert synthetic.SWEEP_LENGTHS == tuple(1024 * 2 ** i for i in range(7))
    for L in synthetic.SWEEP_LENGTHS:
        g = synthetic.SWEEP[f"gqa_sweep_{L // 1024}k"]
        lat = synthetic.SWEEP[f"latent_sweep_{L // 1024}k"]
        assert (g["B"], g["h_q"], g["h_kv"], g["d"], g["s_q"], g["L_lo"], g["L_hi"]) == (64, 32, 8, 128, 1, L, L)
        assert (lat["B"], lat["h_q"], lat["r_kv"], lat["d_r"], lat["s_q"], lat["L_hi"]) == (64, 128, 512, 64, 1, L)
        lens = [L] * 64
        assert costs.gqa_bytes(lens, 32, 8, 128, 1) == 64 * L * 4096 + 64 * 32 * 128 * 2 * 2
        assert costs.latent_core_flops(lens, 128, 512, 64, 1, True) == 64 * L * 278528
    assert costs.gqa_bytes([65536] * 64, 32, 8, 128, 1) / 1e9 == pytest.approx(17.18, abs=0.01)
