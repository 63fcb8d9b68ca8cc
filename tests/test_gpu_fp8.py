"""GPU parity of the e4m3-cache entry points (gqa_attn_fp8kv, latent_absorbed_attn_fp8kv) against the fp64 oracle
(marked gpu)."""
import pytest
import torch

import latent_kv_attention_b200 as lka
import oracle
import synthetic
from parity import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _clean_status():
    lka.clear_status()
    yield
    assert lka.device_status() == 0, lka.status_string(lka.device_status())


CASES = [
    # (B, h_q, h_kv, d, s_q, L_lo, L_hi, Lmax, causal)
    (3, 32, 8, 128, 1, 1, 900, 1024, True),    # Llama-3.1-8B heads, ragged, L=1 possible
    (2, 8, 2, 128, 1, 100, 700, 768, False),   # 4 heads per group, no mask
    (2, 32, 8, 128, 2, 2, 600, 640, True),     # MTP: 8 rows per group in two row blocks
    (2, 8, 8, 128, 1, 60, 130, 130, True),     # MHA
    (2, 16, 2, 256, 1, 50, 400, 512, True),    # d=256, 8 heads per group
    (1, 16, 1, 128, 3, 3, 70, 80, True),       # MQA, s_q=3
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}sq{c[4]}" for c in CASES])
def test_fp8kv(case):
    B, h_q, h_kv, d, s_q, lo, hi, Lmax, causal = case
    inp = synthetic.gqa_fp8_inputs(700 + B * h_q + d + s_q, B, h_q, h_kv, d, s_q, lo, hi, Lmax=Lmax)
    dd = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse = lka.gqa_attn_fp8kv(dd["q"], dd["k"], dd["v"], dd["k_scale"], dd["v_scale"], dd["cache_lens"],
                                  causal=causal, scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle.gqa_fp8kv(inp["q"], inp["k"], inp["v"], inp["k_scale"], inp["v_scale"], inp["cache_lens"],
                                    causal, inp["scale"])
    assert_close(out, ref, torch.bfloat16, "fp8kv out")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "fp8kv lse")


def test_fp8kv_matches_bf16_path_on_the_dequantised_cache():
    """The same attention through gqa_attn on the dequantised cache (rounded to bf16) agrees within bf16 noise."""
    inp = synthetic.gqa_fp8_inputs(790, 4, 32, 8, 128, 1, 500, 2000, Lmax=2048)
    dd = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    a = lka.gqa_attn_fp8kv(dd["q"], dd["k"], dd["v"], dd["k_scale"], dd["v_scale"], dd["cache_lens"],
                           scale=inp["scale"])
    k16 = (dd["k"].float() * dd["k_scale"][None, :, None, None]).to(torch.bfloat16)
    v16 = (dd["v"].float() * dd["v_scale"][None, :, None, None]).to(torch.bfloat16)
    b = lka.gqa_attn(dd["q"], k16, v16, dd["cache_lens"], scale=inp["scale"])
    assert (a.float() - b.float()).abs().max().item() <= 2e-2


@pytest.mark.parametrize("split_tokens", [64, 192, 0], ids=["one_tile_items", "uneven_items", "auto"])
@pytest.mark.parametrize("s_q,causal", [(1, True), (2, True), (1, False), (3, False), (4, True)])
def test_fp8kv_split_sizes_are_repeatable(split_tokens, s_q, causal):
    """The e4m3 tensor-core kernels under forced split sizes (s_q <= 2: the 8-row form, 4 or 8 rows per KV head;
    s_q 3, 4: the 16-row form, 12 or 16 rows): one-tile splits, splits that end mid-tile, empty last splits of
    short sequences; three calls in a row give the same bytes, and the first matches the oracle."""
    inp = synthetic.gqa_fp8_inputs(811 + s_q + split_tokens, 6, 32, 8, 128, s_q, s_q, 3000, Lmax=3072)
    dd = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    prev = lka.set_split_tokens(split_tokens)
    try:
        outs = [lka.gqa_attn_fp8kv(dd["q"], dd["k"], dd["v"], dd["k_scale"], dd["v_scale"], dd["cache_lens"],
                                   causal=causal, scale=inp["scale"], return_lse=True) for _ in range(3)]
    finally:
        lka.set_split_tokens(prev)
    ref, ref_lse = oracle.gqa_fp8kv(inp["q"], inp["k"], inp["v"], inp["k_scale"], inp["v_scale"], inp["cache_lens"],
                                    causal, inp["scale"])
    assert_close(outs[0][0], ref, torch.bfloat16, "fp8kv split out")
    assert_lse_close(outs[0][1], ref_lse, torch.bfloat16, "fp8kv split lse")
    for o, l in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(l, outs[0][1])


# ------------------------------------------------------------------ FP8 latent cache (MQA-absorbed path) -----
LATENT_CASES = [
    # (B, s_q, L_lo, L_hi, Lmax, causal)
    (2, 1, 1, 700, 768, True),      # ragged, L = 1 possible, several tiles and a ragged tail
    (3, 2, 2, 500, 520, True),      # MTP, bottom-right causal
    (2, 1, 60, 130, 130, False),    # no mask
]


@pytest.mark.parametrize("case", LATENT_CASES, ids=[f"B{c[0]}sq{c[1]}L{c[3]}" for c in LATENT_CASES])
def test_latent_fp8kv(case):
    B, s_q, lo, hi, Lmax, causal = case
    inp = synthetic.latent_fp8_inputs(810 + B * 7 + s_q, B, 128, 8, 128, 512, 64, s_q, lo, hi, Lmax=Lmax)
    dd = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse = lka.latent_absorbed_attn_fp8kv(dd["q_c"], dd["q_r"], dd["w_uk"], dd["w_uv"], dd["latent8"],
                                              dd["kv_scale"], dd["cache_lens"], causal=causal, scale=inp["scale"],
                                              return_lse=True)
    ref, ref_lse = oracle.latent_absorbed_fp8kv(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent8"],
                                                inp["kv_scale"], inp["cache_lens"], causal, inp["scale"])
    assert_close(out, ref, torch.bfloat16, "latent fp8kv out")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "latent fp8kv lse")


def test_latent_fp8kv_forced_splits_and_bf16_agreement():
    """Key splits (merged partials) give the same result within tolerance, and the bf16 path over the dequantised
    cache (rounded to bf16, exact for these values) agrees within bf16 noise."""
    inp = synthetic.latent_fp8_inputs(850, 2, 128, 8, 128, 512, 64, 1, 300, 900, Lmax=960)
    dd = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    a = lka.latent_absorbed_attn_fp8kv(dd["q_c"], dd["q_r"], dd["w_uk"], dd["w_uv"], dd["latent8"], dd["kv_scale"],
                                       dd["cache_lens"], scale=inp["scale"])
    prev = lka.set_split_tokens(128)
    try:
        b = lka.latent_absorbed_attn_fp8kv(dd["q_c"], dd["q_r"], dd["w_uk"], dd["w_uv"], dd["latent8"],
                                           dd["kv_scale"], dd["cache_lens"], scale=inp["scale"])
    finally:
        lka.set_split_tokens(prev)
    ref, _ = oracle.latent_absorbed_fp8kv(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent8"],
                                          inp["kv_scale"], inp["cache_lens"], True, inp["scale"])
    assert_close(b, ref, torch.bfloat16, "latent fp8kv split")
    lat = dd["latent8"].to(torch.float32)
    lat[..., :512] *= dd["kv_scale"][0]
    lat[..., 512:] *= dd["kv_scale"][1]
    c = lka.latent_absorbed_attn(dd["q_c"], dd["q_r"], dd["w_uk"], dd["w_uv"], lat.to(torch.bfloat16),
                                 dd["cache_lens"], scale=inp["scale"])
    assert (a.float() - c.float()).abs().max().item() <= 2e-2
    assert (a.float() - b.float()).abs().max().item() <= 2e-2


def test_latent_fp8kv_rejects_bad_arguments():
    inp = synthetic.latent_fp8_inputs(860, 1, 128, 8, 128, 512, 64, 1, 10, 20)
    dd = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    with pytest.raises(Exception):
        lka.latent_absorbed_attn_fp8kv(dd["q_c"], dd["q_r"], dd["w_uk"], dd["w_uv"], dd["latent8"],
                                       dd["kv_scale"][:1], dd["cache_lens"])
    with pytest.raises(Exception):  # a bf16 cache is not an e4m3 cache
        lka.latent_absorbed_attn_fp8kv(dd["q_c"], dd["q_r"], dd["w_uk"], dd["w_uv"],
                                       dd["latent8"].to(torch.bfloat16), dd["kv_scale"], dd["cache_lens"])
