"""GPU parity of the GQLA latent paths against the fp64 oracle (marked gpu; C ABI through the binding)."""
import numpy as np
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


def dev(inp):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def absorbed_case(seed, B, s_q, L_lo, L_hi, Lmax, causal=True, g=8, rows_b=None, split=None):
    inp = synthetic.latent_inputs(seed, B, 128, g, 128, 512, 64, s_q, L_lo, L_hi, Lmax=Lmax)
    d = dev(inp)
    prev = lka.set_split_tokens(split) if split is not None else None
    try:
        out, lse = lka.latent_absorbed_attn(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"], d["latent"], d["cache_lens"],
                                            causal=causal, scale=inp["scale"], return_lse=True)
    finally:
        if split is not None:
            lka.set_split_tokens(prev)
    ref, ref_lse = oracle.latent_absorbed(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                          inp["cache_lens"], causal, inp["scale"], rows_b=rows_b)
    if rows_b is not None:
        out, lse, ref, ref_lse = out[rows_b], lse[rows_b], ref[rows_b], ref_lse[rows_b]
    assert_close(out, ref, torch.bfloat16, "latent_absorbed_attn")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "latent lse")
    return out


@pytest.mark.parametrize("s_q", [1, 2])
def test_absorbed_small_ragged(s_q):
    absorbed_case(41, 3, s_q, 2, 300, 300)


def test_absorbed_single_key_and_short():
    absorbed_case(42, 2, 1, 1, 33, 40)


def test_absorbed_noncausal_groups_of_32():
    absorbed_case(43, 2, 2, 50, 200, 256, causal=False, g=4)


@pytest.mark.parametrize("split", [64, 96, 1024])
def test_absorbed_forced_splits(split):
    absorbed_case(44, 2, 2, 100, 700, 700, split=split)


def test_absorbed_full_size_sampled():
    """GQLA/MLA decode layer at full size (B = 64, context 4096, s_q = 2); sampled sequences checked."""
    w = synthetic.WORKLOADS["latent_decode_4k_sq2"]
    inp = synthetic.make(w, device=DEV)
    out = lka.latent_absorbed_attn(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                   inp["cache_lens"], causal=True, scale=inp["scale"])
    rows = [0, 1, 31, 63]
    sub = {k: (v[rows].cpu() if isinstance(v, torch.Tensor) and k not in ("w_uk", "w_uv") else
               (v.cpu() if isinstance(v, torch.Tensor) else v)) for k, v in inp.items()}
    ref, _ = oracle.latent_absorbed(sub["q_c"], sub["q_r"], sub["w_uk"], sub["w_uv"], sub["latent"],
                                    sub["cache_lens"], True, inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "latent full-size sample")


def test_expand_cache_matches_oracle():
    inp = synthetic.latent_inputs(45, 2, 128, 8, 128, 512, 64, 1, 1, 200, Lmax=200)
    d = dev(inp)
    kc, vc, kr = lka.latent_expand_cache(d["latent"], d["w_uk"], d["w_uv"])
    rkc, rvc, rkr = oracle.latent_expand_cache(inp["latent"], inp["w_uk"], inp["w_uv"])
    assert_close(kc, rkc, torch.bfloat16, "kc")
    assert_close(vc, rvc, torch.bfloat16, "vc")
    assert np.array_equal(kr.cpu().double().numpy(), rkr)  # a copy: exact


@pytest.mark.parametrize("mul", [2, 4])
def test_absorbed_peaked_scores(mul):
    """Queries scaled up (by a power of two, exactly) make the softmax peakier and the score partials that the
    two CTAs of a cluster exchange larger; the result stays within the bf16 tolerance up to 4x the workload's
    query magnitude (beyond that the bf16 rounding of P, not the exchange, exceeds the max-abs bound)."""
    inp = synthetic.latent_inputs(47, 2, 128, 8, 128, 512, 64, 2, 500, 900, Lmax=900)
    q_c, q_r = inp["q_c"] * mul, inp["q_r"] * mul
    out = lka.latent_absorbed_attn(q_c.to(DEV), q_r.to(DEV), inp["w_uk"].to(DEV), inp["w_uv"].to(DEV),
                                   inp["latent"].to(DEV), inp["cache_lens"].to(DEV), causal=True, scale=inp["scale"])
    ref, _ = oracle.latent_absorbed(q_c, q_r, inp["w_uk"], inp["w_uv"], inp["latent"], inp["cache_lens"], True,
                                    inp["scale"])
    assert_close(out, ref, torch.bfloat16, f"latent, queries x{mul}")


def test_absorbed_exchange_beyond_fp16_range_is_reported():
    """The two CTAs of a cluster exchange their partial scores as fp16 after multiplying them by
    scale * log2(e).  Inputs whose scaled partials exceed the fp16 range (here: queries and latent x64, scale 1)
    must not turn into NaN silently: the partial is saturated, the output stays finite and the workspace status
    reports LKA_ERR_RANGE."""
    inp = synthetic.latent_inputs(48, 2, 128, 8, 128, 512, 64, 1, 200, 300, Lmax=300)
    q_c, q_r, latent = inp["q_c"] * 64, inp["q_r"] * 64, inp["latent"] * 64
    out = lka.latent_absorbed_attn(q_c.to(DEV), q_r.to(DEV), inp["w_uk"].to(DEV), inp["w_uv"].to(DEV),
                                   latent.to(DEV), inp["cache_lens"].to(DEV), causal=True, scale=1.0)
    assert lka.device_status() == 8, lka.status_string(lka.device_status())  # LKA_ERR_RANGE
    assert torch.isfinite(out).all()
    lka.clear_status()
    # ordinary magnitudes raise nothing
    absorbed_case(49, 2, 1, 200, 300, 300)
