"""GPU parity of the GQLA per-group GQA path (latent_expand_gqa_attn) against the fp64 oracle (marked gpu)."""
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


def oracle_expanded(inp, causal):
    """GQA over key [kc ; kr] (RoPE key shared by the groups) and value vc: the oracle's GQA routine with the
    value zero-padded to the key width (the padding columns of the result are dropped)."""
    kc, vc, kr = inp["kc"].double(), inp["vc"].double(), inp["kr"].double()
    key = torch.cat([kc, kr[:, None].expand(-1, kc.shape[1], -1, -1)], -1)
    val = torch.cat([vc, torch.zeros_like(kr[:, None].expand(-1, kc.shape[1], -1, -1))], -1)
    q = torch.cat([inp["q_c"].double(), inp["q_r"].double()], -1)
    out, lse = oracle.gqa(q, key, val, inp["cache_lens"], causal, inp["scale"])
    return out[..., :kc.shape[-1]], lse


@pytest.mark.parametrize("s_q", [1, 2])
@pytest.mark.parametrize("causal", [True, False])
def test_expanded_random(s_q, causal):
    inp = synthetic.expanded_inputs(51, 3, 128, 8, 128, 64, s_q, 2, 333, Lmax=340)
    d = dev(inp)
    out, lse = lka.latent_expand_gqa_attn(d["q_c"], d["q_r"], d["kc"], d["vc"], d["kr"], d["cache_lens"],
                                          causal=causal, scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle_expanded(inp, causal)
    assert_close(out, ref, torch.bfloat16, "expanded")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "expanded lse")


@pytest.mark.parametrize("split", [128, 384])
def test_expanded_forced_splits(split):
    inp = synthetic.expanded_inputs(52, 2, 64, 4, 128, 64, 2, 300, 1000, Lmax=1000)
    d = dev(inp)
    prev = lka.set_split_tokens(split)
    try:
        out = lka.latent_expand_gqa_attn(d["q_c"], d["q_r"], d["kc"], d["vc"], d["kr"], d["cache_lens"],
                                         causal=True, scale=inp["scale"])
    finally:
        lka.set_split_tokens(prev)
    ref, _ = oracle_expanded(inp, True)
    assert_close(out, ref, torch.bfloat16, "expanded split")


@pytest.mark.parametrize("s_q", [1, 2])
def test_absorbed_equals_expanded_on_gpu(s_q):
    """GQLA sec. 3.1: both decode paths give the same output. The expanded cache is made on the GPU from the
    latent; each path is checked against the oracle's latent definition and against each other."""
    inp = synthetic.latent_inputs(53, 2, 128, 8, 128, 512, 64, s_q, 50, 400, Lmax=400)
    d = dev(inp)
    kc, vc, kr = lka.latent_expand_cache(d["latent"], d["w_uk"], d["w_uv"])
    a = lka.latent_absorbed_attn(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"], d["latent"], d["cache_lens"],
                                 causal=True, scale=inp["scale"])
    e = lka.latent_expand_gqa_attn(d["q_c"], d["q_r"], kc, vc, kr, d["cache_lens"], causal=True, scale=inp["scale"])
    ref, _ = oracle.latent_expanded(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                    inp["cache_lens"], True, inp["scale"])
    assert_close(a, ref, torch.bfloat16, "absorbed")
    assert_close(e, ref, torch.bfloat16, "expanded (GPU-expanded cache)")
    assert_close(a, e.double().cpu().numpy(), torch.bfloat16, "absorbed vs expanded")


def test_expanded_full_size_sampled():
    w = synthetic.WORKLOADS["latent_decode_4k_sq2"]
    inp = synthetic.make(w, device=DEV)
    kc, vc, kr = lka.latent_expand_cache(inp["latent"], inp["w_uk"], inp["w_uv"])
    out = lka.latent_expand_gqa_attn(inp["q_c"], inp["q_r"], kc, vc, kr, inp["cache_lens"], causal=True,
                                     scale=inp["scale"])
    rows = [0, 17, 63]
    ref, _ = oracle.latent_absorbed(inp["q_c"][rows].cpu(), inp["q_r"][rows].cpu(), inp["w_uk"].cpu(),
                                    inp["w_uv"].cpu(), inp["latent"][rows].cpu(), inp["cache_lens"][rows].cpu(),
                                    True, inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "expanded full-size sample")


# ---- prefill (s_q >= 64): the per-group path on the tcgen05 prefill kernel, any h_q / g ----
# GQLA section 1: during prefill the per-group (MHA-like) form is the compute-efficient one; query t of s_q over a
# cache of L_b tokens sees keys 0 .. L_b - s_q + t (bottom-right causal), keys [kc[gamma] ; k^R] of 192 values.
PREFILL_CASES = [
    # (B, h_q, g, s_q, L_lo, L_hi, Lmax, causal)
    (2, 16, 2, 130, 130, 130, 130, True),    # pure prefill, two query tiles with a ragged tail
    (2, 8, 2, 200, 300, 650, 660, True),     # chunked prefill over a cached prefix, ragged lengths
    (1, 8, 8, 64, 64, 200, 200, False),      # one head per group (plain MHA with a shared RoPE key)
    (2, 32, 2, 96, 96, 300, 300, True),      # 16 query heads per group, as in the decode configuration
    (1, 128, 8, 128, 128, 128, 128, True),   # the 128-head, 8-group layer
]


@pytest.mark.parametrize("case", PREFILL_CASES)
def test_expanded_prefill_matches_oracle(case):
    B, h_q, g, s_q, lo, hi, Lmax, causal = case
    inp = synthetic.expanded_inputs(61, B, h_q, g, 128, 64, s_q, lo, hi, Lmax=Lmax)
    d = dev(inp)
    out, lse = lka.latent_expand_gqa_attn(d["q_c"], d["q_r"], d["kc"], d["vc"], d["kr"], d["cache_lens"],
                                          causal=causal, scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle_expanded(inp, causal)
    assert_close(out, ref, torch.bfloat16, "expanded prefill")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "expanded prefill lse")


@pytest.mark.parametrize("split", [128, 256])
def test_expanded_prefill_key_splits(split):
    inp = synthetic.expanded_inputs(62, 1, 16, 2, 128, 64, 150, 400, 900, Lmax=900)
    d = dev(inp)
    prev = lka.set_split_tokens(split)
    try:
        out = lka.latent_expand_gqa_attn(d["q_c"], d["q_r"], d["kc"], d["vc"], d["kr"], d["cache_lens"],
                                         causal=True, scale=inp["scale"])
    finally:
        lka.set_split_tokens(prev)
    ref, _ = oracle_expanded(inp, True)
    assert_close(out, ref, torch.bfloat16, f"expanded prefill, splits of {split}")


@pytest.mark.parametrize("page_size", [16, 128])
def test_expanded_prefill_paged(page_size):
    inp = synthetic.expanded_paged_inputs(63, 2, 16, 2, 128, 64, 100, 100, 350, page_size, Lmax=400)
    d = dev(inp)
    out = lka.latent_expand_gqa_attn_paged(d["q_c"], d["q_r"], d["kc_pages"], d["vc_pages"], d["kr_pages"],
                                           d["block_table"], d["cache_lens"], causal=True, scale=inp["scale"])
    ref, _ = oracle_expanded(inp, True)
    assert_close(out, ref, torch.bfloat16, f"expanded paged prefill, pages of {page_size}")


def test_expanded_prefill_equals_latent_definition():
    """GQLA sec. 3.1: the per-group keys and values are the up-projected latent; a prefill over a cache that
    latent_expand_cache made on the GPU matches the oracle's latent definition (eq. (1), expanded form)."""
    inp = synthetic.latent_inputs(64, 1, 32, 4, 128, 512, 64, 80, 80, 260, Lmax=260)
    d = dev(inp)
    kc, vc, kr = lka.latent_expand_cache(d["latent"], d["w_uk"], d["w_uv"])
    out = lka.latent_expand_gqa_attn(d["q_c"], d["q_r"], kc, vc, kr, d["cache_lens"], causal=True,
                                     scale=inp["scale"])
    ref, _ = oracle.latent_expanded(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                    inp["cache_lens"], True, inp["scale"])
    assert_close(out, ref, torch.bfloat16, "expanded prefill vs latent definition")
