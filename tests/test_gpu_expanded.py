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
