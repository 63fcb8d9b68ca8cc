"""Full-size parity of the long-context decode sweep: batch 64, s_q 1, every sequence's cache 1K, 2K, ... 64K
tokens, over the GQA layout (32 query / 8 KV heads, d_h 128) and the GQLA latent layout on the MQA-absorbed path
(128 heads, 512 + 64 latent values).  Each point runs the bench's own inputs through the public entry point with
its automatic split plan; the fp64 oracle checks a sample of sequences (first, last, and one in the middle), with
the lse for GQA (marked gpu)."""
import pytest
import torch

import latent_kv_attention_b200 as lka
import oracle
import synthetic
from parity import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
ROWS = [0, 37, 63]


@pytest.fixture(autouse=True)
def _clean_status():
    lka.clear_status()
    yield
    assert lka.device_status() == 0, lka.status_string(lka.device_status())
    torch.cuda.empty_cache()


def _sub(inp, keys):
    return {k: inp[k][ROWS].cpu() for k in keys}


@pytest.mark.parametrize("L", synthetic.SWEEP_LENGTHS)
def test_gqa_sweep_point(L):
    name = f"gqa_sweep_{L // 1024}k"
    inp = synthetic.make(synthetic.SWEEP[name], device=DEV)
    out, lse = lka.gqa_attn(inp["q"], inp["k"], inp["v"], inp["cache_lens"], causal=True, scale=inp["scale"],
                            return_lse=True)
    s, scale = _sub(inp, ("q", "k", "v", "cache_lens")), inp["scale"]
    del inp
    ref, ref_lse = oracle.gqa(s["q"], s["k"], s["v"], s["cache_lens"], True, scale)
    assert_close(out[ROWS], ref, torch.bfloat16, name)
    assert_lse_close(lse[ROWS], ref_lse, torch.bfloat16, f"{name} lse")


@pytest.mark.parametrize("L", synthetic.SWEEP_LENGTHS)
def test_latent_sweep_point(L):
    name = f"latent_sweep_{L // 1024}k"
    inp = synthetic.make(synthetic.SWEEP[name], device=DEV)
    out = lka.latent_absorbed_attn(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                   inp["cache_lens"], causal=True, scale=inp["scale"])
    s = _sub(inp, ("q_c", "q_r", "latent", "cache_lens"))
    w_uk, w_uv, scale = inp["w_uk"].cpu(), inp["w_uv"].cpu(), inp["scale"]
    del inp
    ref, _ = oracle.latent_absorbed(s["q_c"], s["q_r"], w_uk, w_uv, s["latent"], s["cache_lens"], True, scale)
    assert_close(out[ROWS], ref, torch.bfloat16, name)
