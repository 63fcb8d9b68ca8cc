"""GPU parity of the tensor-core prefill of gqa_attn (bf16, d = 128, s_q >= 64) against the fp64 oracle.

"Grouped Query Attention (GQA)" glossary page, "How GQA works": every query head attends with the keys and
values of its KV head; the page's worked example is a causal prefill.  With s_q query tokens over a cache of
L_b tokens (the last s_q of them the queries' own), query t sees keys 0 .. L_b - s_q + t (bottom-right causal).
These shapes run on the tcgen05 prefill kernel (128-query tiles, 128-key tiles); the cases cover several tiles
with ragged tails, chunked prefill over a cached prefix, MHA / MQA groupings, key splits with their merge, paged
pools, and the Llama-3.1-8B layer at 4096 tokens (sampled query positions).
"""
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


def run_case(inp, causal, split=None):
    q, k, v, lens = (inp[n].to(DEV) for n in ("q", "k", "v", "cache_lens"))
    prev = lka.set_split_tokens(split) if split is not None else None
    try:
        out, lse = lka.gqa_attn(q, k, v, lens, causal=causal, scale=inp["scale"], return_lse=True)
    finally:
        if split is not None:
            lka.set_split_tokens(prev)
    ref, ref_lse = oracle.gqa(inp["q"], inp["k"], inp["v"], inp["cache_lens"], causal, inp["scale"])
    assert_close(out, ref, torch.bfloat16, "prefill out")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "prefill lse")
    return out


CASES = [
    # (B, h_q, h_kv, s_q, L_lo, L_hi, Lmax, causal)
    (2, 8, 2, 130, 130, 130, 130, True),    # pure prefill, two query tiles with a ragged tail
    (2, 8, 2, 300, 300, 700, 704, True),    # chunked prefill over a cached prefix, ragged lengths
    (2, 8, 2, 200, 200, 450, 450, False),   # every query sees the whole cache
    (1, 4, 4, 64, 64, 64, 64, True),        # MHA, the smallest prefill the kernel takes
    (2, 8, 1, 96, 96, 333, 333, True),      # MQA
    (1, 32, 8, 256, 256, 256, 256, True),   # the Llama-3.1-8B grouping (4 query heads per KV head)
]


@pytest.mark.parametrize("case", CASES)
def test_prefill_matches_oracle(case):
    B, h_q, h_kv, s_q, lo, hi, Lmax, causal = case
    inp = synthetic.gqa_inputs(91, B, h_q, h_kv, 128, s_q, lo, hi, Lmax=Lmax, dtype=torch.bfloat16)
    run_case(inp, causal)


@pytest.mark.parametrize("scale", [-0.05, 0.0])
def test_prefill_any_scale(scale):
    """The prefill kernel applies the scale inside the exponent (raw scores masked, their maximum scaled): a negative
    scale flips the scores, a zero scale gives the mean of the visible values, both as in the definition."""
    inp = synthetic.gqa_inputs(95, 1, 8, 2, 128, 130, 130, 260, Lmax=260, dtype=torch.bfloat16)
    inp["scale"] = scale
    run_case(inp, True)


@pytest.mark.parametrize("split", [128, 256])
def test_prefill_key_splits(split):
    """Key splits (the merge of normalised partials by their lse) give the same result as one pass."""
    inp = synthetic.gqa_inputs(92, 1, 8, 2, 128, 160, 500, 1000, Lmax=1024, dtype=torch.bfloat16)
    out = run_case(inp, True, split=split)
    base = lka.gqa_attn(inp["q"].to(DEV), inp["k"].to(DEV), inp["v"].to(DEV), inp["cache_lens"].to(DEV), causal=True,
                        scale=inp["scale"])
    assert (out.float() - base.float()).abs().max().item() <= 2e-2


@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_prefill_paged(page_size):
    inp = synthetic.gqa_paged_inputs(93, 2, 8, 2, 128, 150, 150, 400, page_size, Lmax=512)
    out = lka.gqa_attn_paged(inp["q"].to(DEV), inp["k_pages"].to(DEV), inp["v_pages"].to(DEV),
                             inp["block_table"].to(DEV), inp["cache_lens"].to(DEV), causal=True, scale=inp["scale"])
    ref, _ = oracle.gqa(inp["q"], inp["k"], inp["v"], inp["cache_lens"], True, inp["scale"])
    assert_close(out, ref, torch.bfloat16, f"paged prefill, pages of {page_size}")


def test_prefill_llama8b_layer_4k_sampled_positions():
    """The Llama-3.1-8B layer (32 query / 8 KV heads, d 128) prefilling 4096 tokens.  Query position t of a
    causal prefill sees keys 0 .. t, so the oracle checks sampled positions as single-query problems over the
    first t + 1 keys (the first and last rows, tile boundaries, and random positions)."""
    w = synthetic.WORKLOADS["gqa_prefill_llama8b_4k"]
    inp = synthetic.make(w, device=DEV)
    out, lse = lka.gqa_attn(inp["q"], inp["k"], inp["v"], inp["cache_lens"], causal=True, scale=inp["scale"],
                            return_lse=True)
    S = w["s_q"]
    gen = np.random.default_rng(94)
    pos = sorted({0, 1, 127, 128, 129, 2047, 2048, S - 129, S - 128, S - 1, *gen.integers(0, S, 6).tolist()})
    q, k, v = inp["q"][:1].cpu(), inp["k"][:1].cpu(), inp["v"][:1].cpu()
    for t in pos:
        ref, ref_lse = oracle.gqa(q[:, :, t:t + 1], k[:, :, :t + 1], v[:, :, :t + 1],
                                  torch.tensor([t + 1], dtype=torch.int32), True, inp["scale"])
        assert_close(out[:1, :, t:t + 1], ref, torch.bfloat16, f"4K prefill, query {t}")
        assert_lse_close(lse[:1, :, t:t + 1], ref_lse, torch.bfloat16, f"4K prefill lse, query {t}")
