"""GPU parity of top-k sparse attention on both GQLA paths against the fp64 oracle (marked gpu)."""
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


@pytest.mark.parametrize("s_q,topk,junk", [(1, 64, 0.0), (1, 300, 0.2), (2, 128, 0.1), (2, 1024, 0.0)])
def test_latent_sparse(s_q, topk, junk):
    inp = synthetic.latent_inputs(600 + topk + s_q, 3, 128, 8, 128, 512, 64, s_q, 40, 700, Lmax=704)
    idx = synthetic.sparse_indices(610 + topk, inp["cache_lens"], s_q, topk, junk=junk)
    d = dev(inp)
    out, lse = lka.latent_absorbed_attn_sparse(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"], d["latent"], idx.to(DEV),
                                               d["cache_lens"], scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle.latent_absorbed_sparse(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"], idx,
                                                 inp["cache_lens"], inp["scale"])
    assert_close(out, ref, torch.bfloat16, "latent sparse out")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "latent sparse lse")


@pytest.mark.parametrize("s_q,topk,junk", [(1, 96, 0.1), (2, 256, 0.2), (2, 1000, 0.0)])
def test_expanded_sparse(s_q, topk, junk):
    inp = synthetic.expanded_inputs(620 + topk + s_q, 3, 128, 8, 128, 64, s_q, 30, 600, Lmax=640)
    idx = synthetic.sparse_indices(630 + topk, inp["cache_lens"], s_q, topk, junk=junk)
    d = dev(inp)
    out, lse = lka.latent_expand_gqa_attn_sparse(d["q_c"], d["q_r"], d["kc"], d["vc"], d["kr"], idx.to(DEV),
                                                 d["cache_lens"], scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle.expanded_sparse(inp["q_c"], inp["q_r"], inp["kc"], inp["vc"], inp["kr"], idx,
                                          inp["cache_lens"], inp["scale"])
    assert_close(out, ref, torch.bfloat16, "expanded sparse out")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "expanded sparse lse")


def test_sparse_full_selection_matches_dense_and_empty_lists():
    inp = synthetic.latent_inputs(640, 2, 128, 8, 128, 512, 64, 2, 100, 300, Lmax=320)
    idx = synthetic.sparse_indices(641, inp["cache_lens"], 2, 320)  # every visible key, shuffled
    idx[1, 0] = -1  # one query with nothing to attend to
    d = dev(inp)
    sp, sp_lse = lka.latent_absorbed_attn_sparse(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"], d["latent"], idx.to(DEV),
                                                 d["cache_lens"], scale=inp["scale"], return_lse=True)
    dense = lka.latent_absorbed_attn(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"], d["latent"], d["cache_lens"],
                                     causal=True, scale=inp["scale"])
    keep = torch.ones(2, 2, dtype=torch.bool)
    keep[1, 0] = False
    for b in range(2):
        for t in range(2):
            if keep[b, t]:
                assert (sp[b, :, t].float() - dense[b, :, t].float()).abs().max().item() <= 2e-2
    assert torch.all(sp[1, :, 0] == 0) and torch.all(torch.isneginf(sp_lse[1, :, 0]))
