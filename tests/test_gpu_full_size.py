"""Full-size parity of the benchmarked workloads that the per-path test files check only at small sizes: the
bench's own inputs and launch (same entry point, same sizes, automatic split plan), with the fp64 oracle on a
sample of sequences (marked gpu).

For the paged workloads the oracle reads the contiguous tensors the page pools were cut from (the pools are
copies of them, laid out by the block table); the oracle pins check that the paged definition equals the
contiguous one."""
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
    torch.cuda.empty_cache()


def _rows(inp, B):
    lens = inp["cache_lens"].cpu()
    return sorted({0, 1, B // 2, B - 1, int(lens.argmax())})


def _sub(inp, rows, batched):
    return {k: (v[rows].cpu() if k in batched else (v.cpu() if isinstance(v, torch.Tensor) else v))
            for k, v in inp.items()}


def test_gqa_paged_full_size():
    w = synthetic.WORKLOADS["gqa_decode_llama8b_paged"]
    inp = synthetic.make(w, device=DEV)
    out, lse = lka.gqa_attn_paged(inp["q"], inp["k_pages"], inp["v_pages"], inp["block_table"], inp["cache_lens"],
                                  causal=True, scale=inp["scale"], return_lse=True)
    rows = _rows(inp, w["B"])
    s = _sub(inp, rows, ("q", "k", "v", "cache_lens"))
    ref, ref_lse = oracle.gqa(s["q"], s["k"], s["v"], s["cache_lens"], True, inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "paged llama8b sample")
    assert_lse_close(lse[rows], ref_lse, torch.bfloat16, "paged llama8b lse")


def test_gqa_fp8_full_size():
    w = synthetic.WORKLOADS["gqa_decode_llama8b_fp8"]
    inp = synthetic.make(w, device=DEV)
    out = lka.gqa_attn_fp8kv(inp["q"], inp["k"], inp["v"], inp["k_scale"], inp["v_scale"], inp["cache_lens"],
                             causal=True, scale=inp["scale"])
    rows = _rows(inp, w["B"])
    s = _sub(inp, rows, ("q", "k", "v", "cache_lens"))
    ref, _ = oracle.gqa_fp8kv(s["q"], s["k"], s["v"], s["k_scale"], s["v_scale"], s["cache_lens"], True,
                              inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "fp8 llama8b sample")


@pytest.mark.parametrize("name", ["latent_decode_4k_sq1", "latent_decode_4k_sq1_paged"])
def test_latent_sq1_full_size(name):
    w = synthetic.WORKLOADS[name]
    inp = synthetic.make(w, device=DEV)
    if "latent_pages" in inp:
        out = lka.latent_absorbed_attn_paged(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent_pages"],
                                             inp["block_table"], inp["cache_lens"], causal=True, scale=inp["scale"])
    else:
        out = lka.latent_absorbed_attn(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                       inp["cache_lens"], causal=True, scale=inp["scale"])
    rows = [0, 1, 31, 63]
    s = _sub(inp, rows, ("q_c", "q_r", "latent", "cache_lens"))
    ref, _ = oracle.latent_absorbed(s["q_c"], s["q_r"], s["w_uk"], s["w_uv"], s["latent"], s["cache_lens"], True,
                                    inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, f"{name} sample")


def test_latent_fp8_full_size():
    w = synthetic.WORKLOADS["latent_decode_4k_sq1_fp8"]
    inp = synthetic.make(w, device=DEV)
    out = lka.latent_absorbed_attn_fp8kv(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent8"],
                                         inp["kv_scale"], inp["cache_lens"], causal=True, scale=inp["scale"])
    rows = [0, 17, 63]
    s = _sub(inp, rows, ("q_c", "q_r", "latent8", "cache_lens"))
    ref, _ = oracle.latent_absorbed_fp8kv(s["q_c"], s["q_r"], s["w_uk"], s["w_uv"], s["latent8"], s["kv_scale"],
                                          s["cache_lens"], True, inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "fp8 latent sample")


def test_latent_sparse_full_size():
    w = synthetic.WORKLOADS["latent_sparse_16k_top2048"]
    inp = synthetic.make(w, device=DEV)
    out = lka.latent_absorbed_attn_sparse(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                          inp["indices"], inp["cache_lens"], scale=inp["scale"])
    rows = [0, 40, 63]
    s = _sub(inp, rows, ("q_c", "q_r", "latent", "indices", "cache_lens"))
    ref, _ = oracle.latent_absorbed_sparse(s["q_c"], s["q_r"], s["w_uk"], s["w_uv"], s["latent"], s["indices"],
                                           s["cache_lens"], inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "sparse latent sample")


def test_gta_chunked_prefill_paged_full_size():
    w = synthetic.WORKLOADS["gta_chunked_prefill_4k_paged"]
    inp = synthetic.make(w, device=DEV)
    out, lse = lka.gta_shared_score_attn_paged(inp["q_g"], inp["k_pages"], inp["v_pages"], inp["block_table"],
                                               inp["cache_lens"], causal=True, scale=inp["scale"], return_lse=True)
    rows = [0, 5]
    s = _sub(inp, rows, ("q_g", "k_g", "v", "cache_lens"))
    ref, ref_lse = oracle.gta(s["q_g"], s["k_g"], s["v"], s["cache_lens"], True, inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "chunked gta sample")
    assert_lse_close(lse[rows], ref_lse, torch.bfloat16, "chunked gta lse")
