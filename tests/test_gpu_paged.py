"""GPU parity of the paged-cache entry points (GQA, both GQLA paths, GTA) against the fp64 oracle (marked gpu)."""
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


def run_paged(inp, causal, dtype):
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse = lka.gqa_attn_paged(d["q"], d["k_pages"], d["v_pages"], d["block_table"], d["cache_lens"],
                                  causal=causal, scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle.gqa_paged(inp["q"], inp["k_pages"], inp["v_pages"], inp["block_table"], inp["cache_lens"],
                                    causal, inp["scale"])
    assert_close(out, ref, dtype, "paged out")
    assert_lse_close(lse, ref_lse, dtype, "paged lse")
    # the same call on the contiguous cache the table describes gives the same bits
    cont = lka.gqa_attn(d["q"], d["k"], d["v"], d["cache_lens"], causal=causal, scale=inp["scale"])
    assert torch.equal(out, cont)
    return out


CASES = [
    # (B, h_q, h_kv, d, s_q, L_lo, L_hi, Lmax, causal)
    (3, 32, 8, 128, 1, 1, 700, 768, True),     # Llama-3.1-8B heads, ragged, L=1 possible
    (2, 8, 2, 64, 3, 3, 300, 512, True),       # d=64, s_q=3 bottom-right causal
    (2, 8, 8, 128, 1, 40, 250, 256, False),    # MHA
    (2, 16, 2, 256, 1, 60, 333, 512, True),    # d=256, 8 heads per group
    (1, 32, 2, 128, 2, 300, 900, 1024, True),  # 16 heads per group, MTP
]


@pytest.mark.parametrize("page_size", [16, 64, 128, 256])
@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}sq{c[4]}" for c in CASES])
def test_paged_bf16(case, page_size):
    B, h_q, h_kv, d, s_q, lo, hi, Lmax, causal = case
    inp = synthetic.gqa_paged_inputs(200 + page_size + B * d, B, h_q, h_kv, d, s_q, lo, hi, page_size, Lmax=Lmax,
                                     dtype=torch.bfloat16)
    run_paged(inp, causal, torch.bfloat16)


@pytest.mark.parametrize("page_size", [8, 32, 128])
def test_paged_fp32(page_size):
    inp = synthetic.gqa_paged_inputs(300 + page_size, 2, 8, 2, 64, 1, 1, 200, page_size, Lmax=256,
                                     dtype=torch.float32)
    run_paged(inp, True, torch.float32)


def test_paged_out_of_pool_entry_is_replaced_and_reported():
    inp = synthetic.gqa_paged_inputs(301, 2, 8, 2, 128, 1, 100, 120, 16, Lmax=128, dtype=torch.bfloat16)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    bt = d["block_table"].clone()
    bt[1, 0] = d["k_pages"].shape[0] + 5  # a page the second sequence needs, outside the pool
    lka.gqa_attn_paged(d["q"], d["k_pages"], d["v_pages"], bt, d["cache_lens"], scale=inp["scale"])
    assert lka.device_status() == 7  # LKA_ERR_BAD_PAGE
    lka.clear_status()


@pytest.mark.parametrize("page_size,s_q", [(16, 1), (64, 2), (128, 1), (256, 2)])
def test_latent_absorbed_paged(page_size, s_q):
    inp = synthetic.latent_paged_inputs(400 + page_size + s_q, 2, 128, 8, 128, 512, 64, s_q, s_q, 700, page_size,
                                        Lmax=768)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse = lka.latent_absorbed_attn_paged(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"], d["latent_pages"],
                                              d["block_table"], d["cache_lens"], causal=True, scale=inp["scale"],
                                              return_lse=True)
    ref, ref_lse = oracle.latent_absorbed_paged(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent_pages"],
                                                inp["block_table"], inp["cache_lens"], True, inp["scale"])
    assert_close(out, ref, torch.bfloat16, "latent paged out")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "latent paged lse")
    cont = lka.latent_absorbed_attn(d["q_c"], d["q_r"], d["w_uk"], d["w_uv"], d["latent"], d["cache_lens"],
                                    causal=True, scale=inp["scale"])
    assert torch.equal(out, cont)


@pytest.mark.parametrize("page_size,s_q", [(16, 2), (64, 1), (128, 2), (256, 1)])
def test_expanded_paged(page_size, s_q):
    from test_gpu_expanded import oracle_expanded

    inp = synthetic.expanded_paged_inputs(500 + page_size + s_q, 3, 128, 8, 128, 64, s_q, s_q, 600, page_size,
                                          Lmax=640)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse = lka.latent_expand_gqa_attn_paged(d["q_c"], d["q_r"], d["kc_pages"], d["vc_pages"], d["kr_pages"],
                                                d["block_table"], d["cache_lens"], causal=True, scale=inp["scale"],
                                                return_lse=True)
    ref, ref_lse = oracle_expanded(inp, True)
    assert_close(out, ref, torch.bfloat16, "expanded paged out")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "expanded paged lse")
    cont = lka.latent_expand_gqa_attn(d["q_c"], d["q_r"], d["kc"], d["vc"], d["kr"], d["cache_lens"], causal=True,
                                      scale=inp["scale"])
    assert torch.equal(out, cont)


@pytest.mark.parametrize("page_size,s_q", [(16, 200), (64, 1), (128, 130), (256, 5)])
def test_gta_paged(page_size, s_q):
    """Chunked GTA prefill against a paged cache: s_q new queries over a ragged cached prefix (bottom-right
    causal), two query tiles at s_q = 200, ragged last page and last key tile."""
    inp = synthetic.gta_paged_inputs(600 + page_size + s_q, 3, 3, 12, 64, 64, s_q, s_q + 17, 470, page_size,
                                     Lmax=512)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    out, lse = lka.gta_shared_score_attn_paged(d["q_g"], d["k_pages"], d["v_pages"], d["block_table"],
                                               d["cache_lens"], causal=True, scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle.gta_paged(inp["q_g"], inp["k_pages"], inp["v_pages"], inp["block_table"], inp["cache_lens"],
                                    True, inp["scale"])
    assert_close(out, ref, torch.bfloat16, "gta paged out")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "gta paged lse")
    cont = lka.gta_shared_score_attn(d["q_g"], d["k_g"], d["v"], d["cache_lens"], causal=True, scale=inp["scale"])
    assert torch.equal(out, cont)


def test_gta_paged_out_of_pool_entry_is_replaced_and_reported():
    inp = synthetic.gta_paged_inputs(650, 2, 2, 4, 64, 64, 4, 100, 120, 32, Lmax=128)
    d = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    bt = d["block_table"].clone()
    bt[0, 1] = -3  # a page the first sequence needs, outside the pool
    lka.gta_shared_score_attn_paged(d["q_g"], d["k_pages"], d["v_pages"], bt, d["cache_lens"], scale=inp["scale"])
    assert lka.device_status() == 7  # LKA_ERR_BAD_PAGE
    lka.clear_status()
