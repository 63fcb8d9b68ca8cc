"""GPU parity of gqa_attn against the fp64 oracle (marked gpu; calls the C ABI through the binding)."""
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


def run_case(inp, causal, dtype, rows_b=None):
    q, k, v, lens = (inp["q"].to(DEV), inp["k"].to(DEV), inp["v"].to(DEV), inp["cache_lens"].to(DEV))
    out, lse = lka.gqa_attn(q, k, v, lens, causal=causal, scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle.gqa(inp["q"], inp["k"], inp["v"], inp["cache_lens"], causal, inp["scale"], rows_b=rows_b)
    if rows_b is not None:
        out, lse, ref, ref_lse = out[rows_b], lse[rows_b], ref[rows_b], ref_lse[rows_b]
    assert_close(out, ref, dtype, "out")
    assert_lse_close(lse, ref_lse, dtype, "lse")
    return out


# ------------------------------------------------------------------ the glossary page's example, fp32
def test_glossary_example_prefill_and_decode_fp32():
    ex = synthetic.gqa_page_example()
    lens16 = torch.tensor([16], dtype=torch.int32)
    inp = dict(q=ex["q"], k=ex["k"], v=ex["v"], cache_lens=lens16, scale=1 / 8)
    out = run_case(inp, True, torch.float32)
    # GQA equals MHA over repeat_interleave'd K/V, on the GPU path too
    mha = lka.gqa_attn(ex["q"].to(DEV), ex["k"].repeat_interleave(4, 1).to(DEV), ex["v"].repeat_interleave(4, 1).to(DEV),
                       lens16.to(DEV), causal=True, scale=1 / 8)
    assert torch.allclose(out, mha, atol=1e-6)
    # decode step appending the 17th token
    k = torch.cat([ex["k"], ex["k17"]], 2)
    v = torch.cat([ex["v"], ex["v17"]], 2)
    dec = dict(q=ex["q17"], k=k, v=v, cache_lens=torch.tensor([17], dtype=torch.int32), scale=1 / 8)
    run_case(dec, True, torch.float32)


# ------------------------------------------------------------------ random shapes, tails, ragged lengths
CASES = [
    # (B, h_q, h_kv, d, s_q, L_lo, L_hi, Lmax, causal)
    (3, 32, 8, 128, 1, 1, 300, 300, True),      # L=1 possible, ragged tails
    (4, 32, 8, 128, 2, 2, 777, 800, True),      # MTP, bottom-right causal
    (2, 8, 8, 128, 1, 50, 130, 130, False),     # MHA
    (2, 16, 1, 128, 1, 1, 65, 65, True),        # MQA
    (2, 8, 2, 64, 3, 3, 200, 256, True),        # d=64, s_q=3
    (2, 16, 2, 256, 1, 100, 333, 333, True),    # d=256, 8 heads per group
    (1, 32, 2, 128, 1, 500, 1000, 1024, True),  # 16 heads per group (two row blocks of 8... or one of 16)
    (2, 4, 4, 128, 37, 37, 90, 96, True),       # prefill-like s_q
    (1, 2, 1, 128, 1, 63, 63, 64, True),        # L < tile
    (2, 24, 2, 128, 1, 70, 500, 512, True),     # 12 rows: the 16-row tensor-core form with padding rows
    (1, 64, 2, 128, 1, 200, 400, 400, True),    # 32 rows: two row blocks of 16
    (2, 8, 2, 128, 3, 3, 300, 320, True),       # 12 rows of 3 query tokens (per-row causal limits)
    (2, 8, 4, 64, 4, 4, 150, 160, True),        # 8 rows of 4 query tokens: the 8-row form, d = 64
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}h{c[1]}kv{c[2]}d{c[3]}sq{c[4]}L{c[6]}" for c in CASES])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_gqa_random(case, dtype):
    B, h_q, h_kv, d, s_q, lo, hi, Lmax, causal = case
    if dtype == torch.float32 and d == 256:
        pytest.skip("fp32 supports d_h in {64, 128}")
    inp = synthetic.gqa_inputs(100 + len(str(case)), B, h_q, h_kv, d, s_q, lo, hi, Lmax=Lmax, dtype=dtype)
    run_case(inp, causal, dtype)


def test_fused_split_merge_is_repeatable():
    """Repeated calls with different key-split plans on one workspace (rows of one block needing different
    split counts, s_q = 4 causal) give the oracle's result every time, and the same bits for the same plan:
    nothing a call leaves in the workspace changes the next one."""
    inp = synthetic.gqa_inputs(8, 3, 16, 4, 128, 4, 300, 1000, Lmax=1024, dtype=torch.bfloat16)
    q, k, v, lens = (inp[n].to(DEV) for n in ("q", "k", "v", "cache_lens"))
    ref, _ = oracle.gqa(inp["q"], inp["k"], inp["v"], inp["cache_lens"], True, inp["scale"])
    outs = []
    for split in (128, 64, 128, 0, 128):
        prev = lka.set_split_tokens(split)
        try:
            out = lka.gqa_attn(q, k, v, lens, causal=True, scale=inp["scale"])
        finally:
            lka.set_split_tokens(prev)
        assert_close(out, ref, torch.bfloat16, f"splits of {split}")
        outs.append(out)
    assert torch.equal(outs[0], outs[2]) and torch.equal(outs[0], outs[4])


@pytest.mark.parametrize("split", [64, 128, 448, 4096])
def test_split_count_does_not_change_result(split):
    inp = synthetic.gqa_inputs(7, 3, 32, 8, 128, 1, 900, 2000, Lmax=2048, dtype=torch.bfloat16)
    prev = lka.set_split_tokens(split)
    try:
        out = run_case(inp, True, torch.bfloat16)
    finally:
        lka.set_split_tokens(prev)
    base = lka.gqa_attn(inp["q"].to(DEV), inp["k"].to(DEV), inp["v"].to(DEV), inp["cache_lens"].to(DEV),
                        causal=True, scale=inp["scale"])
    assert (out.float() - base.float()).abs().max().item() <= 2e-2


def test_full_size_llama8b_decode_sampled_rows():
    """The Llama-3.1-8B decode layer at full size (B=64, lengths in [1024, 8192]); the oracle checks a
    sample of sequences: the first, second, middle, last and the longest."""
    w = synthetic.WORKLOADS["gqa_decode_llama8b"]
    inp = synthetic.make(w, device=DEV)
    lens = inp["cache_lens"].cpu()
    rows = sorted({0, 1, w["B"] // 2, w["B"] - 1, int(lens.argmax())})
    out = lka.gqa_attn(inp["q"], inp["k"], inp["v"], inp["cache_lens"], causal=True, scale=inp["scale"])
    sub = {kk: (vv[rows].cpu() if isinstance(vv, torch.Tensor) else vv) for kk, vv in inp.items()}
    ref, _ = oracle.gqa(sub["q"], sub["k"], sub["v"], sub["cache_lens"], True, inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "llama8b decode sample")


def test_empty_batch_is_noop():
    q = torch.empty(0, 8, 1, 128, dtype=torch.bfloat16, device=DEV)
    k = torch.empty(0, 2, 16, 128, dtype=torch.bfloat16, device=DEV)
    out = lka.gqa_attn(q, k, k, torch.empty(0, dtype=torch.int32, device=DEV))
    assert out.shape == q.shape


def test_bad_length_is_clamped_and_reported():
    inp = synthetic.gqa_inputs(9, 2, 8, 2, 128, 1, 40, 40, Lmax=40, dtype=torch.bfloat16)
    lens = torch.tensor([40, 999], dtype=torch.int32, device=DEV)  # 999 > Lmax
    lka.gqa_attn(inp["q"].to(DEV), inp["k"].to(DEV), inp["v"].to(DEV), lens)
    assert lka.device_status() == 6  # LKA_ERR_BAD_LENGTH
    lka.clear_status()


def test_bounded_wait_times_out_and_reports():
    lib = lka.library()
    ws = lka.workspaces.get(256, torch.device(DEV))
    rc = lib.lka_selftest_wait_timeout(lka._ptr(ws), ws.numel(), 2000, lka._stream_ptr())
    assert rc == 0
    assert lka.device_status() == 5  # LKA_ERR_TIMEOUT; the context stays usable
    lka.clear_status()
    x = torch.ones(4, device=DEV)
    assert x.sum().item() == 4.0
