"""GPU parity of GTA shared-score attention against the fp64 oracle (marked gpu; C ABI through the binding)."""
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


def run(inp, causal, rows_b=None):
    d = dev(inp)
    out, lse = lka.gta_shared_score_attn(d["q_g"], d["k_g"], d["v"], d["cache_lens"], causal=causal,
                                         scale=inp["scale"], return_lse=True)
    ref, ref_lse = oracle.gta(inp["q_g"], inp["k_g"], inp["v"], inp["cache_lens"], causal, inp["scale"],
                              rows_b=rows_b)
    if rows_b is not None:
        out, lse, ref, ref_lse = out[rows_b], lse[rows_b], ref[rows_b], ref_lse[rows_b]
    assert_close(out, ref, torch.bfloat16, "gta")
    assert_lse_close(lse, ref_lse, torch.bfloat16, "gta lse")
    return out


@pytest.mark.parametrize("causal", [True, False])
def test_gta_prefill_ragged(causal):
    # 200 queries / keys: two query tiles and two key tiles, both ragged
    inp = synthetic.gta_inputs(61, 2, 3, 12, 64, 64, 200, 200, 200)
    run(inp, causal)


@pytest.mark.parametrize("s_q", [1, 2, 5])
def test_gta_decode_bottom_right(s_q):
    inp = synthetic.gta_inputs(62, 3, 3, 12, 64, 64, s_q, s_q, 300, Lmax=320)
    run(inp, True)


@pytest.mark.parametrize("G,H", [(2, 4), (4, 4), (1, 3)])
def test_gta_group_sizes(G, H):
    inp = synthetic.gta_inputs(63, 2, G, H, 64, 64, 130, 130, 130)
    run(inp, True)


def test_gta_single_head_groups_equal_gqa_path():
    """Groups of one head are MHA: the GTA kernel and the GQA kernel agree on the same inputs."""
    inp = synthetic.gta_inputs(64, 2, 4, 4, 64, 64, 1, 1, 257, Lmax=257)
    d = dev(inp)
    a = lka.gta_shared_score_attn(d["q_g"], d["k_g"], d["v"], d["cache_lens"], causal=True, scale=inp["scale"])
    b = lka.gqa_attn(d["q_g"], d["k_g"], d["v"], d["cache_lens"], causal=True, scale=inp["scale"])
    assert (a.float() - b.float()).abs().max().item() <= 2e-2


def test_gta_full_size_sampled():
    """The GTA prefill workload at full size (B = 8, 3 groups x 4 heads, 4096 tokens); two sequences checked."""
    w = synthetic.WORKLOADS["gta_prefill_4k"]
    inp = synthetic.make(w, device=DEV)
    out = lka.gta_shared_score_attn(inp["q_g"], inp["k_g"], inp["v"], inp["cache_lens"], causal=True,
                                    scale=inp["scale"])
    rows = [0, 7]
    sub = {k: (v[rows].cpu() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    ref, _ = oracle.gta(sub["q_g"], sub["k_g"], sub["v"], sub["cache_lens"], True, inp["scale"])
    assert_close(out[rows], ref, torch.bfloat16, "gta full-size sample")


@pytest.mark.parametrize("split", [128, 384])
def test_gta_forced_key_splits(split):
    """Key splits (partials merged by the GTA merge kernel) on a chunked prefill: 200 queries over up to 700 cached
    keys, ragged lengths; the result stays within tolerance of the definition."""
    inp = synthetic.gta_inputs(65, 3, 3, 12, 64, 64, 200, 217, 700, Lmax=704)
    prev = lka.set_split_tokens(split)
    try:
        run(inp, True)
    finally:
        lka.set_split_tokens(prev)


def test_gta_automatic_key_split_chunked_prefill():
    """A small grid (one query tile per group and sequence) is split along the keys automatically."""
    inp = synthetic.gta_inputs(66, 2, 3, 12, 64, 64, 100, 1500, 3000, Lmax=3072)
    run(inp, True)
    nb = lka.library().gta_shared_score_attn_workspace_size(2, 3, 12, 100, 64, 64, 3072)
    assert nb > 256  # split partials in the workspace
