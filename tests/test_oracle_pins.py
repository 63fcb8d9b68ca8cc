"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test ties an oracle routine to something the pages or the mathematics fix:
the glossary page's worked example and its printed facts, a library routine
(torch's float64 scaled_dot_product_attention with an explicit mask) on the
special cases it covers, closed forms, invariants the pages state (GQA with
h_kv = h_q is MHA, h_kv = 1 is MQA, GQA equals MHA over repeat_interleave'd
K/V, the absorbed latent path equals the expanded per-group path, a GTA group
of one head is MHA) and brute-force special cases.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synthetic

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def bottom_right_mask(s_q, L, causal):
    t = torch.arange(s_q)[:, None]
    j = torch.arange(L)[None, :]
    if not causal:
        return torch.ones(s_q, L, dtype=torch.bool)
    return j <= (L - s_q + t)


def sdpa64(q, k, v, L, causal, scale):
    """Library routine: torch float64 SDPA over the first L cache slots, bottom-right causal mask."""
    s_q = q.shape[-2]
    m = bottom_right_mask(s_q, L, causal)
    return F.scaled_dot_product_attention(q.double(), k[..., :L, :].double(), v[..., :L, :].double(),
                                          attn_mask=m, scale=scale)


def rand(*shape, seed=0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g, dtype=torch.float64)


# --------------------------------------------------------------------------- glossary example
def test_glossary_worked_example():
    gd = golden("gqa_glossary_example.json")
    ex = synthetic.gqa_page_example()
    q, k, v = ex["q"], ex["k"], ex["v"]
    assert list(q.shape) == gd["q_shape"] and list(k.shape) == gd["kv_shape"]
    lens = [16]
    out, _ = oracle.gqa(q, k, v, lens, causal=True, scale=1 / 8)
    assert list(out.shape) == gd["printed_output_shape"]
    # "same as copied heads": GQA equals MHA over repeat_interleave'd K/V
    rep = q.shape[1] // k.shape[1]
    out_mha, _ = oracle.gqa(q, k.repeat_interleave(rep, 1), v.repeat_interleave(rep, 1), lens, True, 1 / 8)
    assert np.allclose(out, out_mha, atol=gd["allclose_atol"]) == gd["printed_same_as_copied_heads"]
    # the library routine the page calls, in float64
    ref = F.scaled_dot_product_attention(q.double(), k.double(), v.double(), is_causal=True, enable_gqa=True)
    assert np.abs(out - ref.numpy()).max() < 1e-12
    # the page's second printed line
    assert k[0, :, 0].numel() * 2 == gd["printed_cached_values_per_token_gqa"]
    assert k.repeat_interleave(rep, 1)[0, :, 0].numel() * 2 == gd["printed_cached_values_per_token_mha"]


def test_decode_step_equals_prefill_row():
    """Appending a 17th token and decoding it equals row 17 of a 17-token causal prefill."""
    ex = synthetic.gqa_page_example()
    k = torch.cat([ex["k"], ex["k17"]], 2)
    v = torch.cat([ex["v"], ex["v17"]], 2)
    dec, dlse = oracle.gqa(ex["q17"], k, v, [17], True, 1 / 8)
    pre, plse = oracle.gqa(torch.cat([ex["q"], ex["q17"]], 2), k, v, [17], True, 1 / 8)
    assert np.abs(dec[:, :, 0] - pre[:, :, 16]).max() < 1e-14
    assert np.abs(dlse[:, :, 0] - plse[:, :, 16]).max() < 1e-14


# --------------------------------------------------------------------------- GQA against SDPA
@pytest.mark.parametrize("h_q,h_kv", [(8, 8), (8, 1), (8, 2), (6, 3)])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("s_q", [1, 2, 5])
def test_gqa_matches_library_sdpa(h_q, h_kv, causal, s_q):
    B, d, Lmax = 3, 16, 23
    q, k, v = rand(B, h_q, s_q, d, seed=1), rand(B, h_kv, Lmax, d, seed=2), rand(B, h_kv, Lmax, d, seed=3)
    lens = [23, 7, s_q]
    scale = 0.37
    out, lse = oracle.gqa(q, k, v, lens, causal, scale)
    rep = h_q // h_kv
    for b, L in enumerate(lens):
        ref = sdpa64(q[b:b + 1], k[b:b + 1].repeat_interleave(rep, 1), v[b:b + 1].repeat_interleave(rep, 1), L,
                     causal, scale)
        assert np.abs(out[b] - ref[0].numpy()).max() < 1e-12
        # lse from its definition: log of the softmax normaliser of the scaled scores
        kk = k[b].repeat_interleave(rep, 0)[:, :L]
        s = scale * torch.einsum("htd,hjd->htj", q[b], kk)
        s = s.masked_fill(~bottom_right_mask(s_q, L, causal), -math.inf)
        assert np.abs(lse[b] - torch.logsumexp(s, -1).numpy()).max() < 1e-12


def test_bottom_right_reading_differs_from_top_left():
    """The decode/MTP reading: query t sees keys <= L - s_q + t (torch's is_causal is top-left)."""
    q, k, v = rand(1, 2, 2, 8, seed=4), rand(1, 2, 9, 8, seed=5), rand(1, 2, 9, 8, seed=6)
    out, _ = oracle.gqa(q, k, v, [9], True, 0.5)
    br = sdpa64(q, k, v, 9, True, 0.5).numpy()
    tl = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=0.5).numpy()
    assert np.abs(out - br).max() < 1e-12
    assert np.abs(out - tl).max() > 1e-3


def test_grouping_is_contiguous():
    """Head i uses KV head floor(i / (h_q/h_kv)) -- repeat_interleave, not i % h_kv."""
    q, k, v = rand(1, 4, 1, 8, seed=7), rand(1, 2, 5, 8, seed=8), rand(1, 2, 5, 8, seed=9)
    out, _ = oracle.gqa(q, k, v, [5], False, 1.0)
    wrong = sdpa64(q, k.repeat(1, 2, 1, 1), v.repeat(1, 2, 1, 1), 5, False, 1.0).numpy()
    right = sdpa64(q, k.repeat_interleave(2, 1), v.repeat_interleave(2, 1), 5, False, 1.0).numpy()
    assert np.abs(out - right).max() < 1e-12 and np.abs(out - wrong).max() > 1e-3


# --------------------------------------------------------------------------- brute-force special cases
def test_single_key_returns_its_value():
    q, k, v = rand(2, 4, 1, 8, seed=10), rand(2, 2, 4, 8, seed=11), rand(2, 2, 4, 8, seed=12)
    out, lse = oracle.gqa(q, k, v, [1, 1], True, 0.3)
    for i in range(4):
        assert np.abs(out[:, i, 0] - v[:, i // 2, 0].numpy()).max() < 1e-15
        s0 = 0.3 * (q[:, i, 0] * k[:, i // 2, 0]).sum(-1).numpy()
        assert np.abs(lse[:, i, 0] - s0).max() < 1e-14


def test_zero_scale_is_prefix_mean():
    q, k, v = rand(1, 2, 3, 8, seed=13), rand(1, 1, 10, 8, seed=14), rand(1, 1, 10, 8, seed=15)
    out, lse = oracle.gqa(q, k, v, [10], True, 0.0)
    for t in range(3):
        n = 10 - 3 + t + 1
        assert np.abs(out[0, :, t] - v[0, 0, :n].mean(0).numpy()).max() < 1e-14
        assert abs(lse[0, 0, t] - math.log(n)) < 1e-14


def test_equal_keys_give_mean_of_values():
    q = rand(1, 2, 1, 8, seed=16)
    k = rand(1, 1, 1, 8, seed=17).expand(1, 1, 12, 8).contiguous()
    v = rand(1, 1, 12, 8, seed=18)
    out, _ = oracle.gqa(q, k, v, [12], False, 0.9)
    assert np.abs(out[0, :, 0] - v[0, 0].mean(0).numpy()).max() < 1e-14


def test_key_permutation_invariance():
    q, k, v = rand(1, 2, 2, 8, seed=19), rand(1, 1, 11, 8, seed=20), rand(1, 1, 11, 8, seed=21)
    perm = torch.randperm(11, generator=torch.Generator().manual_seed(3))
    a, la = oracle.gqa(q, k, v, [11], False, 0.7)
    b, lb = oracle.gqa(q, k[:, :, perm], v[:, :, perm], [11], False, 0.7)
    assert np.abs(a - b).max() < 1e-13 and np.abs(la - lb).max() < 1e-13


def test_dominant_score_selects_value():
    d = 8
    q = torch.zeros(1, 1, 1, d, dtype=torch.float64)
    q[..., 0] = 1.0
    k = rand(1, 1, 6, d, seed=22) * 0.01
    k[0, 0, 4, 0] = 50.0
    v = rand(1, 1, 6, d, seed=23)
    out, _ = oracle.gqa(q, k, v, [6], False, 1.0)
    assert np.abs(out[0, 0, 0] - v[0, 0, 4].numpy()).max() < 1e-15


def test_probabilities_sum_to_one_and_reproduce_output():
    q, k, v = rand(2, 4, 2, 16, seed=24), rand(2, 2, 30, 16, seed=25), rand(2, 2, 30, 16, seed=26)
    lens = [30, 13]
    out, _ = oracle.gqa(q, k, v, lens, True, 0.25)
    for b in range(2):
        for i in range(4):
            for t in range(2):
                p = oracle.gqa_probs(q, k, lens, True, 0.25, b, i, t, h_kv=2)
                assert len(p) == lens[b] - 2 + t + 1
                assert abs(p.sum() - 1.0) < 1e-12 and (p >= 0).all()
                assert np.abs(p @ v[b, i // 2, :len(p)].numpy() - out[b, i, t]).max() < 1e-13


def test_merge_of_disjoint_partials_equals_full_attention():
    """The split-KV combine, pinned against attention over the whole key set."""
    q, k, v = rand(1, 1, 1, 16, seed=27), rand(1, 1, 40, 16, seed=28), rand(1, 1, 40, 16, seed=29)
    full, flse = oracle.gqa(q, k, v, [40], False, 0.5)
    cuts = [0, 7, 8, 25, 40]
    po, pl = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        o, l = oracle.gqa(q, k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous(), [b - a], False, 0.5)
        po.append(o[0, 0, 0])
        pl.append(l[0, 0, 0])
    m, ml = oracle.merge_partials(np.stack(po), np.array(pl))
    assert np.abs(m - full[0, 0, 0]).max() < 1e-13 and abs(ml - flse[0, 0, 0]) < 1e-13


def test_invalid_arguments_rejected():
    q, k, v = rand(1, 2, 2, 8), rand(1, 1, 5, 8), rand(1, 1, 5, 8)
    with pytest.raises(ValueError):
        oracle.gqa(q, k, v, [6], True, 1.0)  # L > Lmax
    with pytest.raises(ValueError):
        oracle.gqa(q, k, v, [1], True, 1.0)  # causal with L < s_q
    with pytest.raises(ValueError):
        oracle.gqa(rand(1, 3, 1, 8), rand(1, 2, 5, 8), rand(1, 2, 5, 8), [5], False, 1.0)  # h_q % h_kv


# --------------------------------------------------------------------------- GQLA latent
def latent_case(B=2, h_q=8, g=2, d_h=16, r_kv=32, d_r=8, s_q=2, Lmax=19, seed=40):
    lat = synthetic.latent_inputs(seed, B, h_q, g, d_h, r_kv, d_r, s_q, 3, Lmax, dtype=torch.float64)
    return lat


def torch_latent_expanded(lat, causal):
    """Eq. (1) with torch ops: k^C = W^UK_gamma c, v^C = W^UV_gamma c, key [k^C; k^R], query [q^C; q^R]."""
    q_c, q_r, w_uk, w_uv, c = lat["q_c"], lat["q_r"], lat["w_uk"], lat["w_uv"], lat["latent"]
    g, d_h, r_kv = w_uk.shape
    B, h_q, s_q, _ = q_c.shape
    rep = h_q // g
    outs = []
    for b, L in enumerate(lat["cache_lens"].tolist()):
        cb = c[b, :L, :r_kv]
        kr = c[b, :L, r_kv:]
        kc = torch.einsum("gdr,jr->gjd", w_uk, cb)          # [g, L, d_h]
        vc = torch.einsum("gdr,jr->gjd", w_uv, cb)
        key = torch.cat([kc, kr.expand(g, L, kr.shape[-1])], -1).repeat_interleave(rep, 0)
        val = vc.repeat_interleave(rep, 0)
        qry = torch.cat([q_c[b], q_r[b]], -1)
        outs.append(sdpa64(qry, key, val, L, causal, lat["scale"]))
    return torch.stack(outs).numpy()


@pytest.mark.parametrize("causal", [True, False])
def test_latent_expanded_matches_library(causal):
    lat = latent_case()
    out, _ = oracle.latent_expanded(lat["q_c"], lat["q_r"], lat["w_uk"], lat["w_uv"], lat["latent"],
                                    lat["cache_lens"], causal, lat["scale"])
    ref = torch_latent_expanded(lat, causal)
    assert np.abs(out - ref).max() < 1e-12


@pytest.mark.parametrize("s_q", [1, 2])
def test_absorbed_equals_expanded(s_q):
    """GQLA section 3.1 / Figure 2: the two decode paths give the same output."""
    lat = latent_case(s_q=s_q, seed=41)
    args = (lat["q_c"], lat["q_r"], lat["w_uk"], lat["w_uv"], lat["latent"], lat["cache_lens"], True,
            lat["scale"])
    a, la = oracle.latent_absorbed(*args)
    e, le = oracle.latent_expanded(*args)
    assert np.abs(a - e).max() <= 1e-10 * np.abs(e).max()
    assert np.abs(la - le).max() < 1e-11


def test_latent_identity_weights_reduce_to_mqa():
    """g = 1, d_h = r_kv, W^UK = W^UV = I: one shared key [c; k^R] and value c for all heads (MQA)."""
    B, h_q, r, d_r, s_q, Lmax = 2, 4, 16, 8, 2, 9
    lat = synthetic.latent_inputs(42, B, h_q, 1, r, r, d_r, s_q, 4, Lmax, dtype=torch.float64)
    eye = torch.eye(r, dtype=torch.float64)[None]
    args = (lat["q_c"], lat["q_r"], eye, eye, lat["latent"], lat["cache_lens"], True, 0.3)
    a, _ = oracle.latent_absorbed(*args)
    e, _ = oracle.latent_expanded(*args)
    for b, L in enumerate(lat["cache_lens"].tolist()):
        key = lat["latent"][b:b + 1, None, :L].expand(1, h_q, L, r + d_r)
        val = lat["latent"][b:b + 1, None, :L, :r].expand(1, h_q, L, r)
        qry = torch.cat([lat["q_c"][b:b + 1], lat["q_r"][b:b + 1]], -1)
        ref = sdpa64(qry, key, val, L, True, 0.3)[0].numpy()
        assert np.abs(a[b] - ref).max() < 1e-12 and np.abs(e[b] - ref).max() < 1e-12


def test_expand_cache_then_gqa_equals_latent():
    """The one-time cache expansion followed by GQA over [kc; kr] equals the latent definition."""
    lat = latent_case(seed=43)
    kc, vc, kr = oracle.latent_expand_cache(lat["latent"], lat["w_uk"], lat["w_uv"])
    g = lat["w_uk"].shape[0]
    key = np.concatenate([kc, np.broadcast_to(kr[:, None], kc.shape[:3] + (kr.shape[-1],))], -1)
    # GQA over the concatenated key needs equal K/V widths: pad V with zeros, then drop them.
    pad = np.zeros(vc.shape[:3] + (kr.shape[-1],))
    val = np.concatenate([vc, pad], -1)
    q = torch.cat([lat["q_c"], lat["q_r"]], -1)
    out, lse = oracle.gqa(q, key, val, lat["cache_lens"], True, lat["scale"])
    e, le = oracle.latent_expanded(lat["q_c"], lat["q_r"], lat["w_uk"], lat["w_uv"], lat["latent"],
                                   lat["cache_lens"], True, lat["scale"])
    assert np.abs(out[..., :kc.shape[-1]] - e).max() < 1e-12
    assert np.abs(out[..., kc.shape[-1]:]).max() == 0.0
    assert np.abs(lse - le).max() < 1e-12
    assert g == kc.shape[1]


# --------------------------------------------------------------------------- GTA
@pytest.mark.parametrize("G,H", [(3, 12), (2, 2), (1, 4)])
@pytest.mark.parametrize("causal", [True, False])
def test_gta_matches_library(G, H, causal):
    B, s_q, d_qk, d_v, Lmax = 2, 5, 16, 8, 13
    gt = synthetic.gta_inputs(44, B, G, H, d_qk, d_v, s_q, 5, Lmax, dtype=torch.float64)
    out, lse = oracle.gta(gt["q_g"], gt["k_g"], gt["v"], gt["cache_lens"], causal, 0.4)
    rep = H // G
    for b, L in enumerate(gt["cache_lens"].tolist()):
        ref = sdpa64(gt["q_g"][b].repeat_interleave(rep, 0), gt["k_g"][b].repeat_interleave(rep, 0), gt["v"][b], L,
                     causal, 0.4)
        assert np.abs(out[b] - ref.numpy()).max() < 1e-12
        s = 0.4 * torch.einsum("gtd,gjd->gtj", gt["q_g"][b], gt["k_g"][b, :, :L])
        s = s.masked_fill(~bottom_right_mask(s_q, L, causal), -math.inf)
        assert np.abs(lse[b] - torch.logsumexp(s, -1).numpy()).max() < 1e-12


def test_gta_equal_values_give_equal_head_outputs():
    B, G, H, s_q, d, Lmax = 1, 2, 8, 3, 8, 7
    gt = synthetic.gta_inputs(45, B, G, H, d, d, s_q, 7, Lmax, dtype=torch.float64)
    v = gt["v"][:, :1].expand(B, H, Lmax, d).contiguous()
    out, _ = oracle.gta(gt["q_g"], gt["k_g"], v, gt["cache_lens"], True, 0.5)
    for grp in range(G):
        hs = range(grp * 4, grp * 4 + 4)
        for h in hs:
            assert np.abs(out[0, h] - out[0, grp * 4]).max() == 0.0
    assert np.abs(out[0, 0] - out[0, 4]).max() > 1e-6


def test_gta_single_head_groups_is_mha():
    B, H, s_q, d, Lmax = 2, 3, 4, 8, 9
    gt = synthetic.gta_inputs(46, B, H, H, d, d, s_q, 4, Lmax, dtype=torch.float64)
    out, _ = oracle.gta(gt["q_g"], gt["k_g"], gt["v"], gt["cache_lens"], True, 0.6)
    ref, _ = oracle.gqa(gt["q_g"], gt["k_g"], gt["v"], gt["cache_lens"], True, 0.6)
    assert np.abs(out - ref).max() == 0.0


# ------------------------------------------------------------------ paged KV cache (gather) -----------------
def test_paged_oracle_identity_layout_equals_contiguous():
    """Pages cut from the contiguous cache in order (block_table[b, j] = b * max_pages + j): the paged
    definition is the contiguous one ("Grouped Query Attention (GQA)" glossary page, PagedAttention keeps the
    cache in fixed-size blocks)."""
    inp = synthetic.gqa_inputs(61, 3, 8, 2, 32, 2, 2, 48, Lmax=48, dtype=torch.float32)
    ps = 16
    B, h_kv, Lmax, d = inp["k"].shape
    mp = Lmax // ps
    pages = lambda c: c.reshape(B, h_kv, mp, ps, d).permute(0, 2, 1, 3, 4).reshape(B * mp, h_kv, ps, d)  # noqa: E731
    table = torch.arange(B * mp, dtype=torch.int32).reshape(B, mp)
    ref, ref_lse = oracle.gqa(inp["q"], inp["k"], inp["v"], inp["cache_lens"], True, 0.2)
    out, lse = oracle.gqa_paged(inp["q"], pages(inp["k"]), pages(inp["v"]), table, inp["cache_lens"], True, 0.2)
    assert np.array_equal(out, ref) and np.array_equal(lse, ref_lse)


def test_paged_oracle_shuffled_pool_and_shared_prefix():
    # a shuffled pool with unused entries -1 gives the contiguous result
    inp = synthetic.gqa_paged_inputs(62, 4, 8, 4, 32, 1, 1, 60, 8, Lmax=64, dtype=torch.float32)
    ref, _ = oracle.gqa(inp["q"], inp["k"], inp["v"], inp["cache_lens"], False, 0.3)
    out, _ = oracle.gqa_paged(inp["q"], inp["k_pages"], inp["v_pages"], inp["block_table"], inp["cache_lens"],
                              False, 0.3)
    assert np.allclose(out, ref, atol=0, rtol=0)
    # two sequences sharing their first page (a common prompt prefix): equal to duplicating that page
    g = torch.Generator().manual_seed(63)
    pool_k = torch.randn(5, 2, 8, 16, generator=g)
    pool_v = torch.randn(5, 2, 8, 16, generator=g)
    table = torch.tensor([[3, 1], [3, 4]], dtype=torch.int32)
    lens = torch.tensor([13, 16], dtype=torch.int32)
    q = torch.randn(2, 4, 1, 16, generator=g)
    k = torch.stack([torch.cat([pool_k[3], pool_k[1]], 1), torch.cat([pool_k[3], pool_k[4]], 1)])
    v = torch.stack([torch.cat([pool_v[3], pool_v[1]], 1), torch.cat([pool_v[3], pool_v[4]], 1)])
    ref, _ = oracle.gqa(q, k, v, lens, True, 0.25)
    out, _ = oracle.gqa_paged(q, pool_k, pool_v, table, lens, True, 0.25)
    assert np.array_equal(out, ref)


def test_latent_paged_oracle_equals_contiguous():
    inp = synthetic.latent_paged_inputs(64, 2, 16, 1, 16, 32, 8, 2, 2, 40, 8, dtype=torch.float32)
    ref, _ = oracle.latent_absorbed(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                    inp["cache_lens"], True, inp["scale"])
    out, _ = oracle.latent_absorbed_paged(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent_pages"],
                                          inp["block_table"], inp["cache_lens"], True, inp["scale"])
    assert np.array_equal(out, ref)


def test_gta_paged_oracle_equals_contiguous():
    """GTA over shuffled K/V page pools with one block table equals GTA over the contiguous caches."""
    inp = synthetic.gta_paged_inputs(65, 2, 2, 6, 16, 8, 3, 5, 37, 8, dtype=torch.float32)
    ref, ref_lse = oracle.gta(inp["q_g"], inp["k_g"], inp["v"], inp["cache_lens"], True, inp["scale"])
    out, lse = oracle.gta_paged(inp["q_g"], inp["k_pages"], inp["v_pages"], inp["block_table"], inp["cache_lens"],
                                True, inp["scale"])
    assert np.array_equal(out, ref) and np.array_equal(lse, ref_lse)
    assert (inp["block_table"] >= 0).sum() < inp["k_pages"].shape[0]  # spare pages: the pool is not the table


def test_latent_fp8_oracle_is_latent_over_the_dequantised_cache():
    """The fp8 latent oracle equals the latent definition over the cache widened by torch's float8_e4m3fn cast
    and scaled, the latent part and the RoPE key each by its own scale (two different scales)."""
    inp = synthetic.latent_fp8_inputs(66, 2, 16, 1, 16, 32, 8, 2, 5, 30)
    r_kv = 32
    lat = inp["latent8"].to(torch.float64)
    lat[..., :r_kv] *= float(inp["kv_scale"][0])
    lat[..., r_kv:] *= float(inp["kv_scale"][1])
    assert float(inp["kv_scale"][0]) != float(inp["kv_scale"][1])
    ref, ref_lse = oracle.latent_absorbed(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], lat, inp["cache_lens"],
                                          True, inp["scale"])
    out, lse = oracle.latent_absorbed_fp8kv(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent8"],
                                            inp["kv_scale"], inp["cache_lens"], True, inp["scale"])
    assert np.array_equal(out, ref) and np.array_equal(lse, ref_lse)


# ------------------------------------------------------------------ top-k sparse attention ------------------
def test_sparse_oracle_full_selection_equals_dense_causal():
    """Selecting every key a query may see (in a shuffled order) is the dense causal attention ("GQLA ..."
    sections 1-2: sparse GQLA attends over a top-k subset of past keys)."""
    inp = synthetic.latent_inputs(71, 2, 16, 1, 16, 32, 8, 2, 5, 30, dtype=torch.float32)
    idx = synthetic.sparse_indices(72, inp["cache_lens"], 2, 40)  # topk >= every visible count
    ref, ref_lse = oracle.latent_absorbed(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"],
                                          inp["cache_lens"], True, inp["scale"])
    out, lse = oracle.latent_absorbed_sparse(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"], idx,
                                             inp["cache_lens"], inp["scale"])
    assert np.allclose(out, ref, atol=1e-12, rtol=1e-12) and np.allclose(lse, ref_lse, atol=1e-12, rtol=1e-12)


def test_sparse_oracle_subset_equals_dense_over_the_subset_and_skips_junk():
    inp = synthetic.expanded_inputs(73, 2, 32, 2, 16, 8, 1, 10, 30, dtype=torch.float32)
    idx = synthetic.sparse_indices(74, inp["cache_lens"], 1, 6, junk=0.3)
    out, lse = oracle.expanded_sparse(inp["q_c"], inp["q_r"], inp["kc"], inp["vc"], inp["kr"], idx,
                                      inp["cache_lens"], 0.3)
    for b in range(2):
        keys = [int(j) for j in idx[b, 0] if 0 <= j < int(inp["cache_lens"][b])]
        kc, vc, kr = inp["kc"][b:b + 1, :, keys], inp["vc"][b:b + 1, :, keys], inp["kr"][b:b + 1, keys]
        key = torch.cat([kc, kr[:, None].expand(-1, kc.shape[1], -1, -1)], -1)
        val = torch.cat([vc, torch.zeros_like(key[..., vc.shape[-1]:])], -1)
        q = torch.cat([inp["q_c"][b:b + 1], inp["q_r"][b:b + 1]], -1)
        ref, ref_lse = oracle.gqa(q, key, val, torch.tensor([len(keys)], dtype=torch.int32), False, 0.3)
        assert np.allclose(out[b], ref[0, ..., :16], atol=1e-13) and np.allclose(lse[b], ref_lse[0], atol=1e-13)


def test_expanded_sparse_full_selection_equals_latent_definition():
    """GQLA section 3.1: the per-group GQA path over the expanded cache computes the latent attention of eq. (1).
    A selection listing every position a query may see (in a scrambled order, causal, s_q = 2) makes the sparse
    composition the dense per-group path, so expanded_sparse over the caches of latent_expand_cache must equal
    latent_expanded -- eq. (1) evaluated from the latent and the weights, not a restatement of the composition."""
    s_q = 2
    inp = synthetic.latent_inputs(76, 2, 32, 2, 16, 32, 8, s_q, 5, 20, dtype=torch.float32)
    lens = inp["cache_lens"]
    kc, vc, kr = oracle.latent_expand_cache(inp["latent"], inp["w_uk"], inp["w_uv"])
    gen = torch.Generator().manual_seed(77)
    idx = torch.full((2, s_q, int(lens.max())), -1, dtype=torch.int32)
    for b in range(2):
        for t in range(s_q):
            n = int(lens[b]) - s_q + t + 1
            idx[b, t, :n] = torch.randperm(n, generator=gen).to(torch.int32)
    out, lse = oracle.expanded_sparse(inp["q_c"], inp["q_r"], kc, vc, kr, idx, lens, inp["scale"])
    ref, ref_lse = oracle.latent_expanded(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"], lens, True,
                                          inp["scale"])
    assert np.allclose(out, ref, rtol=1e-11, atol=1e-12) and np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_sparse_oracle_empty_selection():
    inp = synthetic.latent_inputs(75, 1, 16, 1, 16, 32, 8, 1, 9, 9, dtype=torch.float32)
    idx = torch.full((1, 1, 4), -1, dtype=torch.int32)
    out, lse = oracle.latent_absorbed_sparse(inp["q_c"], inp["q_r"], inp["w_uk"], inp["w_uv"], inp["latent"], idx,
                                             inp["cache_lens"], inp["scale"])
    assert np.all(out == 0) and np.all(np.isneginf(lse))


# ------------------------------------------------------------------ FP8 (e4m3) KV cache ----------------------
def test_e4m3_decoding_and_fp8_oracle():
    """The oracle's e4m3 decode (bit fields: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals,
    NaN, no infinities) on codes whose values the format fixes, on all 256 codes against torch's float8_e4m3fn
    cast (a second, independent decoder), and the per-KV-head scaling of the fp8 GQA oracle."""
    codes = torch.tensor([0x38, 0x40, 0x01, 0x08, 0x7E, 0xB8, 0x00, 0x3C, 0x07, 0x77, 0x80], dtype=torch.uint8)
    vals = oracle.decode_e4m3(codes).tolist()
    assert vals == [1.0, 2.0, 2.0 ** -9, 2.0 ** -6, 448.0, -1.0, 0.0, 1.5, 7 * 2.0 ** -9, 240.0, -0.0]
    assert math.copysign(1.0, vals[-1]) == -1.0
    allc = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    mine = oracle.decode_e4m3(allc)
    lib = allc.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(lib)) and np.isnan(mine).sum() == 2  # 0x7F and 0xFF
    ok = ~np.isnan(mine)
    assert np.array_equal(mine[ok], lib[ok])
    inp = synthetic.gqa_fp8_inputs(81, 2, 8, 2, 128, 1, 5, 40)
    k = inp["k"].to(torch.float64) * inp["k_scale"].double()[None, :, None, None]
    v = inp["v"].to(torch.float64) * inp["v_scale"].double()[None, :, None, None]
    assert inp["k_scale"][0] != inp["k_scale"][1]
    ref, ref_lse = oracle.gqa(inp["q"], k, v, inp["cache_lens"], True, inp["scale"])
    out, lse = oracle.gqa_fp8kv(inp["q"], inp["k"], inp["v"], inp["k_scale"], inp["v_scale"], inp["cache_lens"], True,
                                inp["scale"])
    assert np.array_equal(out, ref) and np.array_equal(lse, ref_lse)
