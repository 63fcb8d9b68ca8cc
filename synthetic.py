"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds no attention arithmetic: it only draws seeded random tensors
with the shapes, dtypes and value distributions of the workloads on the pages
(a Llama-3.1-8B-shaped GQA decode layer, a GQLA/MLA latent decode layer with
(h_q, d_h, r_kv, d_h^R) = (128, 128, 512, 64), a GTA grouped shared-score
prefill).  There is no public dataset behind any of them; the values are
N(0, 1) (or N(0, 1/512) for the latent up-projections), cast to the compute
dtype with round-to-nearest-even.

Both sides of every parity check consume the tensors returned here: the CUDA
library receives them on the device, the oracle receives the same values
widened to float64.

Layouts (row-major, last dimension contiguous):
  GQA      q [B,h_q,s_q,d]   k,v [B,h_kv,Lmax,d]   cache_lens int32 [B]
  latent   q_c [B,h_q,s_q,d_h]  q_r [B,h_q,s_q,d_r]  w_uk,w_uv [g,d_h,r_kv]
           latent [B,Lmax,r_kv+d_r] (c^KV then k^R)
  expanded kc,vc [B,g,Lmax,d_h]  kr [B,Lmax,d_r]
  GTA      q_g [B,G,s_q,d_qk]  k_g [B,G,Lmax,d_qk]  v [B,H,Lmax,d_v]
cache_lens[b] counts the valid tokens of sequence b including the s_q new
query tokens.
"""
from __future__ import annotations

import math

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, g, dtype, device, std: float = 1.0, chunk_elems: int = 1 << 28):
    """N(0, std^2) in `dtype`, drawn in fp32 (in chunks along dim 0 to bound peak memory)."""
    out = torch.empty(shape, dtype=dtype, device=device)
    n0 = shape[0]
    per = max(1, math.prod(shape[1:]))
    step = max(1, chunk_elems // per)
    for s in range(0, n0, step):
        e = min(n0, s + step)
        x = torch.randn((e - s,) + tuple(shape[1:]), generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[s:e].copy_(x)
    return out


def _lens(g, B, lo, hi, device):
    if lo == hi:
        return torch.full((B,), hi, dtype=torch.int32, device=device)
    return torch.randint(lo, hi + 1, (B,), generator=g, device=device, dtype=torch.int64).to(torch.int32)


def gqa_page_example():
    """The glossary page's worked example: seed 0, q (1,8,16,64), k,v (1,2,16,64), fp32 on the CPU,
    drawn in that order; then one decode step continuing the same generator:
    q17 (1,8,1,64), k17, v17 (1,2,1,64)."""
    torch.manual_seed(0)
    q = torch.randn(1, 8, 16, 64)
    k = torch.randn(1, 2, 16, 64)
    v = torch.randn(1, 2, 16, 64)
    q17 = torch.randn(1, 8, 1, 64)
    k17 = torch.randn(1, 2, 1, 64)
    v17 = torch.randn(1, 2, 1, 64)
    return dict(q=q, k=k, v=v, q17=q17, k17=k17, v17=v17)


def gqa_inputs(seed, B, h_q, h_kv, d, s_q, L_lo, L_hi, Lmax=None, dtype=torch.bfloat16, device="cpu"):
    """GQA decode/prefill inputs; cache lengths uniform in [L_lo, L_hi] (inclusive)."""
    Lmax = L_hi if Lmax is None else Lmax
    g = _gen(seed, device)
    lens = _lens(g, B, L_lo, L_hi, device)
    q = _randn((B, h_q, s_q, d), g, dtype, device)
    k = _randn((B, h_kv, Lmax, d), g, dtype, device)
    v = _randn((B, h_kv, Lmax, d), g, dtype, device)
    return dict(q=q, k=k, v=v, cache_lens=lens, scale=1.0 / math.sqrt(d))


def gqa_fp8_inputs(seed, B, h_q, h_kv, d, s_q, L_lo, L_hi, Lmax=None, device="cpu"):
    """GQA inputs with an e4m3 K/V cache: q bf16 N(0,1); K, V drawn N(0,1) in fp32 and stored as e4m3 with one
    scale per KV head (the head's max |value| / 448, so the largest value maps to e4m3's largest); the scales are
    returned alongside (K = k_scale[h] * k)."""
    Lmax = L_hi if Lmax is None else Lmax
    g = _gen(seed, device)
    lens = _lens(g, B, L_lo, L_hi, device)
    q = _randn((B, h_q, s_q, d), g, torch.bfloat16, device)
    out = dict(q=q, cache_lens=lens, scale=1.0 / math.sqrt(d))
    for name in ("k", "v"):
        x = torch.randn((B, h_kv, Lmax, d), generator=g, device=device, dtype=torch.float32)
        sc = x.abs().amax(dim=(0, 2, 3)).clamp_min(1e-12) / 448.0
        out[name] = (x / sc[None, :, None, None]).to(torch.float8_e4m3fn)
        out[name + "_scale"] = sc.contiguous()
    return out


def latent_fp8_inputs(seed, B, h_q, g_groups, d_h, r_kv, d_r, s_q, L_lo, L_hi, Lmax=None, device="cpu"):
    """GQLA latent inputs (as latent_inputs, bf16 queries and weights) with the latent cache drawn N(0,1) in fp32 and
    stored as e4m3 with one scale for the latent part and one for the RoPE key (each part's max |value| / 448);
    kv_scale = [scale of c^KV, scale of k^R] (c^KV = kv_scale[0] * latent8[..., :r_kv])."""
    inp = latent_inputs(seed, B, h_q, g_groups, d_h, r_kv, d_r, s_q, L_lo, L_hi, Lmax=Lmax, device=device)
    g = _gen(seed + 104729, device)
    x = torch.randn(inp["latent"].shape, generator=g, device=device, dtype=torch.float32)
    sc = torch.stack([x[..., :r_kv].abs().amax(), x[..., r_kv:].abs().amax()]).clamp_min(1e-12) / 448.0
    widths = torch.cat([sc[0].expand(r_kv), sc[1].expand(d_r)])
    inp["latent8"] = (x / widths).to(torch.float8_e4m3fn)
    inp["kv_scale"] = sc.contiguous()
    del inp["latent"]
    return inp


def to_pages(caches, lens, page_size, gen, spare_pages=0):
    """Scatters contiguous caches [B, heads, Lmax, width] (e.g. K and V) into shuffled page pools [num_pages, heads,
    page_size, width] sharing one block table [B, Lmax / page_size] (int32): the pages a sequence uses
    (ceil(len / page_size)) go to slots of a random permutation of the pool; its unused table entries are -1 and
    unused pool slots hold random values.  Layout only: no attention arithmetic."""
    B, h_kv, Lmax, d = caches[0].shape
    assert Lmax % page_size == 0
    max_pages = Lmax // page_size
    num_pages = B * max_pages + spare_pages
    dev = caches[0].device
    perm = torch.randperm(num_pages, generator=gen, device=dev).tolist()
    pools = [torch.randn((num_pages, c.shape[1], page_size, c.shape[3]), generator=gen, device=dev,
                         dtype=torch.float32).to(c.dtype) for c in caches]
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    lens_l = lens.tolist()
    for b in range(B):
        used = -(-int(lens_l[b]) // page_size)
        for j in range(used):
            slot = perm[b * max_pages + j]
            table[b, j] = slot
            for pool, c in zip(pools, caches):
                pool[slot] = c[b, :, j * page_size:(j + 1) * page_size, :]
    return pools, table.to(dev)


def gqa_paged_inputs(seed, B, h_q, h_kv, d, s_q, L_lo, L_hi, page_size, Lmax=None, dtype=torch.bfloat16,
                     device="cpu", spare_pages=3):
    """GQA inputs (as gqa_inputs) with the K/V cache moved into shuffled page pools and a block table; the
    capacity Lmax (default L_hi) is rounded up to whole pages."""
    Lmax = L_hi if Lmax is None else Lmax
    Lmax = -(-Lmax // page_size) * page_size
    inp = gqa_inputs(seed, B, h_q, h_kv, d, s_q, L_lo, L_hi, Lmax=Lmax, dtype=dtype, device=device)
    g = _gen(seed + 7919, device)
    (k_pages, v_pages), table = to_pages([inp["k"], inp["v"]], inp["cache_lens"], page_size, g, spare_pages)
    inp.update(k_pages=k_pages, v_pages=v_pages, block_table=table, page_size=page_size)
    return inp


def gta_paged_inputs(seed, B, G, H, d_qk, d_v, s_q, L_lo, L_hi, page_size, Lmax=None, dtype=torch.bfloat16,
                     device="cpu", spare_pages=3):
    """GTA inputs (as gta_inputs) with k_g and v moved into shuffled page pools sharing one block table; the
    capacity is rounded up to whole pages."""
    Lmax = L_hi if Lmax is None else Lmax
    Lmax = -(-Lmax // page_size) * page_size
    inp = gta_inputs(seed, B, G, H, d_qk, d_v, s_q, L_lo, L_hi, Lmax=Lmax, dtype=dtype, device=device)
    g = _gen(seed + 7919, device)
    (k_pages, v_pages), table = to_pages([inp["k_g"], inp["v"]], inp["cache_lens"], page_size, g, spare_pages)
    inp.update(k_pages=k_pages, v_pages=v_pages, block_table=table, page_size=page_size)
    return inp


def latent_paged_inputs(seed, B, h_q, g_groups, d_h, r_kv, d_r, s_q, L_lo, L_hi, page_size, Lmax=None,
                        dtype=torch.bfloat16, device="cpu", spare_pages=3):
    """GQLA latent inputs (as latent_inputs) with the latent cache moved into a shuffled page pool
    [num_pages, page_size, r_kv + d_r] and a block table; the capacity is rounded up to whole pages."""
    Lmax = L_hi if Lmax is None else Lmax
    Lmax = -(-Lmax // page_size) * page_size
    inp = latent_inputs(seed, B, h_q, g_groups, d_h, r_kv, d_r, s_q, L_lo, L_hi, Lmax=Lmax, dtype=dtype,
                        device=device)
    g = _gen(seed + 7919, device)
    (pool,), table = to_pages([inp["latent"][:, None]], inp["cache_lens"], page_size, g, spare_pages)
    inp.update(latent_pages=pool[:, 0].contiguous(), block_table=table, page_size=page_size)
    return inp


def latent_inputs(seed, B, h_q, g_groups, d_h, r_kv, d_r, s_q, L_lo, L_hi, Lmax=None, dtype=torch.bfloat16,
                  device="cpu"):
    """GQLA latent decode inputs: c^KV, k^R, q^C, q^R ~ N(0,1); W^UK, W^UV ~ N(0, 1/r_kv)."""
    Lmax = L_hi if Lmax is None else Lmax
    g = _gen(seed, device)
    lens = _lens(g, B, L_lo, L_hi, device)
    q_c = _randn((B, h_q, s_q, d_h), g, dtype, device)
    q_r = _randn((B, h_q, s_q, d_r), g, dtype, device)
    w_std = 1.0 / math.sqrt(r_kv)
    w_uk = _randn((g_groups, d_h, r_kv), g, dtype, device, std=w_std)
    w_uv = _randn((g_groups, d_h, r_kv), g, dtype, device, std=w_std)
    latent = _randn((B, Lmax, r_kv + d_r), g, dtype, device)
    return dict(q_c=q_c, q_r=q_r, w_uk=w_uk, w_uv=w_uv, latent=latent, cache_lens=lens,
                scale=1.0 / math.sqrt(d_h + d_r))


def expanded_inputs(seed, B, h_q, g_groups, d_h, d_r, s_q, L_lo, L_hi, Lmax=None, dtype=torch.bfloat16,
                    device="cpu"):
    """Inputs of the expanded (per-group GQA) latent path drawn directly: kc, vc, kr ~ N(0,1)."""
    Lmax = L_hi if Lmax is None else Lmax
    g = _gen(seed, device)
    lens = _lens(g, B, L_lo, L_hi, device)
    q_c = _randn((B, h_q, s_q, d_h), g, dtype, device)
    q_r = _randn((B, h_q, s_q, d_r), g, dtype, device)
    kc = _randn((B, g_groups, Lmax, d_h), g, dtype, device)
    vc = _randn((B, g_groups, Lmax, d_h), g, dtype, device)
    kr = _randn((B, Lmax, d_r), g, dtype, device)
    return dict(q_c=q_c, q_r=q_r, kc=kc, vc=vc, kr=kr, cache_lens=lens, scale=1.0 / math.sqrt(d_h + d_r))


def expanded_paged_inputs(seed, B, h_q, g_groups, d_h, d_r, s_q, L_lo, L_hi, page_size, Lmax=None,
                          dtype=torch.bfloat16, device="cpu", spare_pages=3):
    """Expanded-path inputs (as expanded_inputs) with kc, vc and kr moved into shuffled page pools sharing one
    block table; the capacity is rounded up to whole pages."""
    Lmax = L_hi if Lmax is None else Lmax
    Lmax = -(-Lmax // page_size) * page_size
    inp = expanded_inputs(seed, B, h_q, g_groups, d_h, d_r, s_q, L_lo, L_hi, Lmax=Lmax, dtype=dtype, device=device)
    g = _gen(seed + 7919, device)
    (kc_p, vc_p, kr_p), table = to_pages([inp["kc"], inp["vc"], inp["kr"][:, None]], inp["cache_lens"], page_size, g,
                                         spare_pages)
    inp.update(kc_pages=kc_p, vc_pages=vc_p, kr_pages=kr_p[:, 0].contiguous(), block_table=table,
               page_size=page_size)
    return inp


def sparse_indices(seed, cache_lens, s_q, topk, device="cpu", junk=0.0):
    """Top-k selections for sparse attention: int32 [B, s_q, topk]; for query t of sequence b, distinct positions
    drawn uniformly from the keys it may see ([0, L_b - s_q + t]), in random order, padded with -1 when fewer
    are visible.  A fraction `junk` of the entries is replaced by positions the query may not see (beyond its
    causal limit) or -1, which the attention must skip."""
    g = _gen(seed, "cpu")
    lens = cache_lens.cpu().tolist()
    B = len(lens)
    out = torch.full((B, s_q, topk), -1, dtype=torch.int32)
    for b in range(B):
        for t in range(s_q):
            vis = int(lens[b]) - s_q + t + 1
            n = min(topk, vis)
            out[b, t, :n] = torch.randperm(vis, generator=g)[:n].to(torch.int32)
            if junk > 0:
                bad = torch.rand(topk, generator=g) < junk
                beyond = torch.randint(vis, vis + 50, (topk,), generator=g, dtype=torch.int32)
                out[b, t] = torch.where(bad, torch.where(torch.rand(topk, generator=g) < 0.5, beyond,
                                                         torch.full_like(beyond, -1)), out[b, t])
    return out.to(device)


def gta_inputs(seed, B, G, H, d_qk, d_v, s_q, L_lo, L_hi, Lmax=None, dtype=torch.bfloat16, device="cpu"):
    """GTA shared-score inputs, all N(0,1). For prefill pass s_q == L_lo == L_hi."""
    Lmax = L_hi if Lmax is None else Lmax
    g = _gen(seed, device)
    lens = _lens(g, B, L_lo, L_hi, device)
    q_g = _randn((B, G, s_q, d_qk), g, dtype, device)
    k_g = _randn((B, G, Lmax, d_qk), g, dtype, device)
    v = _randn((B, H, Lmax, d_v), g, dtype, device)
    return dict(q_g=q_g, k_g=k_g, v=v, cache_lens=lens, scale=1.0 / math.sqrt(d_qk))


# The five workloads, by name.  Sizes follow the pages' layer shapes.
WORKLOADS = {
    "gqa_decode_llama8b": dict(kind="gqa", seed=2, B=64, h_q=32, h_kv=8, d=128, s_q=1, L_lo=1024, L_hi=8192,
                               causal=True),
    # the same layer with a quarter of the batch: the small case for full ncu captures (K/V still > L2)
    "gqa_decode_llama8b_b16": dict(kind="gqa", seed=2, B=16, h_q=32, h_kv=8, d=128, s_q=1, L_lo=1024, L_hi=8192,
                                   causal=True),
    # the same layer with an e4m3 cache (one scale per KV head)
    "gqa_decode_llama8b_fp8": dict(kind="gqa_fp8", seed=2, B=64, h_q=32, h_kv=8, d=128, s_q=1, L_lo=1024,
                                   L_hi=8192, causal=True),
    # the same layer over a paged cache: 64-token pages in a shuffled pool, addressed through a block table
    "gqa_decode_llama8b_paged": dict(kind="gqa_paged", seed=2, B=64, h_q=32, h_kv=8, d=128, s_q=1, L_lo=1024,
                                     L_hi=8192, causal=True, page_size=64),
    # causal prefill of the same layer: 4096 query tokens per sequence over their own 4096-token cache
    "gqa_prefill_llama8b_4k": dict(kind="gqa", seed=6, B=2, h_q=32, h_kv=8, d=128, s_q=4096, L_lo=4096, L_hi=4096,
                                   causal=True),
    # a small case of the same layer for profiler captures (the full prefill holds ~300 MB)
    "gqa_prefill_llama8b_2k_b1": dict(kind="gqa", seed=6, B=1, h_q=32, h_kv=8, d=128, s_q=2048, L_lo=2048, L_hi=2048,
                                      causal=True),
    "gta_prefill_4k": dict(kind="gta", seed=3, B=8, G=3, H=12, d_qk=64, d_v=64, s_q=4096, L_lo=4096,
                           L_hi=4096, causal=True),
    "latent_decode_4k_sq1": dict(kind="latent", seed=4, B=64, h_q=128, g=8, d_h=128, r_kv=512, d_r=64, s_q=1,
                                 L_lo=4096, L_hi=4096, causal=True),
    "latent_decode_4k_sq2": dict(kind="latent", seed=4, B=64, h_q=128, g=8, d_h=128, r_kv=512, d_r=64, s_q=2,
                                 L_lo=4096, L_hi=4096, causal=True),
    # the s_q = 1 layer over a paged latent cache (64-token pages, shuffled pool, block table)
    "latent_decode_4k_sq1_paged": dict(kind="latent_paged", seed=4, B=64, h_q=128, g=8, d_h=128, r_kv=512, d_r=64,
                                       s_q=1, L_lo=4096, L_hi=4096, causal=True, page_size=64),
    # the same layer with the latent cache in e4m3 (one scale for c^KV, one for k^R)
    "latent_decode_4k_sq1_fp8": dict(kind="latent_fp8", seed=4, B=64, h_q=128, g=8, d_h=128, r_kv=512, d_r=64,
                                     s_q=1, L_lo=4096, L_hi=4096, causal=True),
    # top-k sparse decode: 2048 of the 16K cached tokens per query, selected uniformly at random
    "latent_sparse_16k_top2048": dict(kind="latent_sparse", seed=8, B=64, h_q=128, g=8, d_h=128, r_kv=512, d_r=64,
                                      s_q=1, L_lo=16384, L_hi=16384, causal=True, topk=2048),
    # half the batch: the small case for full ncu captures of the latent kernels (latent cache 151 MB > L2)
    "latent_decode_4k_sq1_b32": dict(kind="latent", seed=4, B=32, h_q=128, g=8, d_h=128, r_kv=512, d_r=64, s_q=1,
                                     L_lo=4096, L_hi=4096, causal=True),
    "latent_expanded_4k_sq2_b16": dict(kind="latent", seed=4, B=16, h_q=128, g=8, d_h=128, r_kv=512, d_r=64, s_q=2,
                                       L_lo=4096, L_hi=4096, causal=True),
    # chunked prefill against a paged cache: the last 1024 tokens of each 4096-token sequence as queries, the
    # keys/values in 64-token pages of a shuffled pool
    "gta_chunked_prefill_4k_paged": dict(kind="gta_paged", seed=3, B=8, G=3, H=12, d_qk=64, d_v=64, s_q=1024,
                                         L_lo=4096, L_hi=4096, causal=True, page_size=64),
    "gta_prefill_4k_b2": dict(kind="gta", seed=3, B=2, G=3, H=12, d_qk=64, d_v=64, s_q=4096, L_lo=4096, L_hi=4096,
                              causal=True),
    # the same latent inputs, run through the per-group GQA path after the one-time cache expansion
    "latent_expanded_4k_sq1": dict(kind="latent", seed=4, B=64, h_q=128, g=8, d_h=128, r_kv=512, d_r=64, s_q=1,
                                   L_lo=4096, L_hi=4096, causal=True),
    "latent_expanded_4k_sq2": dict(kind="latent", seed=4, B=64, h_q=128, g=8, d_h=128, r_kv=512, d_r=64, s_q=2,
                                   L_lo=4096, L_hi=4096, causal=True),
}


def sweep_workload(kind: str, L: int) -> dict:
    """Long-context sweep points: batch 64, s_q 1, equal cache length L for every sequence."""
    if kind == "gqa":
        return dict(kind="gqa", seed=5, B=64, h_q=32, h_kv=8, d=128, s_q=1, L_lo=L, L_hi=L, causal=True)
    return dict(kind="latent", seed=5, B=64, h_q=128, g=8, d_h=128, r_kv=512, d_r=64, s_q=1, L_lo=L, L_hi=L,
                causal=True)


# The long-context decode sweep: batch 64, s_q 1, cache length 1K ... 64K tokens for every sequence, over the
# GQA layout (32 query / 8 KV heads, d_h 128) and the latent layout (128 heads, 512 + 64 latent values).
SWEEP_LENGTHS = (1024, 2048, 4096, 8192, 16384, 32768, 65536)
SWEEP = {f"{kind}_sweep_{L // 1024}k": sweep_workload(kind, L) for kind in ("gqa", "latent") for L in SWEEP_LENGTHS}
WORKLOADS.update(SWEEP)


def make(w: dict, device="cpu", dtype=torch.bfloat16) -> dict:
    """Materialise a workload description from WORKLOADS / sweep_workload."""
    if w["kind"] == "gqa":
        return gqa_inputs(w["seed"], w["B"], w["h_q"], w["h_kv"], w["d"], w["s_q"], w["L_lo"], w["L_hi"],
                          dtype=dtype, device=device)
    if w["kind"] == "gqa_fp8":
        return gqa_fp8_inputs(w["seed"], w["B"], w["h_q"], w["h_kv"], w["d"], w["s_q"], w["L_lo"], w["L_hi"],
                              device=device)
    if w["kind"] == "gqa_paged":
        return gqa_paged_inputs(w["seed"], w["B"], w["h_q"], w["h_kv"], w["d"], w["s_q"], w["L_lo"], w["L_hi"],
                                w["page_size"], dtype=dtype, device=device)
    if w["kind"] == "latent_paged":
        return latent_paged_inputs(w["seed"], w["B"], w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"],
                                   w["L_lo"], w["L_hi"], w["page_size"], dtype=dtype, device=device)
    if w["kind"] == "latent_fp8":
        return latent_fp8_inputs(w["seed"], w["B"], w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"],
                                 w["L_lo"], w["L_hi"], device=device)
    if w["kind"] == "latent_sparse":
        inp = latent_inputs(w["seed"], w["B"], w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"],
                            w["L_lo"], w["L_hi"], dtype=dtype, device=device)
        inp["indices"] = sparse_indices(w["seed"] + 1, inp["cache_lens"], w["s_q"], w["topk"], device=device)
        return inp
    if w["kind"] == "latent":
        return latent_inputs(w["seed"], w["B"], w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"],
                             w["L_lo"], w["L_hi"], dtype=dtype, device=device)
    if w["kind"] == "gta_paged":
        return gta_paged_inputs(w["seed"], w["B"], w["G"], w["H"], w["d_qk"], w["d_v"], w["s_q"], w["L_lo"],
                                w["L_hi"], w["page_size"], dtype=dtype, device=device)
    if w["kind"] == "gta":
        return gta_inputs(w["seed"], w["B"], w["G"], w["H"], w["d_qk"], w["d_v"], w["s_q"], w["L_lo"], w["L_hi"],
                          dtype=dtype, device=device)
    raise ValueError(w["kind"])
