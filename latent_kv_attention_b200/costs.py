"""Algorithmic byte and FLOP counts of the attention paths (host-side arithmetic for the roofline).

These are the counts the roofline fractions are computed from: the bytes an
ideal kernel must move between HBM and the SMs (every cache byte read once,
inputs read once, outputs written once) and the multiply-add work of the
definition (2 FLOPs per multiply-add, causal work counted over visible keys
only).  The pages count arithmetic intensity the same way: the GQLA paper's
"about 242 FLOPs/byte" for the MQA-absorbed path at (h_q, d_h, r_kv, d_h^R) =
(128, 128, 512, 64) and s_q = 1 is 128 * (2*576 + 2*512) FLOPs over 576 * 2
cache bytes per token (section 1).
"""
from __future__ import annotations

from typing import Sequence


def cache_elems_per_token(layout: str, **k) -> int:
    """Cached values per token per layer.

    gqa/mha: 2 * kv_heads * d                    (glossary page, "How GQA shrinks the KV cache")
    latent:  r_kv + d_r                           (GQLA section 1: MQA-absorbed path)
    expanded: 2 * g * d_h + d_r                   (GQLA section 1: GQA path, RoPE key stored once)
    gta:     G * d_qk + H * d_v                   (one key per group, one value per head)
    """
    if layout in ("gqa", "mha", "mqa"):
        return 2 * k["kv_heads"] * k["d"]
    if layout == "latent":
        return k["r_kv"] + k["d_r"]
    if layout == "expanded":
        return 2 * k["g"] * k["d_h"] + k["d_r"]
    if layout == "gta":
        return k["G"] * k["d_qk"] + k["H"] * k["d_v"]
    raise ValueError(layout)


def _visible(L: int, s_q: int, causal: bool) -> int:
    """Sum over the s_q queries of the number of keys each sees (bottom-right causal)."""
    if not causal:
        return s_q * L
    return sum(L - s_q + t + 1 for t in range(s_q))


def gqa_bytes(lens: Sequence[int], h_q: int, h_kv: int, d: int, s_q: int, elem: int = 2, kv_elem: int | None = None) -> int:
    """Cache bytes read once (kv_elem bytes per value, default elem) plus q read and out written (elem bytes)."""
    kv_elem = elem if kv_elem is None else kv_elem
    kv = sum(int(L) for L in lens) * h_kv * 2 * d * kv_elem
    qo = len(lens) * h_q * s_q * d * elem * 2
    return kv + qo


def gqa_flops(lens: Sequence[int], h_q: int, d: int, s_q: int, causal: bool) -> int:
    return sum(_visible(int(L), s_q, causal) for L in lens) * h_q * 4 * d


def latent_bytes(lens: Sequence[int], h_q: int, g: int, d_h: int, r_kv: int, d_r: int, s_q: int,
                 elem: int = 2, cache_elem: int | None = None) -> int:
    """Latent cache read once (cache_elem bytes per value, default elem), both weights, q read, out written."""
    cache = sum(int(L) for L in lens) * (r_kv + d_r) * (elem if cache_elem is None else cache_elem)
    weights = 2 * g * d_h * r_kv * elem
    q = len(lens) * h_q * s_q * (d_h + d_r) * elem
    out = len(lens) * h_q * s_q * d_h * elem
    return cache + weights + q + out


def latent_core_flops(lens: Sequence[int], h_q: int, r_kv: int, d_r: int, s_q: int, causal: bool) -> int:
    """Scores over r_kv + d_r dims and the latent-space weighted sum over r_kv dims."""
    return sum(_visible(int(L), s_q, causal) for L in lens) * h_q * (2 * (r_kv + d_r) + 2 * r_kv)


def latent_proj_flops(B: int, h_q: int, d_h: int, r_kv: int, s_q: int) -> int:
    """W^UK absorption into the query plus the W^UV up-projection of the output."""
    return B * s_q * h_q * 2 * (2 * d_h * r_kv)


def expanded_bytes(lens: Sequence[int], h_q: int, g: int, d_h: int, d_r: int, s_q: int, elem: int = 2) -> int:
    cache = sum(int(L) for L in lens) * (2 * g * d_h + d_r) * elem
    q = len(lens) * h_q * s_q * (d_h + d_r) * elem
    out = len(lens) * h_q * s_q * d_h * elem
    return cache + q + out


def expanded_flops(lens: Sequence[int], h_q: int, d_h: int, d_r: int, s_q: int, causal: bool) -> int:
    return sum(_visible(int(L), s_q, causal) for L in lens) * h_q * (2 * (d_h + d_r) + 2 * d_h)


def gta_bytes(lens: Sequence[int], G: int, H: int, d_qk: int, d_v: int, s_q: int, elem: int = 2) -> int:
    kv = sum(int(L) for L in lens) * (G * d_qk + H * d_v) * elem
    q = len(lens) * G * s_q * d_qk * elem
    out = len(lens) * H * s_q * d_v * elem
    return kv + q + out


def gta_flops(lens: Sequence[int], G: int, H: int, d_qk: int, d_v: int, s_q: int, causal: bool) -> int:
    """One score matrix per group (2*d_qk per visible key) and one weighted sum per head (2*d_v)."""
    return sum(_visible(int(L), s_q, causal) for L in lens) * (G * 2 * d_qk + H * 2 * d_v)


def arithmetic_intensity_per_token(h_q: int, qk_dims: int, v_dims: int, cache_elems: int, s_q: int = 1,
                                   elem: int = 2) -> float:
    """FLOPs per cache byte of one decode step, counted per cached token (s_q query tokens)."""
    return s_q * h_q * (2 * qk_dims + 2 * v_dims) / (cache_elems * elem)
