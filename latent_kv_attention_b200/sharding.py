"""Head-axis sharding of the attention calls across devices (host logic only).

Every query head of a group reads only its group's keys and values, so the heads can be split over devices
with no exchange inside the attention: GQA by KV head (each device takes a contiguous block of KV heads and
their h_q / h_kv query heads each), the GQLA per-group path by group ("GQLA: Group-Query Latent Attention ...",
section 1: tensor parallelism along the group axis, up to the number of groups, without duplicated work; the
shared RoPE key is replicated), GTA by head group (the group's query / key and its value heads).  The
MQA-absorbed latent path shares one latent among all heads and cannot be split this way: each device would
hold the whole latent cache (the same section notes that this path must replicate the latent).

Each function returns the half-open ranges [a, b) of the device's slice; the device calls the ordinary entry
point on those slices, and the outputs put side by side along the head axis are the unsharded call's.
"""
from __future__ import annotations


def _check(world: int, rank: int, units: int, what: str):
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if units % world:
        raise ValueError(f"{units} {what} do not split evenly over {world} devices")


def gqa_head_slice(h_q: int, h_kv: int, rank: int, world: int):
    """(query heads [q0, q1), KV heads [k0, k1)) of `rank`: a contiguous block of h_kv / world KV heads and the
    h_q / h_kv query heads of each (query head i uses KV head i // (h_q / h_kv))."""
    if h_q % h_kv:
        raise ValueError("h_q must be a multiple of h_kv")
    _check(world, rank, h_kv, "KV heads")
    per, ratio = h_kv // world, h_q // h_kv
    k0, k1 = per * rank, per * (rank + 1)
    return (ratio * k0, ratio * k1), (k0, k1)


def group_slice(h_q: int, g: int, rank: int, world: int):
    """(query heads [q0, q1), groups [g0, g1)) of `rank` for the GQLA per-group path: g / world groups of
    h_q / g query heads each (kc / vc are sliced by group, the shared RoPE key kr is replicated)."""
    if h_q % g:
        raise ValueError("h_q must be a multiple of g")
    _check(world, rank, g, "groups")
    per, hpg = g // world, h_q // g
    g0, g1 = per * rank, per * (rank + 1)
    return (hpg * g0, hpg * g1), (g0, g1)


def gta_group_slice(G: int, H: int, rank: int, world: int):
    """(groups [g0, g1) of q_g / k_g, heads [h0, h1) of v / out) of `rank` for GTA: G / world groups and their
    H / G value heads each."""
    if H % G:
        raise ValueError("H must be a multiple of G")
    _check(world, rank, G, "groups")
    per, hpg = G // world, H // G
    g0, g1 = per * rank, per * (rank + 1)
    return (g0, g1), (hpg * g0, hpg * g1)
