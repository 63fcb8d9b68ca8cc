"""Head-axis sharding of the attention calls (marked gpu).

The pages name tensor parallelism along the group axis as the way to spread GQLA's per-group GQA path over
up to 8 devices without duplicated work ("GQLA: Group-Query Latent Attention ...", section 1), and the same
split applies to GQA by KV head and to GTA by head group: every group's heads only read that group's keys
and values, so no exchange is needed inside the attention.  A device then runs the ordinary entry point on
its slice of the heads.  These tests run the slices one after the other on one GPU and check that their
outputs, put side by side, are bit-identical to the unsharded call (the split plan is pinned so that every
(sequence, head) sees the same key splits in both calls)."""
import pytest
import torch

import latent_kv_attention_b200 as lka
import synthetic

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _pinned_splits():
    lka.clear_status()
    prev = lka.set_split_tokens(512)
    yield
    lka.set_split_tokens(prev)
    assert lka.device_status() == 0, lka.status_string(lka.device_status())


def _slice(t, dim, a, b):
    return t.narrow(dim, a, b - a).contiguous()


@pytest.mark.parametrize("world", [2, 4, 8])
def test_gqa_sharded_by_kv_head(world):
    inp = synthetic.gqa_inputs(61, 4, 32, 8, 128, 1, 300, 2000, Lmax=2048, device=DEV)
    full, full_lse = lka.gqa_attn(inp["q"], inp["k"], inp["v"], inp["cache_lens"], scale=inp["scale"],
                                  return_lse=True)
    per = 8 // world  # KV heads per device; its query heads are the contiguous block of 4 * per
    outs, lses = [], []
    for r in range(world):
        o, l = lka.gqa_attn(_slice(inp["q"], 1, 4 * per * r, 4 * per * (r + 1)),
                            _slice(inp["k"], 1, per * r, per * (r + 1)), _slice(inp["v"], 1, per * r, per * (r + 1)),
                            inp["cache_lens"], scale=inp["scale"], return_lse=True)
        outs.append(o)
        lses.append(l)
    assert torch.equal(torch.cat(outs, 1), full)
    assert torch.equal(torch.cat(lses, 1), full_lse)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_expanded_path_sharded_by_group(world):
    inp = synthetic.expanded_inputs(62, 3, 128, 8, 128, 64, 2, 200, 900, Lmax=900, device=DEV)
    full = lka.latent_expand_gqa_attn(inp["q_c"], inp["q_r"], inp["kc"], inp["vc"], inp["kr"], inp["cache_lens"],
                                      scale=inp["scale"])
    per = 8 // world  # groups per device, 16 query heads each; the RoPE key is replicated
    outs = []
    for r in range(world):
        g0, g1 = per * r, per * (r + 1)
        outs.append(lka.latent_expand_gqa_attn(
            _slice(inp["q_c"], 1, 16 * g0, 16 * g1), _slice(inp["q_r"], 1, 16 * g0, 16 * g1),
            _slice(inp["kc"], 1, g0, g1), _slice(inp["vc"], 1, g0, g1), inp["kr"], inp["cache_lens"],
            scale=inp["scale"]))
    assert torch.equal(torch.cat(outs, 1), full)


def test_gta_sharded_by_group():
    inp = synthetic.gta_inputs(63, 2, 3, 12, 64, 64, 1, 700, 1500, device=DEV)
    full, full_lse = lka.gta_shared_score_attn(inp["q_g"], inp["k_g"], inp["v"], inp["cache_lens"],
                                               scale=inp["scale"], return_lse=True)
    outs, lses = [], []
    for grp in range(3):  # one group (and its 4 value heads) per device
        o, l = lka.gta_shared_score_attn(_slice(inp["q_g"], 1, grp, grp + 1), _slice(inp["k_g"], 1, grp, grp + 1),
                                         _slice(inp["v"], 1, 4 * grp, 4 * grp + 4), inp["cache_lens"],
                                         scale=inp["scale"], return_lse=True)
        outs.append(o)
        lses.append(l)
    assert torch.equal(torch.cat(outs, 1), full)
    assert torch.equal(torch.cat(lses, 1), full_lse)
