"""Head-axis sharding on CPU: the slice arithmetic, and two gloo ranks that each compute their slice of the
heads with the fp64 oracle and gather the outputs (no GPU).  The gathered result must equal the unsharded
oracle exactly, because every head's output depends only on its own group's keys and values."""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from latent_kv_attention_b200 import sharding  # noqa: E402


def test_gqa_slices_cover_the_heads_once():
    for world in (1, 2, 4, 8):
        qs, ks = [], []
        for r in range(world):
            (q0, q1), (k0, k1) = sharding.gqa_head_slice(32, 8, r, world)
            qs += list(range(q0, q1))
            ks += list(range(k0, k1))
            # every query head of the slice uses a KV head of the slice
            assert all(k0 <= i // 4 < k1 for i in range(q0, q1))
        assert qs == list(range(32)) and ks == list(range(8))
    with pytest.raises(ValueError):
        sharding.gqa_head_slice(32, 8, 0, 3)


def test_group_and_gta_slices():
    assert sharding.group_slice(128, 8, 3, 4) == ((96, 128), (6, 8))
    assert sharding.gta_group_slice(3, 12, 1, 3) == ((1, 2), (4, 8))
    with pytest.raises(ValueError):
        sharding.group_slice(128, 8, 0, 16)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import synthetic
        from latent_kv_attention_b200 import sharding as sh

        # GQA by KV head: 16 query heads, 4 KV heads, two ranks of 2 KV heads each
        inp = synthetic.gqa_inputs(71, 2, 16, 4, 64, 2, 20, 50, Lmax=50, dtype=torch.float32)
        (q0, q1), (k0, k1) = sh.gqa_head_slice(16, 4, rank, world)
        out, lse = oracle.gqa(inp["q"][:, q0:q1].contiguous(), inp["k"][:, k0:k1].contiguous(),
                              inp["v"][:, k0:k1].contiguous(), inp["cache_lens"], True, inp["scale"])
        out, lse = torch.from_numpy(out).contiguous(), torch.from_numpy(lse).contiguous()
        outs = [torch.empty_like(out) for _ in range(world)]
        lses = [torch.empty_like(lse) for _ in range(world)]
        torch.distributed.all_gather(outs, out)
        torch.distributed.all_gather(lses, lse)
        q.put((rank, torch.cat(outs, 1), torch.cat(lses, 1)))
    finally:
        torch.distributed.destroy_process_group()


def test_gqa_heads_sharded_over_two_gloo_ranks():
    import oracle
    import synthetic

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {r: (o, l) for r, o, l in (q.get(timeout=120) for _ in procs)}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = synthetic.gqa_inputs(71, 2, 16, 4, 64, 2, 20, 50, Lmax=50, dtype=torch.float32)
    ref, ref_lse = oracle.gqa(inp["q"], inp["k"], inp["v"], inp["cache_lens"], True, inp["scale"])
    for r in (0, 1):
        assert torch.equal(res[r][0], torch.from_numpy(ref))
        assert torch.equal(res[r][1], torch.from_numpy(ref_lse))
