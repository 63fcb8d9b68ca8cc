"""gqa_attn_noalloc -- the variant of gqa_attn that allocates nothing -- called through the C ABI.

Callers that cannot allocate device memory (a plugin handed only its input and
output buffers, or code where the host framework forbids device allocations)
cannot pass gqa_attn its workspace; gqa_attn_noalloc keeps the split-KV scratch
in a fixed 16 MiB device array inside the library instead.  Its result must
match gqa_attn's within the parity tolerance, on consecutive calls that reuse
the scratch the previous call left behind.  The file name makes pytest collect
it last.
"""
import ctypes

import pytest
import torch

import latent_kv_attention_b200 as lka
import synthetic
from parity import assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def call_noalloc(q, k, v, lens, out, lse, causal, scale):
    B, h_q, s_q, d = q.shape
    h_kv, Lmax = k.shape[1], k.shape[2]
    P = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
    dtype = 0 if q.dtype == torch.bfloat16 else 1
    return lka.library().gqa_attn_noalloc(P(q), P(k), P(v), P(lens), P(out), P(lse), B, h_q, h_kv, s_q, d, Lmax,
                                          int(causal), float(scale), dtype,
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_gqa_attn_on_two_calls_in_a_row():
    for seed, s_q in ((71, 1), (72, 2)):  # the second call reuses the scratch the first one left behind
        inp = synthetic.gqa_inputs(seed, 4, 32, 8, 128, s_q, 300, 2000, Lmax=2048, device=DEV)
        ref, ref_lse = lka.gqa_attn(inp["q"], inp["k"], inp["v"], inp["cache_lens"], causal=True,
                                    scale=inp["scale"], return_lse=True)
        out = torch.empty_like(inp["q"])
        lse = torch.empty(ref_lse.shape, dtype=torch.float32, device=DEV)
        rc = call_noalloc(inp["q"], inp["k"], inp["v"], inp["cache_lens"], out, lse, True, inp["scale"])
        assert rc == 0, lka.status_string(rc)
        torch.cuda.synchronize()
        assert_close(out, ref, torch.bfloat16, f"noalloc call seed {seed}")
        assert (lse - ref_lse).abs().max().item() <= 1e-4


def test_noalloc_rejects_scratch_beyond_16_mib():
    # 128 splits of 64 keys for 2048 query rows need ~134 MB of partials: rejected before any launch
    B, h_q, h_kv, d, Lmax = 64, 32, 8, 128, 8192
    q = torch.zeros(B, h_q, 1, d, dtype=torch.bfloat16, device=DEV)
    k = torch.zeros(B, h_kv, Lmax, d, dtype=torch.bfloat16, device=DEV)
    lens = torch.full((B,), Lmax, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    prev = lka.set_split_tokens(64)
    try:
        rc = call_noalloc(q, k, k, lens, out, None, True, 0.1)
    finally:
        lka.set_split_tokens(prev)
    assert rc == 3  # LKA_ERR_WORKSPACE
