"""gqa_attn_noalloc -- the variant of gqa_attn that allocates nothing -- called through the C ABI.

Callers that cannot allocate device memory (a plugin handed only its input and
output buffers, or code where the host framework forbids device allocations)
cannot pass gqa_attn its workspace; gqa_attn_noalloc keeps the split-KV scratch
in a fixed 16 MiB device array inside the library instead.  Its result must
match the fp64 oracle within the parity tolerance, and gqa_attn's, on
consecutive calls that reuse the scratch the previous call left behind; its
device-side flags are read back through gqa_attn_noalloc_status.  The file
name makes pytest collect it last.
"""
import ctypes

import pytest
import torch

import latent_kv_attention_b200 as lka
import oracle
import synthetic
from parity import assert_close, assert_lse_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def call_noalloc(q, k, v, lens, out, lse, causal, scale):
    B, h_q, s_q, d = q.shape
    h_kv, Lmax = k.shape[1], k.shape[2]
    P = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None  # noqa: E731
    dtype = 0 if q.dtype == torch.bfloat16 else 1
    return lka.library().gqa_attn_noalloc(P(q), P(k), P(v), P(lens), P(out), P(lse), B, h_q, h_kv, s_q, d, Lmax,
                                          int(causal), float(scale), dtype, _stream())


def noalloc_status():
    return lka.library().gqa_attn_noalloc_status(_stream())


def test_noalloc_matches_oracle_and_gqa_attn_on_two_calls_in_a_row():
    noalloc_status()  # start from a clear status word
    for seed, s_q in ((71, 1), (72, 2)):  # the second call reuses the scratch the first one left behind
        inp = synthetic.gqa_inputs(seed, 4, 32, 8, 128, s_q, 300, 2000, Lmax=2048)
        # the call is split along the keys, so the scratch's partials are written and merged
        assert lka.gqa_split_count(4, 32, 8, s_q, 128, 2048) > 1
        q, k, v, lens = (inp[n].to(DEV) for n in ("q", "k", "v", "cache_lens"))
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
        rc = call_noalloc(q, k, v, lens, out, lse, True, inp["scale"])
        assert rc == 0, lka.status_string(rc)
        torch.cuda.synchronize()
        ref, ref_lse = oracle.gqa(inp["q"], inp["k"], inp["v"], inp["cache_lens"], True, inp["scale"])
        assert_close(out, ref, torch.bfloat16, f"noalloc call seed {seed} vs oracle")
        assert_lse_close(lse, ref_lse, torch.bfloat16, f"noalloc lse seed {seed} vs oracle")
        ws_out, ws_lse = lka.gqa_attn(q, k, v, lens, causal=True, scale=inp["scale"], return_lse=True)
        assert_close(out, ws_out, torch.bfloat16, f"noalloc call seed {seed} vs gqa_attn")
        assert (lse - ws_lse).abs().max().item() <= 1e-4
    assert noalloc_status() == 0


def test_noalloc_reports_a_clamped_length_through_its_status():
    noalloc_status()
    inp = synthetic.gqa_inputs(73, 2, 32, 8, 128, 1, 100, 400, Lmax=512)
    lens = inp["cache_lens"].clone()
    lens[1] = 100000  # beyond Lmax: clamped to Lmax on the device and flagged
    q, k, v = (inp[n].to(DEV) for n in ("q", "k", "v"))
    out = torch.empty_like(q)
    rc = call_noalloc(q, k, v, lens.to(DEV), out, None, True, inp["scale"])
    assert rc == 0  # the device-side clamp cannot be reported by the launch itself
    assert noalloc_status() == 6  # LKA_ERR_BAD_LENGTH, then cleared
    assert noalloc_status() == 0
    # the clamped sequence attends over all Lmax keys
    lens[1] = 512
    ref, _ = oracle.gqa(inp["q"], inp["k"], inp["v"], lens, True, inp["scale"])
    assert_close(out, ref, torch.bfloat16, "noalloc with a clamped length")


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
