"""The C-ABI library: it loads without a GPU, exports every symbol include/lka.h declares, and the
binding's ctypes signatures match the header's parameter lists (CPU only, no compute calls)."""
import ctypes
import os
import re

import pytest

import latent_kv_attention_b200 as lka
from latent_kv_attention_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lka.h")


def declarations():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = {}
    for m in re.finditer(r"LKA_API\s+([\w\s\*]+?)\b(\w+)\s*\(([^;]*?)\)\s*;", text, flags=re.S):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        decls[name] = (ret, n)
    return decls


@pytest.fixture(scope="module")
def lib():
    build.build()
    return lka.library()


def test_header_declares_the_four_entry_points():
    d = declarations()
    for name in ("gqa_attn", "latent_absorbed_attn", "latent_expand_gqa_attn", "gta_shared_score_attn",
                 "latent_expand_cache"):
        assert name in d


def test_library_exports_every_declared_symbol(lib):
    for name in declarations():
        assert hasattr(lib, name), f"liblka.so does not export {name}"


def test_binding_signatures_match_header(lib):
    d = declarations()
    assert set(d) == set(lka.SIGNATURES)
    for name, (ret, n) in d.items():
        assert len(lka.SIGNATURES[name][1]) == n, f"{name}: header has {n} parameters"


def test_status_strings(lib):
    for code, name in lka.STATUS_NAMES.items():
        assert lka.status_string(code) == name
    assert lka.status_string(99) == "LKA_ERR_UNKNOWN"


def test_host_validation_without_gpu(lib):
    # argument errors are caught on the host before anything is enqueued
    P = ctypes.c_void_p
    rc = lib.gqa_attn(P(16), P(16), P(16), P(16), P(16), None, 1, 6, 4, 1, 128, 64, 1, 1.0, 0, P(16), 1 << 20, None)
    assert rc == 1  # h_q % h_kv != 0
    rc = lib.gqa_attn(P(16), P(16), P(16), P(16), P(16), None, 1, 8, 2, 1, 96, 64, 1, 1.0, 0, P(16), 1 << 20, None)
    assert rc == 2  # unsupported head dim
    rc = lib.gqa_attn(P(16), P(16), P(16), P(16), P(16), None, 1, 8, 2, 1, 128, 64, 1, 1.0, 0, None, 0, None)
    assert rc == 3  # no workspace
    rc = lib.gqa_attn(P(18), P(16), P(16), P(16), P(16), None, 1, 8, 2, 1, 128, 64, 1, 1.0, 0, P(16), 1 << 20, None)
    assert rc == 1  # misaligned q
    rc = lib.gqa_attn(None, None, None, None, None, None, 0, 8, 2, 1, 128, 64, 1, 1.0, 0, None, 0, None)
    assert rc == 0  # empty batch is a no-op


def test_workspace_sizes(lib):
    small = lib.gqa_attn_workspace_size(1, 8, 2, 1, 64, 17)
    assert small >= 256
    big = lib.gqa_attn_workspace_size(64, 32, 8, 1, 128, 8192)
    assert big > small
    assert lib.gqa_attn_workspace_size(1, 6, 4, 1, 64, 17) == 0  # invalid grouping


def test_split_knob_roundtrip(lib):
    prev = lka.set_split_tokens(512)
    assert lka.set_split_tokens(prev) == 512


def test_split_knob_is_per_thread(lib):
    """The split knob only changes the plans of calls made from the thread that set it: a caller on another
    thread keeps the automatic plan (the boundary holds no state shared between concurrent callers)."""
    import threading

    auto = lka.gqa_split_count(64, 32, 8, 1, 128, 8192)
    seen = {}

    def other():
        seen["before"] = lka.gqa_split_count(64, 32, 8, 1, 128, 8192)
        lka.set_split_tokens(512)
        seen["set"] = lka.gqa_split_count(64, 32, 8, 1, 128, 8192)

    t = threading.Thread(target=other)
    t.start()
    t.join()
    assert seen == {"before": auto, "set": 16}
    assert lka.gqa_split_count(64, 32, 8, 1, 128, 8192) == auto  # this thread's plan is untouched


def test_gqa_prefill_split_plan(lib):
    """Prefill shapes (bf16, d 128, s_q >= 64) are planned for the tensor-core prefill kernel: one CTA per
    128-query tile and query head; the keys are split only while those CTAs number fewer than two per SM
    (148 SMs), in splits of at least 512 keys (rounded to 128-key tiles)."""
    prev = lka.set_split_tokens(0)
    try:
        assert lka.gqa_split_count(2, 32, 8, 4096, 128, 4096) == 1   # 2048 CTAs already fill the GPU
        assert lka.gqa_split_count(1, 8, 2, 160, 128, 1024) == 2     # 16 CTAs: 512-key splits
        assert lka.gqa_split_count(1, 8, 2, 160, 128, 100000) == 19  # ceil(296 / 16) splits of 5376 keys
        lka.set_split_tokens(128)
        assert lka.gqa_split_count(1, 8, 2, 160, 128, 1024) == 8
        assert lka.gqa_split_count(1, 8, 3, 160, 128, 1024) == 0     # h_q not a multiple of h_kv
    finally:
        lka.set_split_tokens(prev)


def test_gqa_split_plan(lib):
    """The GQA split count chosen by the wave-cost rule (host logic; 148 SMs, two resident CTAs per SM for the
    d_h 128 bf16 kernel): the smallest max(ceil(w), w + 1/4) * (tiles per split + 2) with w = CTAs / 296."""
    prev = lka.set_split_tokens(0)
    try:
        assert lka.gqa_split_count(64, 32, 8, 1, 128, 8192) == 4    # Llama-3.1-8B decode layer, 2048-key splits
        assert lka.gqa_split_count(16, 32, 8, 1, 128, 8192) == 4    # not one long wave of 256 CTAs
        assert lka.gqa_split_count(64, 32, 8, 1, 128, 1024) == 1    # 512 CTAs of 16 tiles
        assert lka.gqa_split_count(64, 32, 8, 1, 128, 4096) == 4
        assert lka.gqa_split_count(64, 32, 8, 1, 128, 65536) == 8
        assert lka.gqa_split_count(1, 8, 2, 1, 64, 17) == 1
        assert lka.gqa_split_count(1, 6, 4, 1, 64, 17) == 0         # invalid grouping
        lka.set_split_tokens(512)
        assert lka.gqa_split_count(64, 32, 8, 1, 128, 8192) == 16   # the knob: splits of at most 512 keys
    finally:
        lka.set_split_tokens(prev)
