"""latent_kv_attention_b200 -- grouped / latent-KV attention on NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in include/lka.h (liblka.so, built from
csrc/).  Every function here only marshals arguments: it checks tensor
devices, dtypes and shapes, allocates outputs and the per-stream workspace with
torch, and passes raw pointers and sizes to the library on the current CUDA
stream.  All arithmetic runs in the library's kernels; there is no CPU or
PyTorch fallback -- if liblka.so is missing or a call fails, an exception is
raised.

Entry points (same names as the C ABI):
  gqa_attn                 GQA decode / prefill          ("Grouped Query Attention (GQA)" glossary page)
  gqa_attn_paged           the same over a paged KV cache (glossary page: PagedAttention comparison)
  gqa_attn_fp8kv           the same over an e4m3 KV cache with per-KV-head scales (GQLA paper, sec. 2)
  latent_absorbed_attn     GQLA MQA-absorbed latent path (GQLA paper, sec. 3.1, Figure 2(b))
  latent_absorbed_attn_paged / _fp8kv / _sparse   ... over a paged, an e4m3, or a top-k selected latent cache
  latent_expand_gqa_attn   GQLA per-group GQA path       (GQLA paper, sec. 3.1, Figure 2(a))
  latent_expand_gqa_attn_paged / _sparse           ... over paged or top-k selected expanded caches
  gta_shared_score_attn    GTA shared score per group    (GTA article, grouped shared attention matrix)
  gta_shared_score_attn_paged  the same over paged K/V pools (chunked prefill against a paged cache)
  latent_expand_cache      one-time latent -> expanded cache conversion (GQLA paper, sec. 3.1)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

from . import costs  # noqa: F401  (host-side byte/FLOP counters)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblka.so")

LKA_OK = 0
STATUS_NAMES = {0: "LKA_OK", 1: "LKA_ERR_INVALID_ARG", 2: "LKA_ERR_UNSUPPORTED", 3: "LKA_ERR_WORKSPACE",
                4: "LKA_ERR_CUDA", 5: "LKA_ERR_TIMEOUT", 6: "LKA_ERR_BAD_LENGTH", 7: "LKA_ERR_BAD_PAGE", 8: "LKA_ERR_RANGE"}
_DT = {torch.bfloat16: 0, torch.float32: 1}

# Every symbol include/lka.h declares, with its ctypes signature (restype, argtypes).
_P, _Z, _I, _F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
_FP = ctypes.POINTER(ctypes.c_float)
SIGNATURES = {
    "gqa_attn_workspace_size": (_Z, [_I] * 6),
    "gqa_attn_split_count": (_I, [_I] * 7),
    "gqa_attn": (_I, [_P] * 6 + [_I] * 7 + [_F, _I, _P, _Z, _P]),
    "gqa_attn_noalloc": (_I, [_P] * 6 + [_I] * 7 + [_F, _I, _P]),
    "gqa_attn_noalloc_status": (_I, [_P]),
    "gqa_attn_fp8kv_workspace_size": (_Z, [_I] * 6),
    "gqa_attn_fp8kv": (_I, [_P] * 8 + [_I] * 7 + [_F, _P, _Z, _P]),
    "gqa_attn_paged_workspace_size": (_Z, [_I] * 7),
    "gqa_attn_paged": (_I, [_P] * 7 + [_I] * 9 + [_F, _I, _P, _Z, _P]),
    "latent_absorbed_attn_workspace_size": (_Z, [_I] * 8),
    "latent_absorbed_attn": (_I, [_P] * 8 + [_I] * 9 + [_F, _I, _P, _Z, _P]),
    "latent_absorbed_attn_fp8kv_workspace_size": (_Z, [_I] * 8),
    "latent_absorbed_attn_fp8kv": (_I, [_P] * 9 + [_I] * 9 + [_F, _P, _Z, _P]),
    "latent_absorbed_attn_paged_workspace_size": (_Z, [_I] * 9),
    "latent_absorbed_attn_paged": (_I, [_P] * 9 + [_I] * 11 + [_F, _I, _P, _Z, _P]),
    "latent_expand_gqa_attn_workspace_size": (_Z, [_I] * 7),
    "latent_expand_gqa_attn": (_I, [_P] * 8 + [_I] * 8 + [_F, _I, _P, _Z, _P]),
    "latent_expand_gqa_attn_paged_workspace_size": (_Z, [_I] * 8),
    "latent_absorbed_attn_sparse_workspace_size": (_Z, [_I] * 8),
    "latent_absorbed_attn_sparse": (_I, [_P] * 9 + [_I] * 9 + [_F, _I, _P, _Z, _P]),
    "latent_expand_gqa_attn_sparse_workspace_size": (_Z, [_I] * 7),
    "latent_expand_gqa_attn_sparse": (_I, [_P] * 9 + [_I] * 8 + [_F, _I, _P, _Z, _P]),
    "latent_expand_gqa_attn_paged": (_I, [_P] * 9 + [_I] * 10 + [_F, _I, _P, _Z, _P]),
    "gta_shared_score_attn_workspace_size": (_Z, [_I] * 7),
    "gta_shared_score_attn": (_I, [_P] * 6 + [_I] * 8 + [_F, _I, _P, _Z, _P]),
    "gta_shared_score_attn_paged_workspace_size": (_Z, [_I] * 8),
    "gta_shared_score_attn_paged": (_I, [_P] * 7 + [_I] * 10 + [_F, _I, _P, _Z, _P]),
    "latent_expand_cache": (_I, [_P] * 3 + [_I] * 6 + [_P] * 3 + [_I, _P]),
    "lka_device_status": (_I, [_P, _P]),
    "lka_clear_status": (_I, [_P, _P]),
    "lka_status_string": (ctypes.c_char_p, [_I]),
    "lka_set_split_tokens": (_I, [_I]),
    "lka_selftest_wait_timeout": (_I, [_P, _Z, _I, _P]),
    "lka_kernel_timing": (_I, [_I]),
    "lka_kernel_timing_read": (_I, [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double)]),
}

_lib = None
_lib_lock = threading.Lock()


class LkaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


def library():
    """The loaded liblka.so (raises if it has not been built)."""
    global _lib
    with _lib_lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with latent_kv_attention_b200.build.build()")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(lib, name)
                f.restype = res
                f.argtypes = args
            _lib = lib
    return _lib


def _check(fn: str, code: int):
    if code != LKA_OK:
        raise LkaError(fn, code)


def _stream_ptr(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class _Workspaces:
    """One zero-initialised device workspace per (device, stream), grown on demand.

    The first 256 bytes of a workspace hold the library's sticky status word;
    the rest is scratch that the kernels overwrite on every call."""

    def __init__(self):
        self._ws = {}
        self._lock = threading.Lock()

    def get(self, nbytes: int, device, stream=None) -> torch.Tensor:
        s = torch.cuda.current_stream(device) if stream is None else stream
        key = (device.index if device.index is not None else torch.cuda.current_device(), s.cuda_stream)
        nbytes = max(int(nbytes), 256)
        with self._lock:
            t = self._ws.get(key)
            if t is None or t.numel() < nbytes:
                t = torch.zeros(nbytes + (1 << 20), dtype=torch.uint8, device=device)
                self._ws[key] = t
            return t


workspaces = _Workspaces()


def _require(cond, msg):
    if not cond:
        raise ValueError(msg)


def _device_tensor(t, name, dtype=None):
    _require(isinstance(t, torch.Tensor) and t.is_cuda, f"{name} must be a CUDA tensor")
    _require(t.is_contiguous(), f"{name} must be contiguous")
    if dtype is not None:
        _require(t.dtype == dtype, f"{name} must be {dtype}, got {t.dtype}")


def _lens_tensor(cache_lens, B, device):
    _device_tensor(cache_lens, "cache_lens", torch.int32)
    _require(cache_lens.numel() == B and cache_lens.device == device, "cache_lens must be int32 [B] on q's device")


def _dtype_code(t):
    _require(t.dtype in _DT, f"unsupported dtype {t.dtype} (bf16 or fp32)")
    return _DT[t.dtype]


def gqa_attn(q, k, v, cache_lens, causal: bool = True, scale: float | None = None, out=None,
             return_lse: bool = False):
    """GQA attention. q [B,h_q,s_q,d], k/v [B,h_kv,Lmax,d] (bf16 or fp32), cache_lens int32 [B] on the device.

    Returns out [B,h_q,s_q,d] (and lse [B,h_q,s_q] fp32, natural log, if return_lse)."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _device_tensor(t, n, q.dtype)
    _require(q.dim() == 4 and k.dim() == 4 and v.shape == k.shape, "q [B,h_q,s_q,d], k/v [B,h_kv,Lmax,d]")
    B, h_q, s_q, d = q.shape
    _, h_kv, Lmax, dk = k.shape
    _require(dk == d and k.shape[0] == B, "q and k/v disagree on B or d")
    _lens_tensor(cache_lens, B, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _device_tensor(out, "out", q.dtype)
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q.device) if return_lse else None
    lib = library()
    nbytes = lib.gqa_attn_workspace_size(B, h_q, h_kv, s_q, d, Lmax)
    ws = workspaces.get(nbytes, q.device)
    rc = lib.gqa_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(cache_lens), _ptr(out), _ptr(lse), B, h_q, h_kv, s_q, d, Lmax,
                      int(bool(causal)), scale, _dtype_code(q), _ptr(ws), ws.numel(), _stream_ptr())
    _check("gqa_attn", rc)
    return (out, lse) if return_lse else out


def gqa_attn_fp8kv(q, k, v, k_scale, v_scale, cache_lens, causal: bool = True, scale: float | None = None, out=None,
                   return_lse: bool = False):
    """GQA attention over an e4m3 KV cache: q [B,h_q,s_q,d] bf16; k, v [B,h_kv,Lmax,d] torch.float8_e4m3fn;
    k_scale, v_scale fp32 [h_kv] (K = k_scale[h] * k, V = v_scale[h] * v); cache_lens int32 [B]."""
    _device_tensor(q, "q", torch.bfloat16)
    for n, t in (("k", k), ("v", v)):
        _device_tensor(t, n, torch.float8_e4m3fn)
    for n, t in (("k_scale", k_scale), ("v_scale", v_scale)):
        _device_tensor(t, n, torch.float32)
    _require(q.dim() == 4 and k.dim() == 4 and v.shape == k.shape, "q [B,h_q,s_q,d], k/v [B,h_kv,Lmax,d]")
    B, h_q, s_q, d = q.shape
    _, h_kv, Lmax, dk = k.shape
    _require(dk == d and k.shape[0] == B and k_scale.numel() == h_kv and v_scale.numel() == h_kv,
             "q, k/v and the scales disagree on B, d or h_kv")
    _lens_tensor(cache_lens, B, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _device_tensor(out, "out", torch.bfloat16)
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q.device) if return_lse else None
    lib = library()
    nbytes = lib.gqa_attn_fp8kv_workspace_size(B, h_q, h_kv, s_q, d, Lmax)
    ws = workspaces.get(nbytes, q.device)
    rc = lib.gqa_attn_fp8kv(_ptr(q), _ptr(k), _ptr(v), _ptr(k_scale), _ptr(v_scale), _ptr(cache_lens), _ptr(out),
                            _ptr(lse), B, h_q, h_kv, s_q, d, Lmax, int(bool(causal)), scale, _ptr(ws), ws.numel(),
                            _stream_ptr())
    _check("gqa_attn_fp8kv", rc)
    return (out, lse) if return_lse else out


def gqa_attn_paged(q, k_pages, v_pages, block_table, cache_lens, causal: bool = True, scale: float | None = None,
                   out=None, return_lse: bool = False):
    """GQA attention over a paged KV cache. q [B,h_q,s_q,d]; k_pages/v_pages [num_pages,h_kv,page_size,d];
    block_table int32 [B,max_pages] (token t of sequence b: row t % page_size of page block_table[b, t // page_size]);
    cache_lens int32 [B]. Returns out [B,h_q,s_q,d] (and lse [B,h_q,s_q] fp32 if return_lse)."""
    for n, t in (("q", q), ("k_pages", k_pages), ("v_pages", v_pages)):
        _device_tensor(t, n, q.dtype)
    _require(q.dim() == 4 and k_pages.dim() == 4 and v_pages.shape == k_pages.shape,
             "q [B,h_q,s_q,d], k_pages/v_pages [num_pages,h_kv,page_size,d]")
    B, h_q, s_q, d = q.shape
    num_pages, h_kv, page_size, dk = k_pages.shape
    _require(dk == d, "q and the pages disagree on d")
    _device_tensor(block_table, "block_table", torch.int32)
    _require(block_table.dim() == 2 and block_table.shape[0] == B and block_table.device == q.device,
             "block_table must be int32 [B, max_pages] on q's device")
    max_pages = block_table.shape[1]
    _lens_tensor(cache_lens, B, q.device)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = torch.empty_like(q) if out is None else out
    _device_tensor(out, "out", q.dtype)
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q.device) if return_lse else None
    lib = library()
    nbytes = lib.gqa_attn_paged_workspace_size(B, h_q, h_kv, s_q, d, page_size, max_pages)
    ws = workspaces.get(nbytes, q.device)
    rc = lib.gqa_attn_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(block_table), _ptr(cache_lens), _ptr(out),
                            _ptr(lse), B, h_q, h_kv, s_q, d, page_size, max_pages, num_pages, int(bool(causal)), scale,
                            _dtype_code(q), _ptr(ws), ws.numel(), _stream_ptr())
    _check("gqa_attn_paged", rc)
    return (out, lse) if return_lse else out


def latent_absorbed_attn(q_c, q_r, w_uk, w_uv, latent, cache_lens, causal: bool = True, scale: float | None = None,
                         out=None, return_lse: bool = False):
    """GQLA MQA-absorbed path. q_c [B,h_q,s_q,d_h], q_r [B,h_q,s_q,d_r], w_uk/w_uv [g,d_h,r_kv],
    latent [B,Lmax,r_kv+d_r] (c^KV then k^R), cache_lens int32 [B]. Returns out [B,h_q,s_q,d_h]."""
    for n, t in (("q_c", q_c), ("q_r", q_r), ("w_uk", w_uk), ("w_uv", w_uv), ("latent", latent)):
        _device_tensor(t, n, q_c.dtype)
    B, h_q, s_q, d_h = q_c.shape
    d_r = q_r.shape[-1]
    g, _, r_kv = w_uk.shape
    Lmax = latent.shape[1]
    _require(q_r.shape[:3] == (B, h_q, s_q) and w_uv.shape == w_uk.shape and w_uk.shape[1] == d_h, "shape mismatch")
    _require(latent.shape == (B, Lmax, r_kv + d_r), "latent must be [B,Lmax,r_kv+d_r]")
    _lens_tensor(cache_lens, B, q_c.device)
    scale = 1.0 / math.sqrt(d_h + d_r) if scale is None else float(scale)
    out = torch.empty_like(q_c) if out is None else out
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q_c.device) if return_lse else None
    lib = library()
    nbytes = lib.latent_absorbed_attn_workspace_size(B, h_q, g, s_q, d_h, r_kv, d_r, Lmax)
    ws = workspaces.get(nbytes, q_c.device)
    rc = lib.latent_absorbed_attn(_ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(w_uv), _ptr(latent), _ptr(cache_lens),
                                  _ptr(out), _ptr(lse), B, h_q, g, s_q, d_h, r_kv, d_r, Lmax, int(bool(causal)),
                                  scale, _dtype_code(q_c), _ptr(ws), ws.numel(), _stream_ptr())
    _check("latent_absorbed_attn", rc)
    return (out, lse) if return_lse else out


def latent_absorbed_attn_fp8kv(q_c, q_r, w_uk, w_uv, latent, kv_scale, cache_lens, causal: bool = True,
                               scale: float | None = None, out=None, return_lse: bool = False):
    """GQLA MQA-absorbed path over an e4m3 latent cache: latent [B,Lmax,r_kv+d_r] torch.float8_e4m3fn with
    kv_scale fp32 [2] (c^KV = kv_scale[0] * latent[..., :r_kv], k^R = kv_scale[1] * latent[..., r_kv:]);
    q_c, q_r, w_uk, w_uv bf16 as in latent_absorbed_attn. Returns out [B,h_q,s_q,d_h] bf16."""
    for n, t in (("q_c", q_c), ("q_r", q_r), ("w_uk", w_uk), ("w_uv", w_uv)):
        _device_tensor(t, n, torch.bfloat16)
    _device_tensor(latent, "latent", torch.float8_e4m3fn)
    _device_tensor(kv_scale, "kv_scale", torch.float32)
    _require(kv_scale.numel() == 2, "kv_scale must hold 2 values (latent part, RoPE key)")
    B, h_q, s_q, d_h = q_c.shape
    d_r = q_r.shape[-1]
    g, _, r_kv = w_uk.shape
    Lmax = latent.shape[1]
    _require(q_r.shape[:3] == (B, h_q, s_q) and w_uv.shape == w_uk.shape and w_uk.shape[1] == d_h, "shape mismatch")
    _require(latent.shape == (B, Lmax, r_kv + d_r), "latent must be [B,Lmax,r_kv+d_r]")
    _lens_tensor(cache_lens, B, q_c.device)
    scale = 1.0 / math.sqrt(d_h + d_r) if scale is None else float(scale)
    out = torch.empty_like(q_c) if out is None else out
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q_c.device) if return_lse else None
    lib = library()
    nbytes = lib.latent_absorbed_attn_fp8kv_workspace_size(B, h_q, g, s_q, d_h, r_kv, d_r, Lmax)
    ws = workspaces.get(nbytes, q_c.device)
    rc = lib.latent_absorbed_attn_fp8kv(_ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(w_uv), _ptr(latent), _ptr(kv_scale),
                                        _ptr(cache_lens), _ptr(out), _ptr(lse), B, h_q, g, s_q, d_h, r_kv, d_r, Lmax,
                                        int(bool(causal)), scale, _ptr(ws), ws.numel(), _stream_ptr())
    _check("latent_absorbed_attn_fp8kv", rc)
    return (out, lse) if return_lse else out


def latent_absorbed_attn_paged(q_c, q_r, w_uk, w_uv, latent_pages, block_table, cache_lens, causal: bool = True,
                               scale: float | None = None, out=None, return_lse: bool = False):
    """latent_absorbed_attn over a paged latent cache: latent_pages [num_pages, page_size, r_kv + d_r], block_table
    int32 [B, max_pages] (token t of sequence b: row t % page_size of page block_table[b, t // page_size])."""
    for n, t in (("q_c", q_c), ("q_r", q_r), ("w_uk", w_uk), ("w_uv", w_uv), ("latent_pages", latent_pages)):
        _device_tensor(t, n, torch.bfloat16)
    B, h_q, s_q, d_h = q_c.shape
    d_r = q_r.shape[-1]
    g, _, r_kv = w_uk.shape
    num_pages, page_size, width = latent_pages.shape
    _require(width == r_kv + d_r, "latent_pages [num_pages, page_size, r_kv + d_r]")
    _device_tensor(block_table, "block_table", torch.int32)
    _require(block_table.dim() == 2 and block_table.shape[0] == B, "block_table must be int32 [B, max_pages]")
    max_pages = block_table.shape[1]
    _lens_tensor(cache_lens, B, q_c.device)
    scale = 1.0 / math.sqrt(d_h + d_r) if scale is None else float(scale)
    out = torch.empty_like(q_c) if out is None else out
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q_c.device) if return_lse else None
    lib = library()
    nbytes = lib.latent_absorbed_attn_paged_workspace_size(B, h_q, g, s_q, d_h, r_kv, d_r, page_size, max_pages)
    _require(nbytes > 0, "unsupported latent shape or page layout")
    ws = workspaces.get(nbytes, q_c.device)
    rc = lib.latent_absorbed_attn_paged(_ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(w_uv), _ptr(latent_pages),
                                        _ptr(block_table), _ptr(cache_lens), _ptr(out), _ptr(lse), B, h_q, g, s_q, d_h,
                                        r_kv, d_r, page_size, max_pages, num_pages, int(bool(causal)), scale, 0,
                                        _ptr(ws), ws.numel(), _stream_ptr())
    _check("latent_absorbed_attn_paged", rc)
    return (out, lse) if return_lse else out


def latent_expand_gqa_attn(q_c, q_r, kc, vc, kr, cache_lens, causal: bool = True, scale: float | None = None,
                           out=None, return_lse: bool = False):
    """GQLA per-group GQA path. kc/vc [B,g,Lmax,d_h], kr [B,Lmax,d_r]; queries as latent_absorbed_attn."""
    for n, t in (("q_c", q_c), ("q_r", q_r), ("kc", kc), ("vc", vc), ("kr", kr)):
        _device_tensor(t, n, q_c.dtype)
    B, h_q, s_q, d_h = q_c.shape
    d_r = q_r.shape[-1]
    _, g, Lmax, _ = kc.shape
    _require(vc.shape == kc.shape and kr.shape == (B, Lmax, d_r), "kc/vc [B,g,Lmax,d_h], kr [B,Lmax,d_r]")
    _lens_tensor(cache_lens, B, q_c.device)
    scale = 1.0 / math.sqrt(d_h + d_r) if scale is None else float(scale)
    out = torch.empty_like(q_c) if out is None else out
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q_c.device) if return_lse else None
    lib = library()
    nbytes = lib.latent_expand_gqa_attn_workspace_size(B, h_q, g, s_q, d_h, d_r, Lmax)
    ws = workspaces.get(nbytes, q_c.device)
    rc = lib.latent_expand_gqa_attn(_ptr(q_c), _ptr(q_r), _ptr(kc), _ptr(vc), _ptr(kr), _ptr(cache_lens), _ptr(out),
                                    _ptr(lse), B, h_q, g, s_q, d_h, d_r, Lmax, int(bool(causal)), scale,
                                    _dtype_code(q_c), _ptr(ws), ws.numel(), _stream_ptr())
    _check("latent_expand_gqa_attn", rc)
    return (out, lse) if return_lse else out


def latent_expand_gqa_attn_paged(q_c, q_r, kc_pages, vc_pages, kr_pages, block_table, cache_lens, causal: bool = True,
                                 scale: float | None = None, out=None, return_lse: bool = False):
    """latent_expand_gqa_attn over paged caches: kc_pages/vc_pages [num_pages, g, page_size, d_h], kr_pages
    [num_pages, page_size, d_r], block_table int32 [B, max_pages]."""
    for n, t in (("q_c", q_c), ("q_r", q_r), ("kc_pages", kc_pages), ("vc_pages", vc_pages), ("kr_pages", kr_pages)):
        _device_tensor(t, n, torch.bfloat16)
    B, h_q, s_q, d_h = q_c.shape
    num_pages, g, page_size, _ = kc_pages.shape
    d_r = kr_pages.shape[-1]
    _require(vc_pages.shape == kc_pages.shape and kr_pages.shape[:2] == (num_pages, page_size),
             "kc/vc pages [num_pages, g, page_size, d_h], kr pages [num_pages, page_size, d_r]")
    _device_tensor(block_table, "block_table", torch.int32)
    _require(block_table.dim() == 2 and block_table.shape[0] == B, "block_table must be int32 [B, max_pages]")
    max_pages = block_table.shape[1]
    _lens_tensor(cache_lens, B, q_c.device)
    scale = 1.0 / math.sqrt(d_h + d_r) if scale is None else float(scale)
    out = torch.empty_like(q_c) if out is None else out
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q_c.device) if return_lse else None
    lib = library()
    nbytes = lib.latent_expand_gqa_attn_paged_workspace_size(B, h_q, g, s_q, d_h, d_r, page_size, max_pages)
    _require(nbytes > 0, "unsupported expanded shape or page layout")
    ws = workspaces.get(nbytes, q_c.device)
    rc = lib.latent_expand_gqa_attn_paged(_ptr(q_c), _ptr(q_r), _ptr(kc_pages), _ptr(vc_pages), _ptr(kr_pages),
                                          _ptr(block_table), _ptr(cache_lens), _ptr(out), _ptr(lse), B, h_q, g, s_q,
                                          d_h, d_r, page_size, max_pages, num_pages, int(bool(causal)), scale, 0,
                                          _ptr(ws), ws.numel(), _stream_ptr())
    _check("latent_expand_gqa_attn_paged", rc)
    return (out, lse) if return_lse else out


def latent_absorbed_attn_sparse(q_c, q_r, w_uk, w_uv, latent, indices, cache_lens, scale: float | None = None,
                                out=None, return_lse: bool = False):
    """Top-k sparse MQA-absorbed latent attention: indices int32 [B, s_q, topk] are the cache positions each query
    token attends to (entries outside [0, L_b - s_q + t] are skipped)."""
    for n, t in (("q_c", q_c), ("q_r", q_r), ("w_uk", w_uk), ("w_uv", w_uv), ("latent", latent)):
        _device_tensor(t, n, torch.bfloat16)
    B, h_q, s_q, d_h = q_c.shape
    d_r = q_r.shape[-1]
    g, _, r_kv = w_uk.shape
    Lmax = latent.shape[1]
    _device_tensor(indices, "indices", torch.int32)
    _require(indices.dim() == 3 and indices.shape[:2] == (B, s_q), "indices must be int32 [B, s_q, topk]")
    topk = indices.shape[2]
    _lens_tensor(cache_lens, B, q_c.device)
    scale = 1.0 / math.sqrt(d_h + d_r) if scale is None else float(scale)
    out = torch.empty_like(q_c) if out is None else out
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q_c.device) if return_lse else None
    lib = library()
    nbytes = lib.latent_absorbed_attn_sparse_workspace_size(B, h_q, g, s_q, d_h, r_kv, d_r, topk)
    _require(nbytes > 0, "unsupported sparse latent shape")
    ws = workspaces.get(nbytes, q_c.device)
    rc = lib.latent_absorbed_attn_sparse(_ptr(q_c), _ptr(q_r), _ptr(w_uk), _ptr(w_uv), _ptr(latent), _ptr(indices),
                                         _ptr(cache_lens), _ptr(out), _ptr(lse), B, h_q, g, s_q, d_h, r_kv, d_r, Lmax,
                                         topk, scale, 0, _ptr(ws), ws.numel(), _stream_ptr())
    _check("latent_absorbed_attn_sparse", rc)
    return (out, lse) if return_lse else out


def latent_expand_gqa_attn_sparse(q_c, q_r, kc, vc, kr, indices, cache_lens, scale: float | None = None, out=None,
                                  return_lse: bool = False):
    """Top-k sparse attention on the per-group GQA path: indices int32 [B, s_q, topk] as in
    latent_absorbed_attn_sparse; kc, vc [B, g, Lmax, d_h], kr [B, Lmax, d_r]."""
    for n, t in (("q_c", q_c), ("q_r", q_r), ("kc", kc), ("vc", vc), ("kr", kr)):
        _device_tensor(t, n, torch.bfloat16)
    B, h_q, s_q, d_h = q_c.shape
    _, g, Lmax, _ = kc.shape
    d_r = kr.shape[-1]
    _device_tensor(indices, "indices", torch.int32)
    _require(indices.dim() == 3 and indices.shape[:2] == (B, s_q), "indices must be int32 [B, s_q, topk]")
    topk = indices.shape[2]
    _lens_tensor(cache_lens, B, q_c.device)
    scale = 1.0 / math.sqrt(d_h + d_r) if scale is None else float(scale)
    out = torch.empty_like(q_c) if out is None else out
    lse = torch.empty((B, h_q, s_q), dtype=torch.float32, device=q_c.device) if return_lse else None
    lib = library()
    nbytes = lib.latent_expand_gqa_attn_sparse_workspace_size(B, h_q, g, s_q, d_h, d_r, topk)
    _require(nbytes > 0, "unsupported sparse expanded shape")
    ws = workspaces.get(nbytes, q_c.device)
    rc = lib.latent_expand_gqa_attn_sparse(_ptr(q_c), _ptr(q_r), _ptr(kc), _ptr(vc), _ptr(kr), _ptr(indices),
                                           _ptr(cache_lens), _ptr(out), _ptr(lse), B, h_q, g, s_q, d_h, d_r, Lmax,
                                           topk, scale, 0, _ptr(ws), ws.numel(), _stream_ptr())
    _check("latent_expand_gqa_attn_sparse", rc)
    return (out, lse) if return_lse else out


def gta_shared_score_attn(q_g, k_g, v, cache_lens, causal: bool = True, scale: float | None = None, out=None,
                          return_lse: bool = False):
    """GTA shared-score attention. q_g [B,G,s_q,d_qk], k_g [B,G,Lmax,d_qk], v [B,H,Lmax,d_v].

    Returns out [B,H,s_q,d_v] (and lse [B,G,s_q] if return_lse)."""
    for n, t in (("q_g", q_g), ("k_g", k_g), ("v", v)):
        _device_tensor(t, n, q_g.dtype)
    B, G, s_q, d_qk = q_g.shape
    _, H, Lmax, d_v = v.shape
    _require(k_g.shape == (B, G, Lmax, d_qk), "k_g must be [B,G,Lmax,d_qk]")
    _lens_tensor(cache_lens, B, q_g.device)
    scale = 1.0 / math.sqrt(d_qk) if scale is None else float(scale)
    out = torch.empty((B, H, s_q, d_v), dtype=q_g.dtype, device=q_g.device) if out is None else out
    lse = torch.empty((B, G, s_q), dtype=torch.float32, device=q_g.device) if return_lse else None
    lib = library()
    nbytes = lib.gta_shared_score_attn_workspace_size(B, G, H, s_q, d_qk, d_v, Lmax)
    ws = workspaces.get(nbytes, q_g.device)
    rc = lib.gta_shared_score_attn(_ptr(q_g), _ptr(k_g), _ptr(v), _ptr(cache_lens), _ptr(out), _ptr(lse), B, G, H,
                                   s_q, d_qk, d_v, Lmax, int(bool(causal)), scale, _dtype_code(q_g), _ptr(ws),
                                   ws.numel(), _stream_ptr())
    _check("gta_shared_score_attn", rc)
    return (out, lse) if return_lse else out


def gta_shared_score_attn_paged(q_g, k_pages, v_pages, block_table, cache_lens, causal: bool = True,
                                scale: float | None = None, out=None, return_lse: bool = False):
    """GTA shared-score attention over paged caches. q_g [B,G,s_q,d_qk]; k_pages [num_pages,G,page_size,d_qk];
    v_pages [num_pages,H,page_size,d_v]; block_table int32 [B,max_pages] (token t of sequence b: row
    t % page_size of page block_table[b, t // page_size] in both pools). Returns out [B,H,s_q,d_v]."""
    for n, t in (("q_g", q_g), ("k_pages", k_pages), ("v_pages", v_pages)):
        _device_tensor(t, n, q_g.dtype)
    _require(q_g.dim() == 4 and k_pages.dim() == 4 and v_pages.dim() == 4,
             "q_g [B,G,s_q,d_qk], k_pages [num_pages,G,page_size,d_qk], v_pages [num_pages,H,page_size,d_v]")
    B, G, s_q, d_qk = q_g.shape
    num_pages, H, page_size, d_v = v_pages.shape
    _require(k_pages.shape == (num_pages, G, page_size, d_qk), "k_pages must be [num_pages,G,page_size,d_qk]")
    _device_tensor(block_table, "block_table", torch.int32)
    _require(block_table.dim() == 2 and block_table.shape[0] == B and block_table.device == q_g.device,
             "block_table must be int32 [B, max_pages] on q_g's device")
    max_pages = block_table.shape[1]
    _lens_tensor(cache_lens, B, q_g.device)
    scale = 1.0 / math.sqrt(d_qk) if scale is None else float(scale)
    out = torch.empty((B, H, s_q, d_v), dtype=q_g.dtype, device=q_g.device) if out is None else out
    lse = torch.empty((B, G, s_q), dtype=torch.float32, device=q_g.device) if return_lse else None
    lib = library()
    nbytes = lib.gta_shared_score_attn_paged_workspace_size(B, G, H, s_q, d_qk, d_v, page_size, max_pages)
    _require(nbytes > 0, "page_size must be a power of two >= 8")
    ws = workspaces.get(nbytes, q_g.device)
    rc = lib.gta_shared_score_attn_paged(_ptr(q_g), _ptr(k_pages), _ptr(v_pages), _ptr(block_table),
                                         _ptr(cache_lens), _ptr(out), _ptr(lse), B, G, H, s_q, d_qk, d_v, page_size,
                                         max_pages, num_pages, int(bool(causal)), scale, _dtype_code(q_g), _ptr(ws),
                                         ws.numel(), _stream_ptr())
    _check("gta_shared_score_attn_paged", rc)
    return (out, lse) if return_lse else out


def latent_expand_cache(latent, w_uk, w_uv):
    """One-time conversion latent [B,Lmax,r_kv+d_r] -> (kc, vc [B,g,Lmax,d_h], kr [B,Lmax,d_r])."""
    for n, t in (("latent", latent), ("w_uk", w_uk), ("w_uv", w_uv)):
        _device_tensor(t, n, latent.dtype)
    B, Lmax, W = latent.shape
    g, d_h, r_kv = w_uk.shape
    d_r = W - r_kv
    kc = torch.empty((B, g, Lmax, d_h), dtype=latent.dtype, device=latent.device)
    vc = torch.empty_like(kc)
    kr = torch.empty((B, Lmax, d_r), dtype=latent.dtype, device=latent.device)
    rc = library().latent_expand_cache(_ptr(latent), _ptr(w_uk), _ptr(w_uv), B, Lmax, g, d_h, r_kv, d_r, _ptr(kc),
                                       _ptr(vc), _ptr(kr), _dtype_code(latent), _stream_ptr())
    _check("latent_expand_cache", rc)
    return kc, vc, kr


def device_status(device=None) -> int:
    """Synchronises the current stream and returns the sticky status code of its workspace."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ws = workspaces.get(256, device)
    return int(library().lka_device_status(_ptr(ws), _stream_ptr()))


def clear_status(device=None):
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    ws = workspaces.get(256, device)
    _check("lka_clear_status", library().lka_clear_status(_ptr(ws), _stream_ptr()))


def gqa_split_count(B: int, h_q: int, h_kv: int, s_q: int, d: int, Lmax: int, dtype=torch.bfloat16) -> int:
    """Key splits per sequence that gqa_attn plans for these sizes (0 if it would reject them); host-only."""
    return int(library().gqa_attn_split_count(B, h_q, h_kv, s_q, d, Lmax, _DT[dtype]))


def set_split_tokens(tokens: int) -> int:
    """KV tokens per split of the split-KV kernels for calls made from this thread (0 = automatic); returns the
    previous value."""
    return int(library().lka_set_split_tokens(int(tokens)))


def kernel_timing(enable: bool):
    """Start (discarding earlier records) or stop recording CUDA events around each call's main kernel."""
    _check("lka_kernel_timing", library().lka_kernel_timing(int(bool(enable))))


def kernel_timing_read():
    """(number of timed launches, their total milliseconds) recorded since kernel_timing(True)."""
    n, ms = ctypes.c_int(0), ctypes.c_double(0.0)
    _check("lka_kernel_timing_read", library().lka_kernel_timing_read(ctypes.byref(n), ctypes.byref(ms)))
    return int(n.value), float(ms.value)


def status_string(code: int) -> str:
    return library().lka_status_string(int(code)).decode()
