"""Plain fp64 CPU oracle for grouped / latent-KV attention (ctypes wrapper).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test-suite, the smoke check
and the benchmark's CPU-baseline leg may import this package.  The product
library (``latent_kv_attention_b200``) never imports it and shares no code with
it; the only thing both sides consume is the seeded inputs of ``synthetic.py``.

The arithmetic lives in ``oracle.c`` (plain C, double precision, one output row
at a time); this module only builds it with gcc, converts arrays to contiguous
float64/int32 numpy arrays, calls it and returns numpy outputs.  See the header
of ``oracle.c`` for the definitions, the pages they follow and the readings
taken where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, pthreads). Returns the path."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load_library(path: str):
    """Open an oracle shared library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    I, D = ctypes.c_int, ctypes.c_double
    lib.oracle_gqa.argtypes = [dp, dp, dp, ip, I, I, I, I, I, I, I, D, dp, dp, ip, I, I]
    lib.oracle_gqa_probs.argtypes = [dp, dp, ip, I, I, I, I, I, I, I, D, I, I, I, dp]
    lat = [dp, dp, dp, dp, dp, ip, I, I, I, I, I, I, I, I, I, D, dp, dp, ip, I, I]
    lib.oracle_latent_expanded.argtypes = lat
    lib.oracle_latent_absorbed.argtypes = lat
    lib.oracle_latent_expand_cache.argtypes = [dp, dp, dp, I, I, I, I, I, I, dp, dp, dp, I]
    lib.oracle_gta.argtypes = [dp, dp, dp, ip, I, I, I, I, I, I, I, I, D, dp, dp, ip, I, I]
    lib.oracle_merge_partials.argtypes = [dp, dp, I, I, dp, dp]
    lib.oracle_threads_used.argtypes = [I, ctypes.c_long]
    for f in ("oracle_gqa", "oracle_gqa_probs", "oracle_latent_expanded", "oracle_latent_absorbed",
              "oracle_latent_expand_cache", "oracle_gta", "oracle_merge_partials", "oracle_threads_used"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = load_library(_LIB_PATH)
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor (any dtype, any device)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _u8(x) -> np.ndarray:
    """The raw bytes of a tensor or array of 8-bit codes (a torch float8 tensor is viewed as uint8)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        if x.dtype != torch.uint8:
            x = x.view(torch.uint8)
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint8))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def _rows(rows_b):
    if rows_b is None:
        return None, 0
    r = _i32(rows_b)
    return r, int(r.size)


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"{name}: invalid argument (oracle returned {rc})")


def threads_used(n_threads: int, n_items: int) -> int:
    """Threads the oracle's pool uses for n_items work items (0 = all online cores)."""
    return int(_load().oracle_threads_used(int(n_threads), int(n_items)))


def gqa(q, k, v, cache_lens, causal: bool, scale: float, rows_b=None, n_threads: int = 0):
    """Grouped-query attention. q [B,h_q,s_q,d], k/v [B,h_kv,Lmax,d], cache_lens [B].

    Returns (out [B,h_q,s_q,d], lse [B,h_q,s_q]) as float64 numpy arrays; with
    ``rows_b`` only those batch rows are evaluated (the others stay NaN)."""
    q, k, v, lens = _f64(q), _f64(k), _f64(v), _i32(cache_lens)
    B, h_q, s_q, d = q.shape
    _, h_kv, Lmax, _ = k.shape
    out = np.full((B, h_q, s_q, d), np.nan)
    lse = np.full((B, h_q, s_q), np.nan)
    r, nr = _rows(rows_b)
    rc = _load().oracle_gqa(_dp(q), _dp(k), _dp(v), _ip(lens), B, h_q, h_kv, s_q, d, Lmax, int(causal),
                            float(scale), _dp(out), _dp(lse), _ip(r), nr, int(n_threads))
    _check(rc, "oracle_gqa")
    return out, lse


def paged_to_contiguous(pages, block_table, Lmax: int):
    """The cache a block table describes, as one slab per sequence: cache[b, h, t] = pages[block_table[b,
    t // page_size], h, t % page_size] for t < Lmax ("Grouped Query Attention (GQA)" glossary page, comparison
    with related techniques: PagedAttention keeps the cache in fixed-size blocks).  pages [num_pages, h_kv,
    page_size, d]; entries of the table past a sequence's pages may hold anything: rows they address are filled
    with NaN, which the attention definition never reads for t >= cache_lens[b]."""
    pages = _f64(pages)
    bt = _i32(block_table)
    num_pages, h_kv, ps, d = pages.shape
    B = bt.shape[0]
    out = np.full((B, h_kv, Lmax, d), np.nan)
    for b in range(B):
        for t0 in range(0, Lmax, ps):
            j = t0 // ps
            if j >= bt.shape[1] or not (0 <= bt[b, j] < num_pages):
                continue
            n = min(ps, Lmax - t0)
            out[b, :, t0:t0 + n, :] = pages[bt[b, j], :, :n, :]
    return out


def gqa_paged(q, k_pages, v_pages, block_table, cache_lens, causal: bool, scale: float, rows_b=None,
              n_threads: int = 0):
    """GQA attention over a paged cache: the contiguous cache the block table describes, then gqa()."""
    bt = _i32(block_table)
    ps = int(np.asarray(k_pages.shape)[2])
    Lmax = bt.shape[1] * ps
    k = paged_to_contiguous(k_pages, bt, Lmax)
    v = paged_to_contiguous(v_pages, bt, Lmax)
    return gqa(q, k, v, cache_lens, causal, scale, rows_b=rows_b, n_threads=n_threads)


def gta_paged(q_g, k_pages, v_pages, block_table, cache_lens, causal: bool, scale: float, n_threads: int = 0):
    """GTA shared-score attention over paged caches (k_pages [num_pages, G, page_size, d_qk], v_pages [num_pages,
    H, page_size, d_v], one block table): the contiguous caches the block table describes, then gta()."""
    bt = _i32(block_table)
    ps = int(np.asarray(k_pages.shape)[2])
    Lmax = bt.shape[1] * ps
    k_g = paged_to_contiguous(k_pages, bt, Lmax)
    v = paged_to_contiguous(v_pages, bt, Lmax)
    return gta(q_g, k_g, v, cache_lens, causal, scale, n_threads=n_threads)


def latent_absorbed_paged(q_c, q_r, w_uk, w_uv, latent_pages, block_table, cache_lens, causal: bool, scale: float,
                          rows_b=None, n_threads: int = 0):
    """The MQA-absorbed latent attention over a paged latent cache [num_pages, page_size, r_kv + d_r]: the
    contiguous latent cache the block table describes, then latent_absorbed()."""
    pages = _f64(latent_pages)
    bt = _i32(block_table)
    Lmax = bt.shape[1] * pages.shape[1]
    latent = paged_to_contiguous(pages[:, None], bt, Lmax)[:, 0]
    return latent_absorbed(q_c, q_r, w_uk, w_uv, latent, cache_lens, causal, scale, rows_b=rows_b,
                           n_threads=n_threads)


def sparse_selection(indices, cache_lens, s_q: int):
    """The keys each query token attends to under top-k sparse attention ("GQLA ..." sections 1 and 2: a
    token-dependent top-k selection of past keys/values): for query t of sequence b, the entries j of
    indices[b, t] with 0 <= j <= L_b - s_q + t, in list order.  Returns a list (over b) of lists (over t)."""
    idx = _i32(indices)
    lens = _i32(cache_lens)
    out = []
    for b in range(idx.shape[0]):
        row = []
        for t in range(s_q):
            last = int(lens[b]) - s_q + t
            row.append([int(j) for j in idx[b, t] if 0 <= j <= last])
        out.append(row)
    return out


def _sparse_apply(dense, q_parts, sel, cache_rows, out_shape, lse_shape):
    """Runs `dense` (a non-causal single-query attention of this module) per (sequence, query token) over the
    selected cache rows; an empty selection gives out = 0, lse = -inf."""
    out = np.zeros(out_shape)
    lse = np.full(lse_shape, -np.inf)
    B, s_q = len(sel), len(sel[0])
    for b in range(B):
        for t in range(s_q):
            keys = sel[b][t]
            if not keys:
                continue
            o, l = dense([qp[b:b + 1, :, t:t + 1] for qp in q_parts], [c(b, keys) for c in cache_rows],
                         np.array([len(keys)], dtype=np.int32))
            out[b, :, t] = o[0, :, 0]
            lse[b, :, t] = l[0, :, 0]
    return out, lse


def latent_absorbed_sparse(q_c, q_r, w_uk, w_uv, latent, indices, cache_lens, scale: float):
    """Top-k sparse attention of the MQA-absorbed latent path: for each query token, latent_absorbed() over the
    selected latent rows only (sparse_selection)."""
    q_c, q_r, lat = _f64(q_c), _f64(q_r), _f64(latent)
    B, h_q, s_q, d_h = q_c.shape
    sel = sparse_selection(indices, cache_lens, s_q)
    dense = lambda qs, cs, lens: latent_absorbed(qs[0], qs[1], w_uk, w_uv, cs[0], lens, False, scale)  # noqa: E731
    return _sparse_apply(dense, [q_c, q_r], sel, [lambda b, keys: lat[b:b + 1, keys]], (B, h_q, s_q, d_h),
                         (B, h_q, s_q))


def expanded_sparse(q_c, q_r, kc, vc, kr, indices, cache_lens, scale: float):
    """Top-k sparse attention of the per-group GQA path: GQA with key [kc[g] ; kr] and value vc[g] over the
    selected tokens only (sparse_selection)."""
    q_c, q_r, kc, vc, kr = _f64(q_c), _f64(q_r), _f64(kc), _f64(vc), _f64(kr)
    B, h_q, s_q, d_h = q_c.shape
    g = kc.shape[1]
    sel = sparse_selection(indices, cache_lens, s_q)

    def dense(qs, cs, lens):
        key = np.concatenate([cs[0], np.broadcast_to(cs[2][:, None], cs[0].shape[:3] + (cs[2].shape[-1],))], -1)
        val = np.concatenate([cs[1], np.zeros(cs[1].shape[:3] + (cs[2].shape[-1],))], -1)
        o, l = gqa(np.concatenate([qs[0], qs[1]], -1), key, val, lens, False, scale)
        return o[..., :d_h], l

    rows = [lambda b, keys: kc[b:b + 1][:, :, keys], lambda b, keys: vc[b:b + 1][:, :, keys],
            lambda b, keys: kr[b:b + 1, keys]]
    return _sparse_apply(dense, [q_c, q_r], sel, rows, (B, h_q, s_q, d_h), (B, h_q, s_q))


def decode_e4m3(x):
    """The values of e4m3 codes (OCP 8-bit floating point E4M3, as torch.float8_e4m3fn or uint8), in float64, from
    the format's bit fields: sign bit 7, exponent bits 6-3 with bias 7, mantissa bits 2-0; exponent 0 encodes the
    subnormals m * 2^-9; S.1111.111 is NaN; there are no infinities (S.1111.000-110 are 256 .. 448)."""
    u = _u8(x).astype(np.int64)
    sign = np.where(u & 0x80, -1.0, 1.0)
    e, m = (u >> 3) & 0xF, u & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def dequantize_e4m3(x, head_scale):
    """An e4m3 cache [B, h_kv, L, d] widened exactly (decode_e4m3) and multiplied by its per-KV-head scale [h_kv],
    in float64."""
    return decode_e4m3(x) * _f64(head_scale)[None, :, None, None]


def latent_absorbed_fp8kv(q_c, q_r, w_uk, w_uv, latent8, kv_scale, cache_lens, causal: bool, scale: float,
                          rows_b=None, n_threads: int = 0):
    """The MQA-absorbed latent attention over an e4m3 latent cache [B, L, r_kv + d_r] with one scale for the
    latent part and one for the RoPE key (kv_scale [2]): the dequantised cache, then latent_absorbed()."""
    r_kv = int(np.asarray(w_uk.shape)[2])
    sc = _f64(kv_scale)
    lat = decode_e4m3(latent8)
    lat[..., :r_kv] *= sc[0]
    lat[..., r_kv:] *= sc[1]
    return latent_absorbed(q_c, q_r, w_uk, w_uv, lat, cache_lens, causal, scale, rows_b=rows_b, n_threads=n_threads)


def gqa_fp8kv(q, k, v, k_scale, v_scale, cache_lens, causal: bool, scale: float, rows_b=None, n_threads: int = 0):
    """GQA attention over an e4m3 KV cache with per-KV-head scales: the dequantised cache, then gqa()."""
    return gqa(q, dequantize_e4m3(k, k_scale), dequantize_e4m3(v, v_scale), cache_lens, causal, scale,
               rows_b=rows_b, n_threads=n_threads)


def gqa_probs(q, k, cache_lens, causal: bool, scale: float, b: int, i: int, t: int, h_kv: int):
    """Softmax probabilities of one query row of the GQA definition (visible keys only)."""
    q, k, lens = _f64(q), _f64(k), _i32(cache_lens)
    B, h_q, s_q, d = q.shape
    Lmax = k.shape[2]
    p = np.zeros(Lmax)
    n = _load().oracle_gqa_probs(_dp(q), _dp(k), _ip(lens), B, h_q, h_kv, s_q, d, Lmax, int(causal),
                                 float(scale), int(b), int(i), int(t), _dp(p))
    if n < 0:
        raise ValueError("oracle_gqa_probs: invalid argument")
    return p[:n]


def _latent(fn_name, q_c, q_r, w_uk, w_uv, latent, cache_lens, causal, scale, rows_b, n_threads):
    q_c, q_r, w_uk, w_uv, latent, lens = (_f64(q_c), _f64(q_r), _f64(w_uk), _f64(w_uv), _f64(latent),
                                          _i32(cache_lens))
    B, h_q, s_q, d_h = q_c.shape
    d_r = q_r.shape[3]
    g, _, r_kv = w_uk.shape
    Lmax = latent.shape[1]
    if latent.shape[2] != r_kv + d_r:
        raise ValueError("latent last dim must be r_kv + d_r")
    out = np.full((B, h_q, s_q, d_h), np.nan)
    lse = np.full((B, h_q, s_q), np.nan)
    r, nr = _rows(rows_b)
    rc = getattr(_load(), fn_name)(_dp(q_c), _dp(q_r), _dp(w_uk), _dp(w_uv), _dp(latent), _ip(lens), B, h_q,
                                   g, s_q, d_h, r_kv, d_r, Lmax, int(causal), float(scale), _dp(out),
                                   _dp(lse), _ip(r), nr, int(n_threads))
    _check(rc, fn_name)
    return out, lse


def latent_expanded(q_c, q_r, w_uk, w_uv, latent, cache_lens, causal: bool, scale: float, rows_b=None,
                    n_threads: int = 0):
    """GQLA attention from its definition (eq. (1)): per-group keys/values expanded from the latent.

    q_c [B,h_q,s_q,d_h], q_r [B,h_q,s_q,d_r], w_uk/w_uv [g,d_h,r_kv], latent [B,Lmax,r_kv+d_r]."""
    return _latent("oracle_latent_expanded", q_c, q_r, w_uk, w_uv, latent, cache_lens, causal, scale,
                   rows_b, n_threads)


def latent_absorbed(q_c, q_r, w_uk, w_uv, latent, cache_lens, causal: bool, scale: float, rows_b=None,
                    n_threads: int = 0):
    """GQLA attention in the MQA-absorbed form (W^UK folded into q, W^UV applied after)."""
    return _latent("oracle_latent_absorbed", q_c, q_r, w_uk, w_uv, latent, cache_lens, causal, scale,
                   rows_b, n_threads)


def latent_expand_cache(latent, w_uk, w_uv, n_threads: int = 0):
    """One-time conversion latent -> (kc [B,g,Lmax,d_h], vc [B,g,Lmax,d_h], kr [B,Lmax,d_r])."""
    latent, w_uk, w_uv = _f64(latent), _f64(w_uk), _f64(w_uv)
    B, Lmax, W = latent.shape
    g, d_h, r_kv = w_uk.shape
    d_r = W - r_kv
    kc = np.zeros((B, g, Lmax, d_h))
    vc = np.zeros((B, g, Lmax, d_h))
    kr = np.zeros((B, Lmax, d_r))
    rc = _load().oracle_latent_expand_cache(_dp(latent), _dp(w_uk), _dp(w_uv), B, Lmax, g, d_h, r_kv, d_r,
                                            _dp(kc), _dp(vc), _dp(kr), int(n_threads))
    _check(rc, "oracle_latent_expand_cache")
    return kc, vc, kr


def gta(q_g, k_g, v, cache_lens, causal: bool, scale: float, rows_b=None, n_threads: int = 0):
    """GTA shared-score attention. q_g [B,G,s_q,d_qk], k_g [B,G,Lmax,d_qk], v [B,H,Lmax,d_v].

    Returns (out [B,H,s_q,d_v], lse [B,G,s_q])."""
    q_g, k_g, v, lens = _f64(q_g), _f64(k_g), _f64(v), _i32(cache_lens)
    B, G, s_q, d_qk = q_g.shape
    _, H, Lmax, d_v = v.shape
    out = np.full((B, H, s_q, d_v), np.nan)
    lse = np.full((B, G, s_q), np.nan)
    r, nr = _rows(rows_b)
    rc = _load().oracle_gta(_dp(q_g), _dp(k_g), _dp(v), _ip(lens), B, G, H, s_q, d_qk, d_v, Lmax, int(causal),
                            float(scale), _dp(out), _dp(lse), _ip(r), nr, int(n_threads))
    _check(rc, "oracle_gta")
    return out, lse


def merge_partials(parts_o, parts_lse):
    """Merge attention partials over disjoint key sets: parts_o [n,dv], parts_lse [n]."""
    po, pl = _f64(parts_o), _f64(parts_lse)
    n, dv = po.shape
    out = np.zeros(dv)
    lse = np.zeros(1)
    rc = _load().oracle_merge_partials(_dp(po), _dp(pl), n, dv, _dp(out), _dp(lse))
    _check(rc, "oracle_merge_partials")
    return out, float(lse[0])
