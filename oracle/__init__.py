"""Oracle for paged MLA decode -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package's ``smoke()`` check and the benchmark's CPU-baseline leg may
import this package.  The product path (the CUDA library and its Python binding) never
does, and shares no code with it.

Contents
  mla_decode / mla_decode_rows   fp64 decode of every (b, s, h), or of listed rows
                                 (plain C, ``mla_oracle.c``; two-pass softmax)
  mla_decode_fp8 / ..._rows_fp8  the same over an FP8 latent cache (E4M3 codes and one fp32
                                 scale per token and latent head, dequantised exactly)
  e4m3_to_float64                OCP E4M3 decoding (the C oracle's, exposed for its pins)
  mla_decode_sparse / ..._rows_sparse
                                 token-level sparse decode: each query token attends to the
                                 key positions of its CSR list (row_ptr, col_idx)
  combine                        log-sum-exp merge of split partials (numpy fp64)
  absorb_query / absorb_output   the weight-absorption products either side of the latent
                                 decode (numpy fp64 einsum)
  metadata                       split-KV scheduler specification (``metadata.py``)

Where each formula comes from is stated in ``mla_oracle.c`` and ``metadata.py``.
Parity of the scheduler specification is unpinned against the pages (they print only
its call signature); it is pinned by its coverage invariants and hand-worked cases.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

from . import metadata  # noqa: F401  (re-exported)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmla_oracle.so")
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, no fast-math) next to its source."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build_oracle()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_mla_decode_rows.argtypes = [
            P, i64, i64, i64, i32, i32, i32, i32,
            P, i64, i32, i32,
            P, i64, P, P, P,
            i32, f64, i32,
            P, i64, P, P]
        lib.oracle_mla_decode_rows.restype = i32
        lib.oracle_mla_decode_rows_fp8.argtypes = [
            P, i64, i64, i64, i32, i32, i32, i32,
            P, P, i64, i32, i32,
            P, i64, P, P, P,
            i32, f64, i32,
            P, i64, P, P]
        lib.oracle_mla_decode_rows_fp8.restype = i32
        lib.oracle_mla_decode_rows_sparse.argtypes = [
            P, i64, i64, i64, i32, i32, i32, i32,
            P, i64, i32, i32,
            P, i64, P, P, P, P, P,
            i32, f64, i32,
            P, i64, P, P]
        lib.oracle_mla_decode_rows_sparse.restype = i32
        lib.oracle_e4m3_to_double.argtypes = [P, i64, P]
        lib.oracle_e4m3_to_double.restype = i32
        lib.oracle_num_threads.restype = i32
        _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loop uses (OMP_NUM_THREADS, else all host cores)."""
    return int(_load().oracle_num_threads())


def _bf16_bits(t) -> np.ndarray:
    """bf16 tensor -> uint16 numpy array of its raw bits (no rounding)."""
    import torch
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def mla_decode_rows(q, k_cache, block_table, cache_seqlens, rows, dv: int = 512,
                    softmax_scale: Optional[float] = None, causal: bool = True,
                    kv_begin=None, kv_end=None):
    """fp64 decode of the listed rows.

    q [b, s_q, h_q, d] bf16, k_cache [num_pages, page, h_kv, d] bf16, block_table
    [b, max_pages] int32, cache_seqlens [b] int32, rows: int array [n, 3] of (b, s, h).
    kv_begin / kv_end (optional [b] int32) restrict each sequence's keys to
    [kv_begin, kv_end) -- a split-KV partial.  Returns (out [n, dv], lse [n]) float64.
    """
    lib = _load()
    b, s_q, h_q, d = (int(x) for x in q.shape)
    num_pages, page, h_kv, d2 = (int(x) for x in k_cache.shape)
    if d2 != d:
        raise ValueError("q and k_cache disagree on the latent width")
    qn = _bf16_bits(q)
    kn = _bf16_bits(k_cache)
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(cache_seqlens, dtype=np.int32))
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    kb = None if kv_begin is None else np.ascontiguousarray(np.asarray(kv_begin, dtype=np.int32))
    ke = None if kv_end is None else np.ascontiguousarray(np.asarray(kv_end, dtype=np.int32))
    n = rows.shape[0]
    out = np.zeros((n, dv), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    scale = d ** -0.5 if softmax_scale is None else float(softmax_scale)
    ptr = lambda a: None if a is None else a.ctypes.data
    rc = lib.oracle_mla_decode_rows(
        ptr(qn), s_q * h_q * d, h_q * d, d, b, s_q, h_q, d,
        ptr(kn), num_pages, page, h_kv,
        ptr(bt), bt.shape[1], ptr(sl), ptr(kb), ptr(ke),
        dv, scale, int(bool(causal)),
        ptr(rows), n, ptr(out), ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle rejected its inputs (status {rc})")
    return out, lse


def e4m3_to_float64(codes) -> np.ndarray:
    """OCP E4M3 codes (uint8 array) -> float64 values (NaN for 0x7F / 0xFF)."""
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(c.shape, dtype=np.float64)
    if _load().oracle_e4m3_to_double(c.ctypes.data, c.size, out.ctypes.data) != 0:
        raise ValueError("bad arguments")
    return out


def _u8(t) -> np.ndarray:
    import torch
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype != torch.uint8:
            t = t.view(torch.uint8)
        return t.numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.uint8))


def mla_decode_rows_fp8(q, k8, k_scale, block_table, cache_seqlens, rows, dv: int = 512,
                        softmax_scale: Optional[float] = None, causal: bool = True,
                        kv_begin=None, kv_end=None):
    """fp64 decode of the listed rows over an FP8 latent cache.

    k8 [num_pages, page, h_kv, d] uint8 E4M3 codes (or a float8_e4m3fn tensor), k_scale
    [h_kv, num_pages, page] fp32; the latent row of a token is scale * e4m3(code).  Other
    arguments and the result as in mla_decode_rows.
    """
    lib = _load()
    b, s_q, h_q, d = (int(x) for x in q.shape)
    num_pages, page, h_kv, d2 = (int(x) for x in k8.shape)
    if d2 != d:
        raise ValueError("q and k8 disagree on the latent width")
    qn = _bf16_bits(q)
    kn = _u8(k8)
    import torch
    ks = k_scale.detach().cpu().contiguous().numpy() if isinstance(k_scale, torch.Tensor) else np.asarray(k_scale)
    ks = np.ascontiguousarray(ks, dtype=np.float32)
    if ks.shape != (h_kv, num_pages, page):
        raise ValueError("k_scale must be [h_kv, num_pages, page]")
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(cache_seqlens, dtype=np.int32))
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    kb = None if kv_begin is None else np.ascontiguousarray(np.asarray(kv_begin, dtype=np.int32))
    ke = None if kv_end is None else np.ascontiguousarray(np.asarray(kv_end, dtype=np.int32))
    n = rows.shape[0]
    out = np.zeros((n, dv), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    scale = d ** -0.5 if softmax_scale is None else float(softmax_scale)
    ptr = lambda a: None if a is None else a.ctypes.data
    rc = lib.oracle_mla_decode_rows_fp8(
        ptr(qn), s_q * h_q * d, h_q * d, d, b, s_q, h_q, d,
        ptr(kn), ptr(ks), num_pages, page, h_kv,
        ptr(bt), bt.shape[1], ptr(sl), ptr(kb), ptr(ke),
        dv, scale, int(bool(causal)),
        ptr(rows), n, ptr(out), ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle rejected its inputs (status {rc})")
    return out, lse


def mla_decode_rows_sparse(q, k_cache, block_table, cache_seqlens, row_ptr, col_idx, rows, dv: int = 512,
                           softmax_scale: Optional[float] = None, causal: bool = True,
                           kv_begin=None, kv_end=None):
    """fp64 token-level sparse decode of the listed rows.

    row_ptr [batch * s_q + 1] int32 (non-decreasing), col_idx [nnz] int32: query token
    (b, s) attends to the positions col_idx[row_ptr[b * s_q + s] : row_ptr[b * s_q + s + 1]]
    that lie in [0, n) with n the row's visible length (causal rule as in the dense
    decode); other entries are pruned, repeated entries count once per listing.  kv_begin /
    kv_end (optional [b]) select list entries by their index in the list.  Other arguments
    and the result as in mla_decode_rows.
    """
    lib = _load()
    b, s_q, h_q, d = (int(x) for x in q.shape)
    num_pages, page, h_kv, d2 = (int(x) for x in k_cache.shape)
    if d2 != d:
        raise ValueError("q and k_cache disagree on the latent width")
    qn = _bf16_bits(q)
    kn = _bf16_bits(k_cache)
    bt = np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(cache_seqlens, dtype=np.int32))
    rp = np.ascontiguousarray(np.asarray(row_ptr, dtype=np.int32).reshape(-1))
    ci = np.ascontiguousarray(np.asarray(col_idx, dtype=np.int32).reshape(-1))
    if rp.shape[0] != b * s_q + 1 or int(rp[-1]) > ci.shape[0]:
        raise ValueError("row_ptr must have batch * s_q + 1 entries within col_idx")
    if ci.shape[0] == 0:
        ci = np.zeros(1, dtype=np.int32)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    kb = None if kv_begin is None else np.ascontiguousarray(np.asarray(kv_begin, dtype=np.int32))
    ke = None if kv_end is None else np.ascontiguousarray(np.asarray(kv_end, dtype=np.int32))
    n = rows.shape[0]
    out = np.zeros((n, dv), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    scale = d ** -0.5 if softmax_scale is None else float(softmax_scale)
    ptr = lambda a: None if a is None else a.ctypes.data
    rc = lib.oracle_mla_decode_rows_sparse(
        ptr(qn), s_q * h_q * d, h_q * d, d, b, s_q, h_q, d,
        ptr(kn), num_pages, page, h_kv,
        ptr(bt), bt.shape[1], ptr(sl), ptr(rp), ptr(ci), ptr(kb), ptr(ke),
        dv, scale, int(bool(causal)),
        ptr(rows), n, ptr(out), ptr(lse))
    if rc != 0:
        raise ValueError(f"oracle rejected its inputs (status {rc})")
    return out, lse


def mla_decode_sparse(q, k_cache, block_table, cache_seqlens, row_ptr, col_idx, dv: int = 512,
                      softmax_scale: Optional[float] = None, causal: bool = True,
                      kv_begin=None, kv_end=None):
    """fp64 token-level sparse decode of the whole batch (see mla_decode_rows_sparse):
    out [b, s_q, h_q, dv], lse [b, h_q, s_q]."""
    b, s_q, h_q, _ = (int(x) for x in q.shape)
    out, lse = mla_decode_rows_sparse(q, k_cache, block_table, cache_seqlens, row_ptr, col_idx,
                                      all_rows(b, s_q, h_q), dv, softmax_scale, causal, kv_begin, kv_end)
    out = out.reshape(b, s_q, h_q, dv)
    lse = lse.reshape(b, s_q, h_q).transpose(0, 2, 1).copy()
    return out, lse


def mla_decode_fp8(q, k8, k_scale, block_table, cache_seqlens, dv: int = 512,
                   softmax_scale: Optional[float] = None, causal: bool = True,
                   kv_begin=None, kv_end=None):
    """fp64 decode of the whole batch over an FP8 latent cache (see mla_decode_rows_fp8)."""
    b, s_q, h_q, _ = (int(x) for x in q.shape)
    out, lse = mla_decode_rows_fp8(q, k8, k_scale, block_table, cache_seqlens, all_rows(b, s_q, h_q),
                                   dv, softmax_scale, causal, kv_begin, kv_end)
    out = out.reshape(b, s_q, h_q, dv)
    lse = lse.reshape(b, s_q, h_q).transpose(0, 2, 1).copy()
    return out, lse


def all_rows(batch: int, s_q: int, h_q: int) -> np.ndarray:
    """Every (b, s, h) triple in output order."""
    b, s, h = np.meshgrid(np.arange(batch), np.arange(s_q), np.arange(h_q), indexing="ij")
    return np.stack([b.ravel(), s.ravel(), h.ravel()], axis=1).astype(np.int32)


def mla_decode(q, k_cache, block_table, cache_seqlens, dv: int = 512,
               softmax_scale: Optional[float] = None, causal: bool = True,
               kv_begin=None, kv_end=None):
    """fp64 decode of the whole batch: out [b, s_q, h_q, dv], lse [b, h_q, s_q]."""
    b, s_q, h_q, _ = (int(x) for x in q.shape)
    out, lse = mla_decode_rows(q, k_cache, block_table, cache_seqlens, all_rows(b, s_q, h_q),
                               dv, softmax_scale, causal, kv_begin, kv_end)
    out = out.reshape(b, s_q, h_q, dv)
    lse = lse.reshape(b, s_q, h_q).transpose(0, 2, 1).copy()
    return out, lse


def combine(lse_parts, o_parts):
    """Log-sum-exp merge of split partials: the online-softmax rescaling of partial
    results by a later maximum (dpshk.com notes, section 2.2) applied across the splits
    that get_mla_metadata's num_splits counts ("OpenSourceWeek Day 1 - FlashMLA", section
    V.2).

    lse_parts [k, ...], o_parts [k, ..., dv] float64.  lse = ln sum_k exp(lse_k),
    out = sum_k exp(lse_k - lse) o_k.  Partials with lse_k = -inf carry no weight; when
    all are -inf the result is out = 0, lse = -inf.
    """
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    o_parts = np.asarray(o_parts, dtype=np.float64)
    m = np.max(lse_parts, axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.exp(lse_parts - m_safe)                 # exp(-inf) = 0
    tot = np.sum(w, axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, tot, 1.0)), -np.inf)
    scale = np.where(finite, np.exp(lse_parts - np.where(finite, lse, 0.0)), 0.0)
    out = np.sum(scale[..., None] * o_parts, axis=0)
    return out, lse


def absorb_query(q_nope, q_rope, w_uk):
    """Query carried into latent space ("DeepSeek FlashMLA ... practitioner notes", dpshk.com,
    section 2.1: the per-head key is the up-projection W^UK_h of the latent row c, so the
    score q_h . (W^UK_h c) is (W^UK_h^T q_h) . c and the projection moves onto the query).

    q_nope [T, H, 128], q_rope [T, H, 64], w_uk [H, 128, 512] (head h's key up-projection,
    rows = key column d, columns = latent column); any float dtype, computed in fp64.
    Returns q' [T, H, 576]: q'[t, h, c] = sum_d q_nope[t, h, d] w_uk[h, d, c] for c < 512,
    then the rope columns unchanged (the positional key part is stored as is in the cache).
    """
    qn = np.asarray(q_nope, dtype=np.float64)
    qr = np.asarray(q_rope, dtype=np.float64)
    w = np.asarray(w_uk, dtype=np.float64)
    return np.concatenate([np.einsum("thd,hdc->thc", qn, w), qr], axis=-1)


def absorb_output(o_latent, w_uv):
    """Attention output taken out of latent space (same notes, section 2.1: the value is
    W^UV_h c, and the weighted sum commutes with the projection, so it is applied once to
    the latent output).  o_latent [T, H, 512], w_uv [H, 128, 512] (head h's value
    up-projection, rows = output column d).  Returns o [T, H, 128] in fp64:
    o[t, h, d] = sum_c w_uv[h, d, c] o_latent[t, h, c]."""
    o = np.asarray(o_latent, dtype=np.float64)
    w = np.asarray(w_uv, dtype=np.float64)
    return np.einsum("thc,hdc->thd", o, w)
