"""Python binding of libpagedmla.so: argument marshalling only.

Every step of the decode path runs in the library's CUDA kernels; this module checks
tensor dtypes, devices and shapes, allocates outputs with torch and passes raw pointers
and the current CUDA stream.  There is no CPU fallback: without the built library every
call raises.

The call sequence mirrors the pages' FlashMLA usage ("OpenSourceWeek Day 1 - FlashMLA",
section V.2):

    tile_metadata, num_splits = get_mla_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv)
    out, lse = flash_mla_with_kvcache(q, k_cache, block_table, cache_seqlens, dv,
                                      tile_metadata, num_splits, causal=True)
"""

from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedmla.so")

MLA_OK = 0
MLA_ERR_TIMEOUT = -4
MLA_FLAG_SKIP_COMBINE = 1
MLA_FLAG_WARP_MMA = 2
MLA_FLAG_TCGEN05 = 4
MLA_FLAG_ONE_SM = 8
KERNELS = {"auto": 0, "warp_mma": MLA_FLAG_WARP_MMA, "tcgen05": MLA_FLAG_TCGEN05, "one_sm": MLA_FLAG_ONE_SM}
PAGE = 64
D_QK = 576
D_V = 512
TILE_FIELDS = 8

EXPORTED = (
    "mla_device_sm_count", "mla_num_parts", "mla_metadata_size", "mla_get_metadata", "mla_workspace_size",
    "mla_decode_paged", "mla_combine", "mla_query_status", "mla_watchdog_selftest",
    "mla_last_error_string", "mla_decode_paged_static", "mla_query_status_static", "mla_decode_paged_fp8",
    "mla_merge_partials", "mla_absorb_query", "mla_absorb_output", "mla_get_metadata_csr", "mla_decode_sparse",
)

_lib = None
_lib_lock = threading.Lock()
_I64x3 = ctypes.c_int64 * 3


class MlaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"pagedmla error {code}: {msg}")
        self.code = code


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libpagedmla.so and declare its C signatures (raises if it is not built)."""
    global _lib
    lib = _lib
    if lib is not None:  # loaded: no lock on the per-call path
        return lib
    with _lib_lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with `python -m paged_mla_decode_11_b200.build`")
        lib = ctypes.CDLL(path)
        P, I, I64, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
        sig = {
            "mla_device_sm_count": [I, P],
            "mla_num_parts": [I, I, I, P],
            "mla_metadata_size": [I, I, I, P],
            "mla_get_metadata": [P, I, I, I, P, P, P],
            "mla_workspace_size": [I, I, I, I, I, P],
            "mla_decode_paged": [P, P, I, I, I, I, P, I64, I, I, P, I64, P, I, P, I, P,
                                 ctypes.c_float, I, P, P, P, ctypes.c_size_t, ctypes.c_uint, P],
            "mla_combine": [P, I, I, I, I, I, I, P, ctypes.c_size_t, P, P, P],
            "mla_query_status": [P, P],
            "mla_watchdog_selftest": [P, U64, P],
            "mla_query_status_static": [P],
            "mla_merge_partials": [P, P, I, I, I, I, I, P, P, P],
            "mla_absorb_query": [P, P, P, P, P, I, I, P, P],
            "mla_absorb_output": [P, P, P, I, I, P, P],
            "mla_decode_paged_fp8": [P, P, I, I, I, I, P, P, I64, I, I, P, I64, P, I, P, I, P,
                                     ctypes.c_float, I, P, P, P, ctypes.c_size_t, ctypes.c_uint, P],
            "mla_get_metadata_csr": [P, I, I, I, P, P, P],
            "mla_decode_sparse": [P, P, I, I, I, I, P, I64, I, I, P, I64, P, P, P, I, P, I, P,
                                  ctypes.c_float, I, P, P, P, ctypes.c_size_t, ctypes.c_uint, P],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = I
        lib.mla_last_error_string.argtypes = []
        lib.mla_last_error_string.restype = ctypes.c_char_p
        _lib = lib
        return lib


def _check(rc: int) -> None:
    if rc != MLA_OK:
        msg = load_library().mla_last_error_string().decode(errors="replace")
        raise MlaError(rc, msg)


def _stream_ptr(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _require_cuda(t: torch.Tensor, name: str, dtype: torch.dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")


_sm_count: dict = {}


def device_sm_count(device: Optional[torch.device] = None) -> int:
    n = _sm_count.get(device)  # keyed by what the caller passed, then by device index
    if n is not None:
        return n
    dev = torch.cuda.current_device() if device is None else torch.device(device).index
    if dev not in _sm_count:
        lib = load_library()
        c = ctypes.c_int(0)
        _check(lib.mla_device_sm_count(dev, ctypes.byref(c)))
        _sm_count[dev] = c.value
    if device is not None:
        _sm_count[device] = _sm_count[dev]
    return _sm_count[dev]


_parts_cache: dict = {}


def num_parts_for(num_sms: int, rows_per_kv_head: int, h_kv: int) -> int:
    key = (num_sms, rows_per_kv_head, h_kv)
    if key not in _parts_cache:  # a pure function of its arguments: asked once per shape
        lib = load_library()
        n = ctypes.c_int(0)
        _check(lib.mla_num_parts(num_sms, rows_per_kv_head, h_kv, ctypes.byref(n)))
        _parts_cache[key] = n.value
    return _parts_cache[key]


def metadata_size(batch: int, rows_per_kv_head: int, h_kv: int) -> int:
    """Part count get_mla_metadata plans on the current CUDA device (tile_metadata rows)."""
    n = ctypes.c_int(0)
    _check(load_library().mla_metadata_size(batch, rows_per_kv_head, h_kv, ctypes.byref(n)))
    return n.value


def get_mla_metadata(cache_seqlens: torch.Tensor, rows_per_kv_head: int, h_kv: int,
                     num_parts: Optional[int] = None, tile_metadata: Optional[torch.Tensor] = None,
                     num_splits: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV plan for one decode step: (tile_metadata [num_parts, 8], num_splits [b+1]).

    ``tile_metadata`` and ``num_splits`` may be passed to reuse buffers (contiguous int32 of
    those shapes on the same device); otherwise they are allocated."""
    _require_cuda(cache_seqlens, "cache_seqlens", torch.int32)
    shape = cache_seqlens.shape
    if len(shape) != 1 or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous 1-D int32 tensor")
    dev = cache_seqlens.device
    if num_parts is None:
        num_parts = num_parts_for(device_sm_count(dev), rows_per_kv_head, h_kv)
    batch = shape[0]
    if tile_metadata is None:
        tile_metadata = torch.empty(num_parts, TILE_FIELDS, dtype=torch.int32, device=dev)
    else:
        _require_cuda(tile_metadata, "tile_metadata", torch.int32)
        if tile_metadata.shape != (num_parts, TILE_FIELDS) or not tile_metadata.is_contiguous():
            raise ValueError(f"tile_metadata must be a contiguous [{num_parts}, {TILE_FIELDS}] tensor")
    if num_splits is None:
        num_splits = torch.empty(batch + 1, dtype=torch.int32, device=dev)
    else:
        _require_cuda(num_splits, "num_splits", torch.int32)
        if num_splits.shape != (batch + 1,) or not num_splits.is_contiguous():
            raise ValueError("num_splits must be a contiguous [batch + 1] tensor")
    _check(load_library().mla_get_metadata(cache_seqlens.data_ptr(), batch, rows_per_kv_head, num_parts,
                                           tile_metadata.data_ptr(), num_splits.data_ptr(), _stream_ptr(dev)))
    return tile_metadata, num_splits


def get_mla_metadata_csr(row_ptr: torch.Tensor, rows_per_kv_head: int, h_kv: int,
                         num_parts: Optional[int] = None, tile_metadata: Optional[torch.Tensor] = None,
                         num_splits: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split plan for the token-level sparse decode: the balanced cuts over key lists whose
    lengths are the differences of ``row_ptr`` (contiguous int32 [n_lists + 1], one list per
    query token).  rows_per_kv_head = h_q / h_kv.  Returns (tile_metadata [num_parts, 8],
    num_splits [n_lists + 1]); buffers may be passed for reuse as in get_mla_metadata."""
    _require_cuda(row_ptr, "row_ptr", torch.int32)
    if row_ptr.dim() != 1 or row_ptr.numel() < 2 or not row_ptr.is_contiguous():
        raise ValueError("row_ptr must be a contiguous 1-D int32 tensor of n_lists + 1 offsets")
    dev = row_ptr.device
    n_lists = row_ptr.numel() - 1
    if num_parts is None:
        num_parts = num_parts_for(device_sm_count(dev), rows_per_kv_head, h_kv)
    if tile_metadata is None:
        tile_metadata = torch.empty(num_parts, TILE_FIELDS, dtype=torch.int32, device=dev)
    elif tile_metadata.shape != (num_parts, TILE_FIELDS) or not tile_metadata.is_contiguous():
        raise ValueError(f"tile_metadata must be a contiguous [{num_parts}, {TILE_FIELDS}] tensor")
    if num_splits is None:
        num_splits = torch.empty(n_lists + 1, dtype=torch.int32, device=dev)
    elif num_splits.shape != (n_lists + 1,) or not num_splits.is_contiguous():
        raise ValueError("num_splits must be a contiguous [n_lists + 1] tensor")
    _check(load_library().mla_get_metadata_csr(row_ptr.data_ptr(), n_lists, rows_per_kv_head, num_parts,
                                               tile_metadata.data_ptr(), num_splits.data_ptr(), _stream_ptr(dev)))
    return tile_metadata, num_splits


_ws_size_cache: dict = {}


def workspace_size(batch: int, s_q: int, h_q: int, h_kv: int, num_parts: int) -> int:
    key = (batch, s_q, h_q, h_kv, num_parts)
    if key not in _ws_size_cache:  # a pure function of the shape: asked once per shape
        n = ctypes.c_size_t(0)
        _check(load_library().mla_workspace_size(batch, s_q, h_q, h_kv, num_parts, ctypes.byref(n)))
        _ws_size_cache[key] = n.value
    return _ws_size_cache[key]


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """A zeroed scratch buffer for mla_decode_paged (its status block must start at 0)."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


_ws_cache: dict = {}


def _default_workspace(nbytes: int, device: torch.device) -> torch.Tensor:
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = new_workspace(nbytes, device)
        _ws_cache[key] = ws
    return ws


def mla_decode_paged(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor,
                     cache_seqlens: torch.Tensor, dv: int, tile_metadata: torch.Tensor,
                     num_splits: torch.Tensor, softmax_scale: Optional[float] = None,
                     causal: bool = False, workspace: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     skip_combine: bool = False, kernel: str = "auto") -> Tuple[torch.Tensor, torch.Tensor]:
    """Paged MLA decode.  q [b, s_q, h_q, 576] bf16, k_cache [pages, 64, h_kv, 576] bf16,
    block_table [b, w] int32, cache_seqlens [b] int32.  Returns (out [b, s_q, h_q, dv]
    bf16, lse [b, h_q, s_q] fp32).  The default softmax_scale is 576 ** -0.5.

    Without ``workspace`` a per-(device, stream) scratch buffer is reused; calls that may
    run concurrently on one stream's buffer must pass their own.  ``kernel`` is "auto"
    (the library's choice by shape), "warp_mma", "tcgen05" or "one_sm" (the 1-SM 64-row
    tcgen05 kernel where the CTA-pair kernel would apply)."""
    _require_cuda(q, "q", torch.bfloat16)
    _require_cuda(k_cache, "k_cache", torch.bfloat16)
    _require_cuda(block_table, "block_table", torch.int32)
    _require_cuda(cache_seqlens, "cache_seqlens", torch.int32)
    _require_cuda(tile_metadata, "tile_metadata", torch.int32)
    _require_cuda(num_splits, "num_splits", torch.int32)
    qshape, kshape, btshape = q.shape, k_cache.shape, block_table.shape
    if len(qshape) != 4 or len(kshape) != 4 or len(btshape) != 2:
        raise ValueError("q and k_cache must be 4-D, block_table 2-D")
    b, s_q, h_q, d = qshape
    num_pages, page, h_kv, d2 = kshape
    if d2 != d:
        raise ValueError("q and k_cache disagree on the latent width")
    qst = q.stride()
    if qst[3] != 1:
        raise ValueError("q's last dimension must be contiguous")
    if not k_cache.is_contiguous():
        raise ValueError("k_cache must be contiguous")
    btst = block_table.stride()
    if btst[1] != 1 or btshape[0] != b:
        raise ValueError("block_table must be [batch, max_pages] with contiguous rows")
    if cache_seqlens.shape != (b,) or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous [batch] tensor")
    tshape = tile_metadata.shape
    if len(tshape) != 2 or tshape[1] != TILE_FIELDS or not tile_metadata.is_contiguous():
        raise ValueError("tile_metadata must be a contiguous [num_parts, 8] tensor")
    if num_splits.shape != (b + 1,):
        raise ValueError("num_splits must be [batch + 1]")
    flags = KERNELS.get(kernel)
    if flags is None:
        raise ValueError(f"kernel must be one of {sorted(KERNELS)}")
    if skip_combine:
        flags |= MLA_FLAG_SKIP_COMBINE
    dev = q.device
    num_parts = tshape[0]
    scale = float(d) ** -0.5 if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty(b, s_q, h_q, dv, dtype=torch.bfloat16, device=dev)
    elif out.shape != (b, s_q, h_q, dv) or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [b, s_q, h_q, dv] tensor")
    if lse is None:
        lse = torch.empty(b, h_q, s_q, dtype=torch.float32, device=dev)
    elif lse.shape != (b, h_q, s_q) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [b, h_q, s_q] tensor")
    if workspace is None:
        workspace = _default_workspace(workspace_size(b, s_q, h_q, h_kv, num_parts), dev)
    _check(load_library().mla_decode_paged(
        q.data_ptr(), _I64x3(qst[0], qst[1], qst[2]), b, s_q, h_q, d, k_cache.data_ptr(), num_pages, page,
        h_kv, block_table.data_ptr(), btst[0], cache_seqlens.data_ptr(), dv, tile_metadata.data_ptr(),
        num_parts, num_splits.data_ptr(), scale, int(bool(causal)), out.data_ptr(), lse.data_ptr(),
        workspace.data_ptr(), workspace.numel(), flags, _stream_ptr(dev)))
    return out, lse


# The pages' name for the decode call.
flash_mla_with_kvcache = mla_decode_paged


def mla_decode_paged_fp8(q: torch.Tensor, k8: torch.Tensor, k_scale: torch.Tensor, block_table: torch.Tensor,
                         cache_seqlens: torch.Tensor, dv: int, tile_metadata: torch.Tensor,
                         num_splits: torch.Tensor, softmax_scale: Optional[float] = None,
                         causal: bool = False, workspace: Optional[torch.Tensor] = None,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                         skip_combine: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Paged MLA decode over an FP8 latent cache: k8 [pages, 64, h_kv, 576] uint8 E4M3 codes
    (or float8_e4m3fn), k_scale [h_kv, pages, 64] fp32, one scale per token and latent head;
    up to 16 query rows per latent head.  Other arguments and results as mla_decode_paged."""
    _require_cuda(q, "q", torch.bfloat16)
    if k8.dtype == torch.float8_e4m3fn:
        k8 = k8.view(torch.uint8)
    _require_cuda(k8, "k8", torch.uint8)
    _require_cuda(k_scale, "k_scale", torch.float32)
    _require_cuda(block_table, "block_table", torch.int32)
    _require_cuda(cache_seqlens, "cache_seqlens", torch.int32)
    _require_cuda(tile_metadata, "tile_metadata", torch.int32)
    _require_cuda(num_splits, "num_splits", torch.int32)
    if q.dim() != 4 or k8.dim() != 4 or block_table.dim() != 2:
        raise ValueError("q and k8 must be 4-D, block_table 2-D")
    b, s_q, h_q, d = q.shape
    num_pages, page, h_kv, d2 = k8.shape
    if d2 != d:
        raise ValueError("q and k8 disagree on the latent width")
    if q.stride(3) != 1:
        raise ValueError("q's last dimension must be contiguous")
    if not k8.is_contiguous():
        raise ValueError("k8 must be contiguous")
    if k_scale.shape != (h_kv, num_pages, page) or not k_scale.is_contiguous():
        raise ValueError("k_scale must be a contiguous [h_kv, num_pages, page] tensor")
    if block_table.stride(1) != 1 or block_table.shape[0] != b:
        raise ValueError("block_table must be [batch, max_pages] with contiguous rows")
    if cache_seqlens.shape != (b,) or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous [batch] tensor")
    tshape = tile_metadata.shape
    if len(tshape) != 2 or tshape[1] != TILE_FIELDS or not tile_metadata.is_contiguous():
        raise ValueError("tile_metadata must be a contiguous [num_parts, 8] tensor")
    if num_splits.shape != (b + 1,):
        raise ValueError("num_splits must be [batch + 1]")
    dev = q.device
    num_parts = tshape[0]
    scale = float(d) ** -0.5 if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty(b, s_q, h_q, dv, dtype=torch.bfloat16, device=dev)
    elif out.shape != (b, s_q, h_q, dv) or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [b, s_q, h_q, dv] tensor")
    if lse is None:
        lse = torch.empty(b, h_q, s_q, dtype=torch.float32, device=dev)
    elif lse.shape != (b, h_q, s_q) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [b, h_q, s_q] tensor")
    if workspace is None:
        workspace = _default_workspace(workspace_size(b, s_q, h_q, h_kv, num_parts), dev)
    qst = q.stride()
    _check(load_library().mla_decode_paged_fp8(
        q.data_ptr(), _I64x3(qst[0], qst[1], qst[2]), b, s_q, h_q, d, k8.data_ptr(), k_scale.data_ptr(),
        num_pages, page, h_kv, block_table.data_ptr(), block_table.stride(0), cache_seqlens.data_ptr(), dv,
        tile_metadata.data_ptr(), num_parts, num_splits.data_ptr(), scale, int(bool(causal)), out.data_ptr(),
        lse.data_ptr(), workspace.data_ptr(), workspace.numel(), MLA_FLAG_SKIP_COMBINE if skip_combine else 0,
        _stream_ptr(dev)))
    return out, lse


def mla_combine(num_splits: torch.Tensor, s_q: int, h_q: int, h_kv: int, num_parts: int,
                workspace: torch.Tensor, out: torch.Tensor, lse: torch.Tensor, dv: int = D_V) -> None:
    """Merge split partials left by mla_decode_paged(..., skip_combine=True) into out/lse."""
    _require_cuda(num_splits, "num_splits", torch.int32)
    b = num_splits.shape[0] - 1
    _check(load_library().mla_combine(num_splits.data_ptr(), b, s_q, h_q, h_kv, dv, num_parts,
                                      workspace.data_ptr(), workspace.numel(), out.data_ptr(),
                                      lse.data_ptr(), _stream_ptr(out.device)))


def mla_decode_sparse(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor,
                      cache_seqlens: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor, dv: int,
                      tile_metadata: torch.Tensor, num_splits: torch.Tensor,
                      softmax_scale: Optional[float] = None, causal: bool = False,
                      workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] = None, skip_combine: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Token-level sparse decode: query token (b, s) attends to the key positions
    col_idx[row_ptr[b * s_q + s] : row_ptr[b * s_q + s + 1]] of sequence b that it may see
    (others pruned).  row_ptr int32 [b * s_q + 1], col_idx int32 [nnz]; the plan comes from
    get_mla_metadata_csr(row_ptr, h_q // h_kv, h_kv).  Up to 16 query heads per latent head.
    Other arguments and results as mla_decode_paged; with skip_combine the split partials stay
    in the workspace (mla_combine over batch * s_q one-position lists merges them)."""
    for t, n in ((q, "q"), (k_cache, "k_cache")):
        _require_cuda(t, n, torch.bfloat16)
    for t, n in ((block_table, "block_table"), (cache_seqlens, "cache_seqlens"), (row_ptr, "row_ptr"),
                 (col_idx, "col_idx"), (tile_metadata, "tile_metadata"), (num_splits, "num_splits")):
        _require_cuda(t, n, torch.int32)
    if q.dim() != 4 or k_cache.dim() != 4 or block_table.dim() != 2:
        raise ValueError("q and k_cache must be 4-D, block_table 2-D")
    b, s_q, h_q, d = q.shape
    num_pages, page, h_kv, d2 = k_cache.shape
    if d2 != d:
        raise ValueError("q and k_cache disagree on the latent width")
    if q.stride(3) != 1 or not k_cache.is_contiguous():
        raise ValueError("q's last dimension and k_cache must be contiguous")
    if block_table.stride(1) != 1 or block_table.shape[0] != b:
        raise ValueError("block_table must be [batch, max_pages] with contiguous rows")
    if cache_seqlens.shape != (b,) or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous [batch] tensor")
    if row_ptr.shape != (b * s_q + 1,) or not row_ptr.is_contiguous() or not col_idx.is_contiguous():
        raise ValueError("row_ptr must be a contiguous [batch * s_q + 1] tensor, col_idx contiguous")
    tshape = tile_metadata.shape
    if len(tshape) != 2 or tshape[1] != TILE_FIELDS or not tile_metadata.is_contiguous():
        raise ValueError("tile_metadata must be a contiguous [num_parts, 8] tensor")
    if num_splits.shape != (b * s_q + 1,):
        raise ValueError("num_splits must be [batch * s_q + 1]")
    dev = q.device
    num_parts = tshape[0]
    scale = float(d) ** -0.5 if softmax_scale is None else float(softmax_scale)
    if out is None:
        out = torch.empty(b, s_q, h_q, dv, dtype=torch.bfloat16, device=dev)
    elif out.shape != (b, s_q, h_q, dv) or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 [b, s_q, h_q, dv] tensor")
    if lse is None:
        lse = torch.empty(b, h_q, s_q, dtype=torch.float32, device=dev)
    elif lse.shape != (b, h_q, s_q) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 [b, h_q, s_q] tensor")
    if workspace is None:
        workspace = _default_workspace(workspace_size(b, s_q, h_q, h_kv, num_parts), dev)
    col = col_idx if col_idx.numel() > 0 else torch.zeros(1, dtype=torch.int32, device=dev)
    qst = q.stride()
    _check(load_library().mla_decode_sparse(
        q.data_ptr(), _I64x3(qst[0], qst[1], qst[2]), b, s_q, h_q, d, k_cache.data_ptr(), num_pages, page, h_kv,
        block_table.data_ptr(), block_table.stride(0), cache_seqlens.data_ptr(), row_ptr.data_ptr(), col.data_ptr(),
        dv, tile_metadata.data_ptr(), num_parts, num_splits.data_ptr(), scale, int(bool(causal)), out.data_ptr(),
        lse.data_ptr(), workspace.data_ptr(), workspace.numel(), MLA_FLAG_SKIP_COMBINE if skip_combine else 0,
        _stream_ptr(dev)))
    return out, lse


def mla_merge_partials(o_parts: torch.Tensor, lse_parts: torch.Tensor, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Log-sum-exp merge of partial decodes over disjoint keys: o_parts [n, b, s_q, h_q, 512]
    bf16, lse_parts [n, b, h_q, s_q] fp32 -> (out [b, s_q, h_q, 512], lse [b, h_q, s_q])."""
    _require_cuda(o_parts, "o_parts", torch.bfloat16)
    _require_cuda(lse_parts, "lse_parts", torch.float32)
    if o_parts.dim() != 5 or lse_parts.dim() != 4:
        raise ValueError("o_parts must be [n, b, s_q, h_q, dv] and lse_parts [n, b, h_q, s_q]")
    n, b, s_q, h_q, dv = o_parts.shape
    if lse_parts.shape != (n, b, h_q, s_q):
        raise ValueError("lse_parts must be [n, b, h_q, s_q] matching o_parts")
    if not o_parts.is_contiguous() or not lse_parts.is_contiguous():
        raise ValueError("o_parts and lse_parts must be contiguous")
    dev = o_parts.device
    if out is None:
        out = torch.empty(b, s_q, h_q, dv, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(b, h_q, s_q, dtype=torch.float32, device=dev)
    _check(load_library().mla_merge_partials(o_parts.data_ptr(), lse_parts.data_ptr(), n, b, s_q, h_q, dv,
                                             out.data_ptr(), lse.data_ptr(), _stream_ptr(dev)))
    return out, lse


_I64x2 = ctypes.c_int64 * 2


def absorb_query(q_nope: torch.Tensor, q_rope: torch.Tensor, w_uk: torch.Tensor,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """q' = [W^UK^T q_nope ; q_rope] per token and head: q_nope [T, H, 128], q_rope [T, H, 64]
    (bf16, last dim contiguous), w_uk [H, 128, 512] -> q' [T, H, 576] bf16."""
    for t, n in ((q_nope, "q_nope"), (q_rope, "q_rope"), (w_uk, "w_uk")):
        _require_cuda(t, n, torch.bfloat16)
    T, H, dn = q_nope.shape
    if dn != 128 or q_rope.shape != (T, H, 64) or w_uk.shape != (H, 128, 512):
        raise ValueError("q_nope [T, H, 128], q_rope [T, H, 64], w_uk [H, 128, 512]")
    if q_nope.stride(2) != 1 or q_rope.stride(2) != 1 or not w_uk.is_contiguous():
        raise ValueError("innermost dimensions must be contiguous, w_uk contiguous")
    if out is None:
        out = torch.empty(T, H, 576, dtype=torch.bfloat16, device=q_nope.device)
    _check(load_library().mla_absorb_query(q_nope.data_ptr(), _I64x2(q_nope.stride(0), q_nope.stride(1)),
                                           q_rope.data_ptr(), _I64x2(q_rope.stride(0), q_rope.stride(1)),
                                           w_uk.data_ptr(), T, H, out.data_ptr(), _stream_ptr(q_nope.device)))
    return out


def absorb_output(o_latent: torch.Tensor, w_uv: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """o = W^UV o_latent per token and head: o_latent [T, H, 512] bf16 (last dim contiguous),
    w_uv [H, 128, 512] -> o [T, H, 128] bf16."""
    _require_cuda(o_latent, "o_latent", torch.bfloat16)
    _require_cuda(w_uv, "w_uv", torch.bfloat16)
    T, H, dc = o_latent.shape
    if dc != 512 or w_uv.shape != (H, 128, 512):
        raise ValueError("o_latent [T, H, 512], w_uv [H, 128, 512]")
    if o_latent.stride(2) != 1 or not w_uv.is_contiguous():
        raise ValueError("o_latent's last dimension and w_uv must be contiguous")
    if out is None:
        out = torch.empty(T, H, 128, dtype=torch.bfloat16, device=o_latent.device)
    _check(load_library().mla_absorb_output(o_latent.data_ptr(), _I64x2(o_latent.stride(0), o_latent.stride(1)),
                                            w_uv.data_ptr(), T, H, out.data_ptr(), _stream_ptr(o_latent.device)))
    return out


def query_status(workspace: torch.Tensor) -> int:
    """Synchronise the current stream; return 0 or MLA_ERR_TIMEOUT (and clear it)."""
    rc = load_library().mla_query_status(workspace.data_ptr(), _stream_ptr(workspace.device))
    if rc not in (MLA_OK, MLA_ERR_TIMEOUT):
        _check(rc)
    return rc


def watchdog_selftest(workspace: torch.Tensor, timeout_ns: int) -> None:
    """Run a bounded wait that can only time out (see mla_watchdog_selftest)."""
    _check(load_library().mla_watchdog_selftest(workspace.data_ptr(), int(timeout_ns),
                                                _stream_ptr(workspace.device)))
