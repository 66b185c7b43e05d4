"""mla_decode_paged_static: decode for callers that cannot allocate device memory.

Such callers (a framework that owns the whole device-memory budget, a server that
reserves everything at start-up, a real-time loop that must not block in an allocator)
get a decode entry point whose split scratch is a fixed static device array carried by
the library.  These tests call it through the C ABI and check it against the regular
entry point, which uses a caller-provided workspace, on two calls in a row (the second
call reuses the array the first one left behind).  This file sorts last so that a run
stopping at the first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from paged_mla_decode_11_b200 import ops
from paged_mla_decode_11_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
LSE_RTOL = 1e-4


def static_entry():
    lib = ops.load_library()
    fn = lib.mla_decode_paged_static
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    fn.argtypes = [P, P, I, I, I, I, P, I64, I, I, P, I64, P, I, P, I, P, ctypes.c_float, I, P, P,
                   ctypes.c_uint, P]
    fn.restype = I
    return lib, fn


def call_static(fn, d, tile, splits, w, out, lse):
    q = d["q"]
    strides = (ctypes.c_int64 * 3)(q.stride(0), q.stride(1), q.stride(2))
    b, s_q, h_q, dd = q.shape
    num_pages, page, h_kv, _ = d["k_cache"].shape
    return fn(q.data_ptr(), strides, b, s_q, h_q, dd, d["k_cache"].data_ptr(), num_pages, page, h_kv,
              d["block_table"].data_ptr(), d["block_table"].stride(0), d["cache_seqlens"].data_ptr(), 512,
              tile.data_ptr(), tile.shape[0], splits.data_ptr(), w.scale, int(w.causal), out.data_ptr(),
              lse.data_ptr(), 0, torch.cuda.current_stream().cuda_stream)


def close(out, lse, ref_out, ref_lse):
    o, r = out.double().cpu(), ref_out.double().cpu()
    assert (o - r).abs().max().item() <= OUT_TOL * r.abs().max().item()
    l, rl = lse.double().cpu().numpy(), ref_lse.double().cpu().numpy()
    np.testing.assert_array_equal(np.isneginf(l), np.isneginf(rl))
    fin = np.isfinite(rl)
    assert (np.abs(l[fin] - rl[fin]) / np.maximum(np.abs(rl[fin]), 1.0)).max() <= LSE_RTOL


@pytest.mark.parametrize("kernel_rows", [(1, 16), (1, 24)], ids=["16-rows", "24-rows"])
def test_static_scratch_matches_workspace_entry_point(kernel_rows):
    s_q, h_q = kernel_rows
    w = W.custom(4, s_q, h_q, 1, [3000, 1, 500, 64], causal=True)
    x = W.make_inputs(w, seed=17)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    tile, splits = ops.get_mla_metadata(d["cache_seqlens"], w.rows_per_kv_head, 1)
    assert int(splits[1] - splits[0]) > 1          # the long sequence is split: scratch is used
    ref_out, ref_lse = ops.mla_decode_paged(d["q"], d["k_cache"], d["block_table"], d["cache_seqlens"], 512,
                                            tile, splits, softmax_scale=w.scale, causal=True)
    lib, fn = static_entry()
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        assert call_static(fn, d, tile, splits, w, out, lse) == 0
        # the array's status block: no device-side wait of this call gave up
        assert lib.mla_query_status_static(torch.cuda.current_stream().cuda_stream) == 0
        close(out, lse, ref_out, ref_lse)


def test_static_scratch_rejects_shapes_beyond_its_size():
    lib, fn = static_entry()
    strides = (ctypes.c_int64 * 3)(576 * 128, 576 * 128, 576)
    # 2048 sequences x 128 rows of fp32 partials need far more than the static array
    rc = fn(None, strides, 2048, 1, 128, 576, None, 1, 64, 1, None, 1, None, 512, None, 148, None,
            ctypes.c_float(0.04), 1, None, None, 0, None)
    assert rc == -3
    assert b"static scratch holds" in lib.mla_last_error_string()
