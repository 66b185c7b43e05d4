"""Host-side checks of the C ABI: the library loads on a machine without a GPU, exports
every entry point include/pagedmla.h declares, and its host-only logic (part count,
workspace size, argument rejection) behaves as documented."""

import ctypes
import os
import re

import pytest

from paged_mla_decode_11_b200 import build as B
from paged_mla_decode_11_b200 import ops
from oracle import metadata as spec

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "pagedmla.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return ops.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*MLA_API\s+(?:const\s+)?\w+\s*\*?\s*(mla_\w+)\s*\(", text, re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 9, names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in pagedmla.h but not exported"
    assert set(names) == set(ops.EXPORTED)


def test_num_parts_matches_scheduler_granularity(lib):
    for sms in (1, 4, 132, 148):
        for R in (1, 16, 63, 64, 65, 128, 256, 1000):
            for h_kv in (1, 2, 3):
                assert ops.num_parts_for(sms, R, h_kv) == spec.num_parts_for(sms, R, h_kv)


def test_workspace_size(lib):
    n = ops.workspace_size(64, 1, 16, 1, 148)
    splits = 64 + 148
    R = 16
    lse_bytes = splits * R * 4
    o_off = (256 + lse_bytes + 255) // 256 * 256
    assert n == o_off + splits * R * 512 * 4


def test_host_side_rejections(lib):
    out = ctypes.c_size_t(0)
    assert lib.mla_workspace_size(4, 1, 16, 3, 10, ctypes.byref(out)) == -1   # h_q % h_kv
    assert b"multiple" in lib.mla_last_error_string()
    assert lib.mla_workspace_size(0, 1, 16, 1, 10, ctypes.byref(out)) == -1
    n = ctypes.c_int(0)
    assert lib.mla_num_parts(0, 16, 1, ctypes.byref(n)) == -1
    assert lib.mla_get_metadata(None, 4, 16, 10, None, None, None) == -1
    strides = (ctypes.c_int64 * 3)(576, 576, 576)
    # d != 576 and dv != 512 are refused before anything touches a device
    rc = lib.mla_decode_paged(16, strides, 1, 1, 16, 512, 16, 1, 64, 1, 16, 1, 16, 512, 16, 1, 16,
                              ctypes.c_float(0.04), 1, 16, 16, 256, 1 << 20, 0, None)
    assert rc == -2 and b"d must be 576" in lib.mla_last_error_string()
    rc = lib.mla_decode_paged(16, strides, 1, 1, 16, 576, 16, 1, 64, 1, 16, 1, 16, 256, 16, 1, 16,
                              ctypes.c_float(0.04), 1, 16, 16, 256, 1 << 20, 0, None)
    assert rc == -2 and b"dv must be 512" in lib.mla_last_error_string()
    rc = lib.mla_decode_paged(16, strides, 1, 1, 16, 576, 16, 1, 32, 1, 16, 1, 16, 512, 16, 1, 16,
                              ctypes.c_float(0.04), 1, 16, 16, 256, 1 << 20, 0, None)
    assert rc == -2 and b"page_size" in lib.mla_last_error_string()
    rc = lib.mla_decode_paged(16, strides, 1, 1, 16, 576, 16, 1, 64, 1, 16, 1, 16, 512, 16, 1, 16,
                              ctypes.c_float(-1.0), 1, 16, 16, 256, 1 << 20, 0, None)
    assert rc == -1 and b"softmax_scale" in lib.mla_last_error_string()


def test_metadata_size_host_checks(lib):
    n = ctypes.c_int(0)
    assert lib.mla_metadata_size(4, 16, 1, None) == -1
    assert lib.mla_metadata_size(0, 16, 1, ctypes.byref(n)) == -1
    assert b"batch" in lib.mla_last_error_string()
    assert lib.mla_metadata_size(4, 0, 1, ctypes.byref(n)) == -1
    # the same row bound as mla_get_metadata, so no part count is given for a shape the
    # scheduler call would refuse
    assert lib.mla_metadata_size(4, (1 << 20) + 1, 1, ctypes.byref(n)) == -1
    assert b"2^20" in lib.mla_last_error_string()
    # without a device it reports a CUDA error; with one, the part count of that device
    rc = lib.mla_metadata_size(4, 16, 1, ctypes.byref(n))
    assert rc in (0, -5)
    if rc == 0:
        assert n.value >= 1


def static_entry(lib):
    fn = lib.mla_decode_paged_static
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    fn.argtypes = [P, P, I, I, I, I, P, I64, I, I, P, I64, P, I, P, I, P, ctypes.c_float, I, P, P,
                   ctypes.c_uint, P]
    fn.restype = I
    return fn


def test_static_entry_host_rejections(lib):
    # Both refusals happen before the library touches a device.
    fn = static_entry(lib)
    strides = (ctypes.c_int64 * 3)(576 * 128, 576 * 128, 576)
    # leaving split partials unmerged is refused: they would stay in the library's own
    # array, which the caller cannot pass to mla_combine
    rc = fn(None, strides, 4, 1, 16, 576, None, 1, 64, 1, None, 1, None, 512, None, 148, None,
            ctypes.c_float(0.04), 1, None, None, ops.MLA_FLAG_SKIP_COMBINE, None)
    assert rc == -1
    assert b"MLA_FLAG_SKIP_COMBINE" in lib.mla_last_error_string()
    # 2048 sequences x 128 rows of fp32 partials need far more than the static array holds
    rc = fn(None, strides, 2048, 1, 128, 576, None, 1, 64, 1, None, 1, None, 512, None, 148, None,
            ctypes.c_float(0.04), 1, None, None, 0, None)
    assert rc == -3
    assert b"static scratch holds" in lib.mla_last_error_string()


def test_sparse_fp8_merge_absorb_host_rejections(lib):
    """The later entry points refuse bad arguments on the host, before any device call."""
    s3 = (ctypes.c_int64 * 3)(576, 576, 576)
    f = ctypes.c_float(0.04)
    # mla_decode_sparse(q, strides, b, s_q, h_q, d, k, pages, page, h_kv, bt, bt_stride, lens,
    #                   row_ptr, col_idx, dv, tile, parts, splits, scale, causal, out, lse, ws, ws_bytes, flags, stream)
    def sparse(h_q=16, d=576, dv=512, flags=0, row_ptr=16):
        return lib.mla_decode_sparse(16, s3, 1, 1, h_q, d, 16, 1, 64, 1, 16, 1, 16, row_ptr, 16, dv, 16, 1, 16, f, 1,
                                     16, 16, 256, 1 << 20, flags, None)
    assert sparse(d=512) == -2 and b"d must be 576" in lib.mla_last_error_string()
    assert sparse(h_q=32) == -2 and b"up to 16 query heads" in lib.mla_last_error_string()
    assert sparse(flags=2) == -1 and b"flags" in lib.mla_last_error_string()
    assert sparse(row_ptr=None) == -1 and b"null" in lib.mla_last_error_string()
    assert sparse(dv=256) == -2
    # mla_get_metadata_csr(row_ptr, n_lists, rows_per_kv_head, num_parts, tile, splits, stream)
    assert lib.mla_get_metadata_csr(None, 4, 16, 10, 16, 16, None) == -1
    assert lib.mla_get_metadata_csr(16, 0, 16, 10, 16, 16, None) == -1
    assert lib.mla_get_metadata_csr(16, 4, 0, 10, 16, 16, None) == -1
    assert lib.mla_get_metadata_csr(16, 4, 16, 0, 16, 16, None) == -1
    # mla_decode_paged_fp8: more than 16 rows per latent head is the 16-row kernel's limit
    rc = lib.mla_decode_paged_fp8(16, s3, 1, 1, 32, 576, 16, 16, 1, 64, 1, 16, 1, 16, 512, 16, 1, 16, f, 1, 16, 16,
                                  256, 1 << 20, 0, None)
    assert rc == -2 and b"16-row kernel" in lib.mla_last_error_string()
    # mla_merge_partials(o_parts, lse_parts, n, b, s_q, h_q, dv, out, lse, stream)
    assert lib.mla_merge_partials(None, 16, 2, 1, 1, 16, 512, 16, 16, None) == -1
    assert lib.mla_merge_partials(16, 16, 0, 1, 1, 16, 512, 16, 16, None) == -1
    assert lib.mla_merge_partials(16, 16, 2, 1, 1, 16, 256, 16, 16, None) == -2
    assert lib.mla_merge_partials(18, 16, 2, 1, 1, 16, 512, 16, 16, None) == -1     # misaligned partials
    # mla_absorb_query(q_nope, strides, q_rope, strides, w_uk, T, H, q_out, stream)
    s2 = (ctypes.c_int64 * 2)(192 * 16, 192)
    bad = (ctypes.c_int64 * 2)(192 * 16, 190)
    assert lib.mla_absorb_query(None, s2, 272, s2, 16, 4, 16, 16, None) == -1
    assert lib.mla_absorb_query(16, s2, 272, s2, 16, 0, 16, 16, None) == -1
    assert lib.mla_absorb_query(16, bad, 272, s2, 16, 4, 16, 16, None) == -1
    assert lib.mla_absorb_query(16, s2, 272, s2, 20, 4, 16, 16, None) == -1           # weights not 16-byte aligned
    # mla_absorb_output(o_latent, strides, w_uv, T, H, out, stream)
    assert lib.mla_absorb_output(None, s2, 16, 4, 16, 16, None) == -1
    assert lib.mla_absorb_output(16, s2, 16, 4, 0, 16, None) == -1
    assert lib.mla_absorb_output(16, bad, 16, 4, 16, 16, None) == -1
    assert lib.mla_absorb_output(16, s2, 24, 4, 16, 16, None) == -1
