"""The Python binding's host logic, without a GPU: what it passes to the C ABI and what it
rejects before any call.

A recording stand-in replaces libpagedmla.so, and the binding's device check is relaxed to
its dtype part, so CPU tensors can stand in for device tensors.  (That the real library
loads and exports every declared entry point is tested in test_boundary.py.)
"""

import math

import pytest
import torch

from paged_mla_decode_11_b200 import ops


class _Recorder:
    def __init__(self, name, calls):
        self.name, self.calls = name, calls
        self.argtypes = self.restype = None

    def __call__(self, *args):
        self.calls.append((self.name, args))
        return 0


class FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        fn = _Recorder(name, self.calls)
        setattr(self, name, fn)
        return fn

    def last(self, name):
        return [a for n, a in self.calls if n == name][-1]


@pytest.fixture
def fake(monkeypatch):
    lib = FakeLib()
    monkeypatch.setattr(ops, "_lib", lib)
    # the binding memoises pure shape functions: keep the stand-in's answers out of them
    monkeypatch.setattr(ops, "_parts_cache", {})
    monkeypatch.setattr(ops, "_ws_size_cache", {})
    monkeypatch.setattr(ops, "_ws_cache", {})

    def dtype_only(t, name, dtype):
        if t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype} (got {t.dtype})")

    monkeypatch.setattr(ops, "_require_cuda", dtype_only)
    monkeypatch.setattr(ops, "_stream_ptr", lambda dev: 4242)
    monkeypatch.setattr(ops, "device_sm_count", lambda dev=None: 148)
    return lib


def _inputs(b=3, s_q=2, h_q=16, h_kv=1, pages=10, width=6):
    q = torch.zeros(b, s_q, h_q, 576, dtype=torch.bfloat16)
    kc = torch.zeros(pages, 64, h_kv, 576, dtype=torch.bfloat16)
    bt = torch.zeros(b, width, dtype=torch.int32)
    sl = torch.zeros(b, dtype=torch.int32)
    tile = torch.zeros(5, 8, dtype=torch.int32)
    splits = torch.zeros(b + 1, dtype=torch.int32)
    ws = torch.zeros(4096, dtype=torch.uint8)
    return q, kc, bt, sl, tile, splits, ws


def test_device_check_rejects_host_tensors():
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops._require_cuda(torch.zeros(1, dtype=torch.int32), "x", torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.get_mla_metadata(torch.zeros(4, dtype=torch.int32), 16, 1)


def test_metadata_marshalling_and_buffers(fake):
    sl = torch.zeros(7, dtype=torch.int32)
    tile, splits = ops.get_mla_metadata(sl, 64, 1, num_parts=9)
    assert tile.shape == (9, 8) and tile.dtype == torch.int32
    assert splits.shape == (8,) and splits.dtype == torch.int32
    args = fake.last("mla_get_metadata")
    assert args == (sl.data_ptr(), 7, 64, 9, tile.data_ptr(), splits.data_ptr(), 4242)
    # caller-owned buffers are filled in place and returned
    t2 = torch.empty(9, 8, dtype=torch.int32)
    s2 = torch.empty(8, dtype=torch.int32)
    r1, r2 = ops.get_mla_metadata(sl, 64, 1, num_parts=9, tile_metadata=t2, num_splits=s2)
    assert r1 is t2 and r2 is s2
    assert fake.last("mla_get_metadata")[4:6] == (t2.data_ptr(), s2.data_ptr())
    with pytest.raises(ValueError, match="tile_metadata"):
        ops.get_mla_metadata(sl, 64, 1, num_parts=9, tile_metadata=torch.empty(8, 8, dtype=torch.int32))
    with pytest.raises(ValueError, match="num_splits"):
        ops.get_mla_metadata(sl, 64, 1, num_parts=9, num_splits=torch.empty(7, dtype=torch.int32))
    with pytest.raises(TypeError):
        ops.get_mla_metadata(sl, 64, 1, num_parts=9, num_splits=torch.empty(8, dtype=torch.int64))
    with pytest.raises(ValueError, match="1-D"):
        ops.get_mla_metadata(torch.zeros(2, 3, dtype=torch.int32), 64, 1, num_parts=9)


def test_decode_marshalling(fake):
    q, kc, bt, sl, tile, splits, ws = _inputs()
    # a strided view of q: heads 2..17 of a wider buffer, padded rows
    big = torch.zeros(3, 2, 24, 640, dtype=torch.bfloat16)
    qv = big[:, :, 2:18, :576]
    out, lse = ops.mla_decode_paged(qv, kc, bt, sl, 512, tile, splits, causal=True, workspace=ws)
    assert out.shape == (3, 2, 16, 512) and out.dtype == torch.bfloat16
    assert lse.shape == (3, 16, 2) and lse.dtype == torch.float32
    a = fake.last("mla_decode_paged")
    assert a[0] == qv.data_ptr()
    assert list(a[1]) == [2 * 24 * 640, 24 * 640, 640]          # q strides (elements)
    assert a[2:6] == (3, 2, 16, 576)                            # batch, s_q, h_q, d
    assert a[6:10] == (kc.data_ptr(), 10, 64, 1)                # pool, pages, page size, h_kv
    assert a[10:14] == (bt.data_ptr(), 6, sl.data_ptr(), 512)   # block table + row stride, lengths, dv
    assert a[14:17] == (tile.data_ptr(), 5, splits.data_ptr())  # plan and its part count
    assert math.isclose(a[17], 576 ** -0.5, rel_tol=1e-12)      # default softmax scale
    assert a[18] == 1                                           # causal
    assert a[19:23] == (out.data_ptr(), lse.data_ptr(), ws.data_ptr(), 4096)
    assert a[23] == 0 and a[24] == 4242                         # flags, stream


@pytest.mark.parametrize("kernel,skip,flags", [
    ("auto", False, 0), ("auto", True, ops.MLA_FLAG_SKIP_COMBINE),
    ("warp_mma", False, ops.MLA_FLAG_WARP_MMA), ("tcgen05", True, ops.MLA_FLAG_TCGEN05 | ops.MLA_FLAG_SKIP_COMBINE),
])
def test_decode_flags_and_scale(fake, kernel, skip, flags):
    q, kc, bt, sl, tile, splits, ws = _inputs()
    ops.mla_decode_paged(q, kc, bt, sl, 512, tile, splits, softmax_scale=0.125, workspace=ws,
                         skip_combine=skip, kernel=kernel)
    a = fake.last("mla_decode_paged")
    assert a[23] == flags and a[17] == 0.125 and a[18] == 0


def test_decode_uses_given_outputs(fake):
    q, kc, bt, sl, tile, splits, ws = _inputs()
    out = torch.empty(3, 2, 16, 512, dtype=torch.bfloat16)
    lse = torch.empty(3, 16, 2, dtype=torch.float32)
    o, l = ops.mla_decode_paged(q, kc, bt, sl, 512, tile, splits, workspace=ws, out=out, lse=lse)
    assert o is out and l is lse


def _bad(**over):
    q, kc, bt, sl, tile, splits, ws = _inputs()
    args = dict(q=q, k_cache=kc, block_table=bt, cache_seqlens=sl, dv=512, tile_metadata=tile,
                num_splits=splits, workspace=ws)
    args.update(over)
    return args


@pytest.mark.parametrize("over,exc,msg", [
    (dict(q=torch.zeros(3, 16, 576, dtype=torch.bfloat16)), ValueError, "4-D"),
    (dict(q=torch.zeros(3, 2, 16, 512, dtype=torch.bfloat16)), ValueError, "latent width"),
    (dict(q=torch.zeros(3, 2, 576, 16, dtype=torch.bfloat16).transpose(2, 3)), ValueError, "last dimension"),
    (dict(k_cache=torch.zeros(10, 64, 1, 1152, dtype=torch.bfloat16)[..., :576]), ValueError, "k_cache must be contiguous"),
    (dict(block_table=torch.zeros(2, 6, dtype=torch.int32)), ValueError, "block_table"),
    (dict(block_table=torch.zeros(6, 3, dtype=torch.int32).t()), ValueError, "block_table"),
    (dict(cache_seqlens=torch.zeros(4, dtype=torch.int32)), ValueError, "cache_seqlens"),
    (dict(tile_metadata=torch.zeros(5, 7, dtype=torch.int32)), ValueError, "tile_metadata"),
    (dict(num_splits=torch.zeros(3, dtype=torch.int32)), ValueError, "num_splits"),
    (dict(out=torch.empty(3, 2, 16, 256, dtype=torch.bfloat16)), ValueError, "out must be"),
    (dict(out=torch.empty(3, 2, 16, 512, dtype=torch.float32)), ValueError, "out must be"),
    (dict(lse=torch.empty(3, 2, 16, dtype=torch.float32)), ValueError, "lse must be"),
    (dict(kernel="fastest"), ValueError, "kernel must be one of"),
    (dict(q=torch.zeros(3, 2, 16, 576, dtype=torch.float16)), TypeError, "q must be"),
    (dict(block_table=torch.zeros(3, 6, dtype=torch.int64)), TypeError, "block_table must be"),
])
def test_decode_rejects_before_calling_the_library(fake, over, exc, msg):
    with pytest.raises(exc, match=msg):
        ops.mla_decode_paged(**_bad(**over))
    assert not [n for n, _ in fake.calls if n == "mla_decode_paged"]


def test_fp8_decode_marshalling(fake):
    q, kc, bt, sl, tile, splits, ws = _inputs(b=3, s_q=1, h_q=16)
    k8 = torch.zeros(10, 64, 1, 576, dtype=torch.uint8)
    ks = torch.zeros(1, 10, 64, dtype=torch.float32)
    out, lse = ops.mla_decode_paged_fp8(q, k8, ks, bt, sl, 512, tile, splits, causal=True, workspace=ws,
                                        skip_combine=True)
    a = fake.last("mla_decode_paged_fp8")
    assert a[0] == q.data_ptr() and a[2:6] == (3, 1, 16, 576)
    assert a[6:11] == (k8.data_ptr(), ks.data_ptr(), 10, 64, 1)
    assert a[11:15] == (bt.data_ptr(), 6, sl.data_ptr(), 512)
    assert a[15:18] == (tile.data_ptr(), 5, splits.data_ptr())
    assert a[19] == 1 and a[20:24] == (out.data_ptr(), lse.data_ptr(), ws.data_ptr(), 4096)
    assert a[24] == ops.MLA_FLAG_SKIP_COMBINE and a[25] == 4242
    # float8 codes are passed as their bytes; a scale tensor of the wrong shape is refused
    ops.mla_decode_paged_fp8(q, k8.view(torch.float8_e4m3fn), ks, bt, sl, 512, tile, splits, workspace=ws)
    with pytest.raises(ValueError, match="k_scale"):
        ops.mla_decode_paged_fp8(q, k8, ks[:, :5], bt, sl, 512, tile, splits, workspace=ws)


def test_sparse_decode_and_plan_marshalling(fake):
    q, kc, bt, sl, tile, splits, ws = _inputs(b=3, s_q=2, h_q=16)
    row_ptr = torch.zeros(3 * 2 + 1, dtype=torch.int32)
    col = torch.zeros(40, dtype=torch.int32)
    t2, s2 = ops.get_mla_metadata_csr(row_ptr, 16, 1)
    a = fake.last("mla_get_metadata_csr")
    assert a[0] == row_ptr.data_ptr() and a[1:4] == (6, 16, ops.num_parts_for(148, 16, 1))
    assert t2.shape == (a[3], 8) and s2.shape == (7,)
    sp = torch.zeros(7, dtype=torch.int32)
    out, lse = ops.mla_decode_sparse(q, kc, bt, sl, row_ptr, col, 512, tile, sp, causal=True, workspace=ws)
    a = fake.last("mla_decode_sparse")
    assert a[2:6] == (3, 2, 16, 576) and a[6:10] == (kc.data_ptr(), 10, 64, 1)
    assert a[10:16] == (bt.data_ptr(), 6, sl.data_ptr(), row_ptr.data_ptr(), col.data_ptr(), 512)
    assert a[16:19] == (tile.data_ptr(), 5, sp.data_ptr()) and a[20] == 1 and a[25] == 0
    assert out.shape == (3, 2, 16, 512) and lse.shape == (3, 16, 2)
    # num_splits is per query token; row_ptr must have batch * s_q + 1 entries
    with pytest.raises(ValueError, match="num_splits"):
        ops.mla_decode_sparse(q, kc, bt, sl, row_ptr, col, 512, tile, splits, workspace=ws)
    with pytest.raises(ValueError, match="row_ptr"):
        ops.mla_decode_sparse(q, kc, bt, sl, row_ptr[:5], col, 512, tile, sp, workspace=ws)


def test_merge_and_absorb_marshalling(fake):
    o = torch.zeros(3, 2, 1, 16, 512, dtype=torch.bfloat16)
    l = torch.zeros(3, 2, 16, 1, dtype=torch.float32)
    out, lse = ops.mla_merge_partials(o, l)
    a = fake.last("mla_merge_partials")
    assert a[:7] == (o.data_ptr(), l.data_ptr(), 3, 2, 1, 16, 512) and a[7:9] == (out.data_ptr(), lse.data_ptr())
    with pytest.raises(ValueError, match="lse_parts"):
        ops.mla_merge_partials(o, l[:2])
    # the two column ranges of one [T, H, 192] projection: strides in elements
    qkv = torch.zeros(5, 4, 192, dtype=torch.bfloat16)
    w = torch.zeros(4, 128, 512, dtype=torch.bfloat16)
    q_abs = ops.absorb_query(qkv[..., :128], qkv[..., 128:], w)
    a = fake.last("mla_absorb_query")
    assert a[0] == qkv.data_ptr() and list(a[1]) == [768, 192] and a[2] == qkv.data_ptr() + 256
    assert list(a[3]) == [768, 192] and a[4] == w.data_ptr() and a[5:7] == (5, 4) and a[7] == q_abs.data_ptr()
    assert q_abs.shape == (5, 4, 576)
    lat = torch.zeros(5, 4, 512, dtype=torch.bfloat16)
    o2 = ops.absorb_output(lat, w)
    a = fake.last("mla_absorb_output")
    assert a[0] == lat.data_ptr() and list(a[1]) == [2048, 512] and a[2:6] == (w.data_ptr(), 5, 4, o2.data_ptr())
    with pytest.raises(ValueError):
        ops.absorb_output(lat[..., :256], w)
