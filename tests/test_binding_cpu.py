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
