"""GPU parity of the token-level sparse decode (mla_decode_sparse) against the fp64 sparse
oracle, through the C ABI.  Tolerances as for the dense decode: max |out - ref| <= 1e-2 *
max |ref|, LSE within relative 1e-4 (against max(|ref|, 1)), query tokens without a visible
listed key exactly out = 0 and lse = -inf."""

import numpy as np
import pytest
import torch

import oracle
from paged_mla_decode_11_b200 import ops
from paged_mla_decode_11_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
LSE_RTOL = 1e-4


def run_sparse(x, num_parts=None):
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    g = x["h_q"] // x["h_kv"]
    tile, splits = ops.get_mla_metadata_csr(d["row_ptr"], g, x["h_kv"], num_parts=num_parts)
    b, s_q, h_q, _ = d["q"].shape
    ws = ops.new_workspace(ops.workspace_size(b, s_q, h_q, x["h_kv"], tile.shape[0]), "cuda")
    out, lse = ops.mla_decode_sparse(d["q"], d["k_cache"], d["block_table"], d["cache_seqlens"], d["row_ptr"],
                                     d["col_idx"], 512, tile, splits, softmax_scale=x["softmax_scale"],
                                     causal=x["causal"], workspace=ws)
    torch.cuda.synchronize()
    assert ops.query_status(ws) == ops.MLA_OK, "a device-side wait timed out"
    return out, lse, splits


def check(out, lse, ref_out, ref_lse, rows=None):
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    inf = np.isneginf(ref_lse)
    np.testing.assert_array_equal(np.isneginf(l), inf)
    scale = max(np.abs(ref_out).max(), 1e-30)
    err = np.abs(o - ref_out).max()
    assert err <= OUT_TOL * scale, f"max abs err {err:.3e} > {OUT_TOL} * {scale:.3e}"
    fin = ~inf
    if fin.any():
        rel = np.abs(l[fin] - ref_lse[fin]) / np.maximum(np.abs(ref_lse[fin]), 1.0)
        assert rel.max() <= LSE_RTOL, f"lse rel err {rel.max():.3e}"
    empty = inf.transpose(0, 2, 1)
    if empty.any():
        assert (o[empty] == 0).all()
    return err / scale


def sparse_parity(x, **kw):
    out, lse, splits = run_sparse(x, **kw)
    ref_out, ref_lse = oracle.mla_decode_sparse(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"],
                                                x["row_ptr"], x["col_idx"], dv=512,
                                                softmax_scale=x["softmax_scale"], causal=x["causal"])
    return check(out, lse, ref_out, ref_lse), splits


SPARSE_CASES = [
    # (batch, s_q, h_q, h_kv, seqlens, topk, causal, pad)
    (2, 1, 16, 1, [37, 130], 16, True, False),             # lists shorter than one chunk
    (3, 1, 16, 1, [0, 500, 2000], 100, True, True),         # an empty sequence, -1 padding
    (2, 2, 16, 1, [66, 300], 40, True, False),              # causal multi-token (lse layout fold)
    (4, 1, 8, 1, [1000, 1, 64, 65], 300, False, True),      # g = 8, ragged lists, no causal
    (2, 2, 16, 2, [700, 1500], 250, True, False),           # two latent heads (g = 8)
    (3, 3, 4, 1, [20000, 3, 9000], 4096, True, True),       # long lists: many splits, s_q = 3
]


@pytest.mark.parametrize("case", SPARSE_CASES)
def test_sparse_parity(case):
    b, s_q, h_q, h_kv, lens, topk, causal, pad = case
    w = W.custom(b, s_q, h_q, h_kv, lens, causal=causal)
    x = W.make_inputs(w, seed=b + s_q + topk)
    x["row_ptr"], x["col_idx"] = W.make_sparse_lists(lens, s_q, topk, seed=topk, causal=causal, pad=pad)
    sparse_parity(x)


def test_sparse_parity_forced_splits():
    # a small part count forces every list over several parts, so the combine merges them
    lens = [3000, 5000, 100]
    x = W.make_inputs(W.custom(3, 2, 16, 1, lens, causal=True), seed=9)
    x["row_ptr"], x["col_idx"] = W.make_sparse_lists(lens, 2, 2048, seed=9)
    for parts in (1, 5, 37):
        sparse_parity(x, num_parts=parts)


def test_sparse_pruned_duplicate_and_unsorted_entries():
    lens = [300, 90]
    x = W.make_inputs(W.custom(2, 2, 16, 1, lens, causal=True), seed=4)
    lists = [
        [299, -1, 5, 5, 17, 400, 3, 298],           # s = 0 may not see 299; 400 is past the end
        [299, 0, 0, 0],                             # s = 1 sees 299
        [-1, -7, 90, 1000],                         # nothing visible
        [89, 88, 60, 2, 89],                        # duplicates, unsorted
    ]
    rp = np.zeros(5, dtype=np.int32)
    rp[1:] = np.cumsum([len(v) for v in lists])
    x["row_ptr"] = torch.tensor(rp)
    x["col_idx"] = torch.tensor(np.concatenate(lists).astype(np.int32))
    sparse_parity(x)


def test_sparse_full_lists_equal_the_dense_decode():
    # the full position list reduces the sparse decode to the dense one (same kernel family)
    lens = [200, 1000, 64]
    x = W.make_inputs(W.custom(3, 1, 16, 1, lens, causal=True), seed=12)
    x["row_ptr"], x["col_idx"] = W.make_sparse_lists(lens, 1, 10 ** 6, seed=0)
    out, lse, _ = run_sparse(x)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    tile, splits = ops.get_mla_metadata(d["cache_seqlens"], 16, 1)
    od, ld = ops.mla_decode_paged(d["q"], d["k_cache"], d["block_table"], d["cache_seqlens"], 512, tile, splits,
                                  softmax_scale=x["softmax_scale"], causal=True)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], dv=512,
                                         softmax_scale=x["softmax_scale"], causal=True)
    check(out, lse, ref_out, ref_lse)
    check(od, ld, ref_out, ref_lse)


def test_sparse_full_size_workload_sampled_rows():
    # the benchmark's workload at full size, in the launch configuration it times; the oracle
    # checks every head of a sample of query tokens, one by one
    x = W.make_inputs_sparse(W.SPARSE, W.SPARSE_TOPK, seed=0)
    out, lse, _ = run_sparse(x)
    rng = np.random.default_rng(0)
    toks = rng.choice(W.SPARSE.batch, 6, replace=False)
    rows = np.array([(b, 0, h) for b in toks for h in range(16)], dtype=np.int32)
    ref_o, ref_l = oracle.mla_decode_rows_sparse(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"],
                                                 x["row_ptr"], x["col_idx"], rows, dv=512,
                                                 softmax_scale=x["softmax_scale"], causal=True)
    o = out.double().cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    l = lse.double().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert np.abs(o - ref_o).max() <= OUT_TOL * np.abs(ref_o).max()
    assert (np.abs(l - ref_l) / np.maximum(np.abs(ref_l), 1.0)).max() <= LSE_RTOL
    assert torch.isfinite(out.float()).all()
