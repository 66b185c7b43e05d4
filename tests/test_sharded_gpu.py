"""Sequence-sharded decode on one GPU: the shards are decoded one after another through the
C ABI (mla_decode_paged, causal only on the last shard) and merged by mla_merge_partials,
as the GPUs of a node would after their all-gather; the result must match the unsplit fp64
oracle within the usual tolerances.  Also the merge kernel alone against the oracle's
combine, with empty parts."""

import numpy as np
import pytest
import torch

import oracle
from paged_mla_decode_11_b200 import ops, sharded
from paged_mla_decode_11_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,s_q,h_q,lens", [
    (2, 1, 16, [5000, 130, 1]),
    (3, 2, 16, [4000, 64, 200]),
    (4, 1, 128, [3000, 700]),          # the CTA-pair kernel on each shard
    (4, 2, 64, [2000, 65, 0]),         # the 64-row kernel, an empty sequence
])
def test_sharded_decode_matches_unsplit(n, s_q, h_q, lens):
    x = W.make_inputs(W.custom(len(lens), s_q, h_q, 1, lens, causal=True), seed=n + h_q)
    q = x["q"].cuda()
    kc = x["k_cache"].cuda()
    outs, lses = [], []
    for k in range(n):
        bt, sl = sharded.shard_block_table(x["block_table"], lens, n, k, s_q=s_q)
        tile, splits = ops.get_mla_metadata(sl.cuda(), s_q * h_q, 1)
        o, l = ops.mla_decode_paged(q, kc, bt.cuda(), sl.cuda(), 512, tile, splits, softmax_scale=x["softmax_scale"],
                                    causal=(k == n - 1))
        outs.append(o)
        lses.append(l)
    out, lse = ops.mla_merge_partials(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], dv=512,
                                         softmax_scale=x["softmax_scale"], causal=True)
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    np.testing.assert_array_equal(np.isneginf(l), np.isneginf(ref_lse))
    # bf16 partials are merged: each shard's output carries its own bf16 rounding
    assert np.abs(o - ref_out).max() <= 1e-2 * np.abs(ref_out).max()
    fin = np.isfinite(ref_lse)
    assert (np.abs(l[fin] - ref_lse[fin]) / np.maximum(np.abs(ref_lse[fin]), 1.0)).max() <= 1e-4


def test_merge_kernel_matches_oracle_combine():
    g = torch.Generator().manual_seed(5)
    n, b, s_q, h_q = 5, 3, 2, 8
    o = torch.randn(n, b, s_q, h_q, 512, generator=g).to(torch.bfloat16)
    lse = torch.randn(n, b, h_q, s_q, generator=g) * 3
    lse[1] = -float("inf")                   # an empty shard
    lse[:, 2, 3, 1] = -float("inf")          # a row with no key anywhere
    out, l = ops.mla_merge_partials(o.cuda(), lse.cuda())
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.combine(lse.double().numpy().transpose(0, 1, 3, 2), o.double().numpy())
    ref_lse = ref_lse.transpose(0, 2, 1)
    got_o, got_l = out.double().cpu().numpy(), l.double().cpu().numpy()
    np.testing.assert_array_equal(np.isneginf(got_l), np.isneginf(ref_lse))
    assert (got_o[2, 1, 3] == 0).all()
    assert np.abs(got_o - ref_out).max() <= 1e-2 * np.abs(ref_out).max()
    fin = np.isfinite(ref_lse)
    assert np.abs(got_l[fin] - ref_lse[fin]).max() <= 1e-4 * max(1.0, np.abs(ref_lse[fin]).max())
