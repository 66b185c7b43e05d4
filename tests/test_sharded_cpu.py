"""Sequence-sharded decode over several GPUs: its host logic on the CPU.

Shard layout (shard_bounds): contiguous page-aligned token ranges covering the sequence, the
causal tail (positions >= L - s_q + 1) always in the last shard.  The whole flow of
sharded_decode -- every rank decodes its shard, one all-gather of the partials, a
log-sum-exp merge -- runs here on two and three gloo processes, with the fp64 oracle standing
in for the GPU decode and merge steps, and must equal the unsplit oracle.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_mla_decode_11_b200 import sharded  # noqa: E402


@pytest.mark.parametrize("n", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("s_q", [1, 2, 3])
def test_shard_bounds_cover_the_sequence(n, s_q):
    for L in [0, 1, 2, 63, 64, 65, 127, 128, 129, 500, 4096, 5000]:
        b = sharded.shard_bounds(L, n, s_q)
        assert len(b) == n
        assert b[0][0] == 0 and b[-1][1] == L
        for (a0, e0), (a1, e1) in zip(b, b[1:]):
            assert e0 == a1                          # contiguous, disjoint
        for a, e in b:
            assert 0 <= a <= e <= L
            assert a % 64 == 0 or a == L             # page aligned starts
        # every key a causal row may not see lies in the last shard
        assert b[-1][0] <= max(0, L - s_q + 1)
        # pages are dealt out evenly up to the tail adjustment
        sizes = [(e - a + 63) // 64 for a, e in b]
        assert max(sizes[:-1] or [0]) - min(sizes[:-1] or [0]) <= 1


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_decode(q, k_cache, bt, lens, causal, scale):
    import oracle
    out, lse = oracle.mla_decode(q, k_cache, bt, lens, dv=512, softmax_scale=scale, causal=causal)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _oracle_merge(o_all, l_all):
    import oracle
    # combine wants the row axes of lse in the order of o's: [k, b, s_q, h_q]
    lse_k = l_all.numpy().transpose(0, 1, 3, 2)
    out, lse = oracle.combine(lse_k, o_all.numpy())
    return torch.from_numpy(out), torch.from_numpy(lse.transpose(0, 2, 1).copy())


def _worker(rank, world, port, results):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "MASTER_ADDR": "127.0.0.1",
                       "MASTER_PORT": str(port)})
    import torch.distributed as dist
    from paged_mla_decode_11_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lens = [5000, 1, 130, 64]
        x = W.make_inputs(W.custom(4, 2, 16, 1, lens, causal=True), seed=3)   # same on every rank
        bt, sl = sharded.shard_block_table(x["block_table"], lens, world, rank, s_q=2)
        out, lse = sharded.sharded_decode(x["q"], x["k_cache"], bt, sl, rank == world - 1, True,
                                          softmax_scale=x["softmax_scale"], decode_fn=_oracle_decode,
                                          merge_fn=_oracle_merge)
        results.put((rank, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_decode_equals_unsplit_on_gloo_ranks(world):
    import oracle
    from paged_mla_decode_11_b200 import workloads as W
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    got = [results.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    lens = [5000, 1, 130, 64]
    x = W.make_inputs(W.custom(4, 2, 16, 1, lens, causal=True), seed=3)
    ref_out, ref_lse = oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], dv=512,
                                         softmax_scale=x["softmax_scale"], causal=True)
    for _, out, lse in got:     # every rank holds the merged result
        np.testing.assert_allclose(out, ref_out, rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(lse, ref_lse, rtol=1e-9, atol=1e-11)
