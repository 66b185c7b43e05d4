"""GPU parity of the CUDA decode path against the fp64 oracle, through the C ABI.

Tolerances (fixed by the specification of this path): bf16 outputs within
max |out - ref| <= 1e-2 * max |ref|, fp32 LSE within relative 1e-4, rows without any
visible key exactly out = 0 and lse = -inf; the split-KV plan bit-exact against the
oracle's scheduler specification.  The LSE's relative error is taken against
max(|ref|, 1): lse = ln Z is the log of the softmax normaliser, so an absolute LSE error
of 1e-4 is a relative error of 1e-4 in Z, and a plain relative test is ill-conditioned
where a single visible key puts the LSE near zero.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import metadata as spec
from paged_mla_decode_11_b200 import ops
from paged_mla_decode_11_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
LSE_RTOL = 1e-4


def to_dev(x):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def run_gpu(x, num_parts=None, q=None, skip_combine=False, kernel="auto"):
    """One decode call on its own workspace; also checks that no device-side wait gave up
    (a pipeline that stalls shows up as a time-out here, not only as wrong values)."""
    d = to_dev(x)
    R = x["s_q"] * x["h_q"] // x["h_kv"]
    tile, splits = ops.get_mla_metadata(d["cache_seqlens"], R, x["h_kv"], num_parts=num_parts)
    qq = d["q"] if q is None else q
    b, s_q, h_q, _ = qq.shape
    ws = ops.new_workspace(ops.workspace_size(b, s_q, h_q, x["h_kv"], tile.shape[0]), qq.device)
    out, lse = ops.mla_decode_paged(qq, d["k_cache"], d["block_table"], d["cache_seqlens"], x["dv"],
                                    tile, splits, softmax_scale=x["softmax_scale"],
                                    causal=x["causal"], workspace=ws, skip_combine=skip_combine,
                                    kernel=kernel)
    torch.cuda.synchronize()
    assert ops.query_status(ws) == ops.MLA_OK, "a device-side wait timed out"
    return out, lse, tile, splits


def check_metadata(x, tile, splits):
    R = x["s_q"] * x["h_q"] // x["h_kv"]
    want_tiles, want_splits = spec.schedule(x["cache_seqlens"].tolist(), tile.shape[0], R)
    assert tile.cpu().tolist() == want_tiles
    assert splits.cpu().tolist() == want_splits


def assert_parity(out, lse, ref_out, ref_lse):
    """Element-wise check of every output and LSE entry; returns the error figures (max abs
    output error over max |ref|, LSE error against max(|ref|, 1), and the plain relative
    LSE error |lse - ref| / |ref|, which is reported, not bounded)."""
    out = out.double().cpu().numpy()
    lse = lse.double().cpu().numpy()
    ref_inf = np.isneginf(ref_lse)
    np.testing.assert_array_equal(np.isneginf(lse), ref_inf)
    scale = max(np.abs(ref_out).max(), 1e-30)
    err = np.abs(out - ref_out).max()
    assert err <= OUT_TOL * scale, f"max abs err {err:.3e} > {OUT_TOL} * {scale:.3e}"
    fin = ~ref_inf
    stats = {"out_err_over_max_ref": err / scale, "lse_rel": 0.0, "lse_plain_rel": 0.0}
    if fin.any():
        d = np.abs(lse[fin] - ref_lse[fin])
        rel = d / np.maximum(np.abs(ref_lse[fin]), 1.0)
        assert rel.max() <= LSE_RTOL, f"lse rel err {rel.max():.3e}"
        stats["lse_rel"] = float(rel.max())
        nz = np.abs(ref_lse[fin]) > 0
        if nz.any():
            stats["lse_plain_rel"] = float((d[nz] / np.abs(ref_lse[fin][nz])).max())
    return stats


def full_parity(x, **kw):
    out, lse, tile, splits = run_gpu(x, **kw)
    check_metadata(x, tile, splits)
    ref_out, ref_lse = oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"],
                                         dv=x["dv"], softmax_scale=x["softmax_scale"], causal=x["causal"])
    assert_parity(out, lse, ref_out, ref_lse)
    # rows that see no key are exactly zero
    empty = np.isneginf(ref_lse).transpose(0, 2, 1)
    if empty.any():
        assert (out.float().cpu().numpy()[empty] == 0).all()
    return out, lse, splits


SMALL_CASES = [
    # (batch, s_q, h_q, h_kv, seqlens, causal)
    (2, 1, 16, 1, [37, 130], True),                      # the tiny decode workload
    (5, 1, 16, 1, [1, 63, 64, 65, 300], False),          # ragged tails around page edges
    (3, 1, 64, 1, [130, 1000, 7], True),                 # 64 rows per latent head
    (2, 1, 128, 1, [500, 77], True),                     # two 64-row blocks
    (3, 2, 128, 1, [2, 129, 700], True),                 # causal multi-token, 256 rows
    (2, 1, 32, 2, [100, 200], False),                    # two latent heads
    (3, 1, 16, 1, [0, 5, 0], True),                      # empty sequences
    (2, 2, 16, 1, [1, 66], True),                        # causal row with no visible key
    (4, 2, 8, 1, [64, 1, 2, 3000], True),                # short causal rows and a long split one
    (1, 1, 16, 1, [6000], False),                        # one long sequence over many splits
]


@pytest.mark.parametrize("kernel", ["auto", "warp_mma", "tcgen05"])
@pytest.mark.parametrize("case", SMALL_CASES, ids=lambda c: f"b{c[0]}sq{c[1]}h{c[2]}kv{c[3]}")
def test_parity_small(case, kernel):
    b, s_q, h_q, h_kv, lens, causal = case
    x = W.make_inputs(W.custom(b, s_q, h_q, h_kv, lens, causal=causal), seed=sum(lens) % 97)
    full_parity(x, kernel=kernel)


WIDE_CASES = [
    # (batch, s_q, h_q, seqlens, causal): the 64-row tcgen05 kernel
    (3, 1, 64, [1, 64, 700], True),           # one 64-row block, ragged pages
    (2, 1, 128, [5000, 33], True),            # two row blocks, a long split sequence
    (2, 2, 128, [700, 2], True),              # causal multi-token: blocks see different key ends
    (3, 3, 32, [129, 1000, 64], True),        # g = 32: a block holds 2 positions x 32 heads
    (2, 4, 16, [300, 65], True),              # g = 16: a block holds 4 positions x 16 heads
    (2, 1, 256, [640, 100], False),           # g = 256: four blocks of 64 heads
    (3, 1, 64, [0, 4000, 0], True),           # empty sequences around a long one
    (1, 2, 64, [1], True),                    # a causal row with no visible key
    (2, 1, 48, [900, 70], True),              # 48 rows: one block with 16 padding rows
    (2, 2, 96, [333, 1200], True),            # g = 96: blocks straddle the two positions
    (3, 3, 24, [64, 2, 777], True),           # g = 24, 72 rows: a second block of 8 rows
]


@pytest.mark.parametrize("case", WIDE_CASES, ids=lambda c: f"b{c[0]}sq{c[1]}h{c[2]}")
@pytest.mark.parametrize("num_parts", [None, 3])
def test_parity_tcgen05_64_row_tiles(case, num_parts):
    b, s_q, h_q, lens, causal = case
    x = W.make_inputs(W.custom(b, s_q, h_q, 1, lens, causal=causal), seed=len(lens) * 13 + h_q)
    full_parity(x, kernel="tcgen05", num_parts=num_parts)


PAIR_CASES = [
    # (batch, s_q, h_q, h_kv, seqlens, causal): the CTA-pair kernel (whole 128-row blocks)
    (2, 1, 128, 1, [5000, 33], True),          # one pair, a long split sequence, a one-page piece
    (3, 1, 128, 1, [64, 65, 191], False),      # exact pages, a lone last page, an odd page count
    (2, 2, 128, 1, [700, 2], True),            # 256 rows: two pairs; their halves see different key ends
    (2, 2, 64, 1, [333, 1000], True),          # g = 64: CTA 0 holds position 0, CTA 1 position 1
    (2, 4, 32, 1, [129, 900], True),           # g = 32: each CTA's rows are 32 heads x 2 positions
    (2, 8, 16, 1, [77, 640], True),            # g = 16: 16 heads x 4 positions per CTA
    (3, 1, 128, 2, [700, 65, 3000], True),     # two latent heads
    (3, 1, 256, 1, [640, 100, 1], False),      # g = 256: two pairs on one position
    (3, 1, 128, 1, [0, 4000, 0], True),        # empty sequences around a long one
    (1, 2, 128, 1, [1], True),                 # a causal row with no visible key
]


@pytest.mark.parametrize("case", PAIR_CASES, ids=lambda c: f"b{c[0]}sq{c[1]}h{c[2]}kv{c[3]}")
@pytest.mark.parametrize("num_parts", [None, 1, 3, 200])
def test_parity_cta_pair_kernel(case, num_parts):
    b, s_q, h_q, h_kv, lens, causal = case
    x = W.make_inputs(W.custom(b, s_q, h_q, h_kv, lens, causal=causal), seed=len(lens) * 7 + h_q + s_q)
    full_parity(x, num_parts=num_parts)


@pytest.mark.parametrize("case", PAIR_CASES[:4], ids=lambda c: f"b{c[0]}sq{c[1]}h{c[2]}kv{c[3]}")
def test_parity_one_sm_kernel_on_pair_shapes(case):
    # the 1-SM 64-row kernel stays available (MLA_FLAG_ONE_SM) on the shapes the pair kernel takes
    b, s_q, h_q, h_kv, lens, causal = case
    x = W.make_inputs(W.custom(b, s_q, h_q, h_kv, lens, causal=causal), seed=len(lens) * 5 + h_q)
    full_parity(x, kernel="one_sm")


@pytest.mark.parametrize("s_q,h_q,h_kv", [(1, 128, 2), (2, 64, 2), (1, 96, 3)], ids=["R64x2", "R64x2-mtp", "R32x3"])
def test_parity_tcgen05_several_latent_heads(s_q, h_q, h_kv):
    # the 64-row kernel with more than one latent head: grid z, page rows of head kvh
    x = W.make_inputs(W.custom(3, s_q, h_q, h_kv, [700, 65, 3000], causal=True), seed=h_q + h_kv)
    full_parity(x)


@pytest.mark.parametrize("h_q", [64, 128], ids=["one-row-block", "two-row-blocks"])
def test_parity_tcgen05_one_part_walks_every_slot_phase(h_q):
    # One part per row block walks 40 sequences of 1 to 5 pages in order, so sequence pieces
    # start in every slot of the three-page ring: page pairs in slots 0-1 and 1-2, pairs back
    # to back on one score buffer, runs of single pages, ragged last pages.
    rng = np.random.default_rng(11)
    lens = (rng.integers(1, 6, size=40) * 64 - rng.integers(0, 64, size=40)).tolist()
    x = W.make_inputs(W.custom(40, 1, h_q, 1, lens, causal=True), seed=12)
    full_parity(x, kernel="tcgen05", num_parts=1)


@pytest.mark.parametrize("h_q", [16, 64, 128])
def test_parity_running_max_grows_every_page(h_q):
    # The p-th page of every sequence is scaled by 1 + 3p, so the row maximum of the scores
    # grows by more than 8 in log2 units from page to page: the output accumulator is
    # rescaled in most score groups (in the 64-row kernel, each time after the previous
    # group's PV has completed).  Both sides read the same scaled bf16 pages.
    x = W.make_inputs(W.custom(3, 1, h_q, 1, [1000, 640, 129], causal=False), seed=31)
    kc, bt = x["k_cache"], x["block_table"]
    for b, L in enumerate(x["cache_seqlens"].tolist()):
        for p in range((L + 63) // 64):
            page = int(bt[b, p])
            kc[page] = (kc[page].float() * (1 + 3 * p)).to(torch.bfloat16)
    full_parity(x)


@pytest.mark.parametrize("kernel", ["auto", "tcgen05"])
@pytest.mark.parametrize("h_q,s_q", [(16, 1), (8, 2), (4, 1), (24, 1), (32, 1), (12, 3), (48, 1), (64, 1), (16, 4)])
def test_parity_row_paddings(h_q, s_q, kernel):
    # every padded tile height of the kernels (16, 32, 48, 64 rows), ragged row counts
    x = W.make_inputs(W.custom(3, s_q, h_q, 1, [1, 200, 1000], causal=True), seed=h_q * 7 + s_q)
    full_parity(x, kernel=kernel)


def test_parity_outlier_rows_and_scale():
    x = W.make_inputs(W.custom(3, 2, 64, 1, [900, 45, 2000], causal=True, outlier_frac=0.05, scale=0.11),
                      seed=21)
    full_parity(x)


@pytest.mark.parametrize("num_parts", [1, 2, 7, 148, 400])
def test_parity_any_part_count(num_parts):
    x = W.make_inputs(W.custom(6, 1, 16, 1, [3000, 1, 0, 640, 64, 999], causal=True), seed=5)
    full_parity(x, num_parts=num_parts)


def test_strided_query_view():
    x = W.make_inputs(W.custom(3, 1, 16, 1, [70, 300, 5], causal=True), seed=8)
    big = torch.zeros(3, 1, 24, 640, dtype=torch.bfloat16, device="cuda")
    big[:, :, 4:20, :576] = x["q"].cuda()
    qv = big[:, :, 4:20, :576]
    assert not qv.is_contiguous()
    out, lse, _, _ = run_gpu(x, q=qv)
    ref_out, ref_lse = oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"],
                                         dv=512, softmax_scale=x["softmax_scale"], causal=True)
    assert_parity(out, lse, ref_out, ref_lse)


def test_separate_combine_matches_fused():
    x = W.make_inputs(W.custom(2, 1, 64, 1, [5000, 300], causal=True), seed=9)
    out_a, lse_a, tile, splits = run_gpu(x)
    d = to_dev(x)
    ws = ops.new_workspace(ops.workspace_size(2, 1, 64, 1, tile.shape[0]), "cuda")
    out_b, lse_b = ops.mla_decode_paged(d["q"], d["k_cache"], d["block_table"], d["cache_seqlens"], 512,
                                        tile, splits, softmax_scale=x["softmax_scale"], causal=True,
                                        workspace=ws, skip_combine=True)
    ops.mla_combine(splits, 1, 64, 1, tile.shape[0], ws, out_b, lse_b)
    torch.cuda.synchronize()
    assert int(splits[1] - splits[0]) > 1
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)


@pytest.mark.parametrize("h_q", [16, 64], ids=["16-row-kernel", "64-row-kernel"])
def test_many_short_sequences_sampled(h_q):
    # 2048 sequences of 1..256 tokens: parts hold many sequence pieces, so the query reload,
    # the per-piece epilogue and the scheduler's block path all run many times
    rng = np.random.default_rng(3)
    lens = rng.integers(1, 257, size=2048).tolist()
    x = W.make_inputs(W.custom(2048, 1, h_q, 1, lens, causal=True), seed=21)
    out, lse, tile, splits = run_gpu(x)
    check_metadata(x, tile, splits)
    rows = sample_rows(x, per_seq=1, seed=4)[::7]
    ro, rl = oracle.mla_decode_rows(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], rows,
                                    dv=512, softmax_scale=x["softmax_scale"], causal=True)
    o = out.double().cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    l = lse.double().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert np.abs(o - ro).max() <= OUT_TOL * np.abs(ro).max()
    assert (np.abs(l - rl) / np.maximum(np.abs(rl), 1.0)).max() <= LSE_RTOL


@pytest.mark.parametrize("h_q", [16, 64], ids=["16-row-kernel", "64-row-kernel"])
def test_all_sequences_empty(h_q):
    x = W.make_inputs(W.custom(3, 1, h_q, 1, [0, 0, 0], causal=True), seed=2)
    out, lse, _, _ = run_gpu(x)
    assert torch.isneginf(lse).all()
    assert (out == 0).all()


@pytest.mark.parametrize("h_q", [16, 128], ids=["16-row-kernel", "cta-pair-kernel"])
def test_no_split_steps_back_to_back(h_q):
    # One part per sequence (num_parts = batch, equal lengths): no sequence is split, so the
    # combine finds nothing to merge (one of its CTAs still waits for the decode kernel).
    # Three decodes of different inputs run back to back on one stream over one plan and
    # one workspace, each checked element-wise afterwards.
    b, lens = 8, [640] * 8
    xs = [W.make_inputs(W.custom(b, 1, h_q, 1, lens, causal=True), seed=s) for s in (31, 32, 33)]
    ds = [to_dev(x) for x in xs]
    tile, splits = ops.get_mla_metadata(ds[0]["cache_seqlens"], h_q, 1, num_parts=b)
    assert splits.cpu().tolist() == list(range(b + 1))
    ws = ops.new_workspace(ops.workspace_size(b, 1, h_q, 1, tile.shape[0]), "cuda")
    res = [ops.mla_decode_paged(d["q"], d["k_cache"], d["block_table"], d["cache_seqlens"], 512, tile, splits,
                                softmax_scale=x["softmax_scale"], causal=True, workspace=ws)
           for x, d in zip(xs, ds)]
    torch.cuda.synchronize()
    assert ops.query_status(ws) == ops.MLA_OK
    for x, (out, lse) in zip(xs, res):
        ref_out, ref_lse = oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"],
                                             dv=512, softmax_scale=x["softmax_scale"], causal=True)
        assert_parity(out, lse, ref_out, ref_lse)


def test_deterministic():
    x = W.make_inputs(W.custom(4, 1, 128, 1, [4000, 100, 2500, 64], causal=True), seed=10)
    a = run_gpu(x)
    b = run_gpu(x)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_watchdog_times_out_and_context_survives():
    ws = ops.new_workspace(256, "cuda")
    ops.watchdog_selftest(ws, 50_000_000)           # 50 ms limit on a wait nothing completes
    assert ops.query_status(ws) == ops.MLA_ERR_TIMEOUT
    assert ops.query_status(ws) == ops.MLA_OK          # cleared
    x = W.make_inputs(W.TINY)
    full_parity(x)                                     # the context is still usable


# ---------------------------------------------------------------------------------------
# Full-size workloads, in the launch configuration the benchmark times: bit-exact plan and
# every output and LSE entry against the oracle.
# ---------------------------------------------------------------------------------------
def sample_rows(x, per_seq=2, seed=0):
    rng = np.random.default_rng(seed)
    b, s_q, h_q = x["q"].shape[:3]
    rows = []
    for i in range(b):
        for _ in range(per_seq):
            rows.append((i, rng.integers(s_q), rng.integers(h_q)))
        rows.append((i, s_q - 1, h_q - 1))
    return np.array(rows, dtype=np.int32)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_full_size_workloads(name):
    x = W.make_inputs(W.WORKLOADS[name], seed=0)
    out, lse, tile, splits = run_gpu(x)
    check_metadata(x, tile, splits)
    ref_out, ref_lse = oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"],
                                         dv=512, softmax_scale=x["softmax_scale"], causal=x["causal"])
    stats = assert_parity(out, lse, ref_out, ref_lse)
    print(f"{name}: " + ", ".join(f"{k} {v:.3e}" for k, v in stats.items()))


# ---------------------------------------------------------------------------------------
# Maximum sizes: the largest batch the scheduler takes, and one sequence long enough that
# every part holds a piece of it (the combine then merges as many partials as there are parts).
# ---------------------------------------------------------------------------------------
def test_largest_batch_sampled():
    # MLA_MAX_BATCH sequences of 1..64 tokens (one page each): the plan's block scans run over
    # 16,384 lengths (shared memory above 48 KB), and parts walk hundreds of sequences each
    batch = 16384
    rng = np.random.default_rng(16)
    lens = rng.integers(1, 65, size=batch).tolist()
    x = W.make_inputs(W.custom(batch, 1, 16, 1, lens, causal=True), seed=16)
    out, lse, tile, splits = run_gpu(x)
    check_metadata(x, tile, splits)
    rows = sample_rows(x, per_seq=1, seed=16)[::61]
    ro, rl = oracle.mla_decode_rows(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], rows,
                                    dv=512, softmax_scale=x["softmax_scale"], causal=True)
    o = out.double().cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    l = lse.double().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert np.abs(o - ro).max() <= OUT_TOL * np.abs(ro).max()
    assert (np.abs(l - rl) / np.maximum(np.abs(rl), 1.0)).max() <= LSE_RTOL
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("h_q", [16, 64, 128], ids=["16-row-kernel", "64-row-kernel", "cta-pair-kernel"])
def test_one_sequence_over_every_part(h_q):
    # 131,072 tokens (2,048 pages) in one sequence: every part decodes a piece of it and the
    # combine merges 148 (or 74) partials per row, more than one warp's worth of split LSEs
    L = 131072
    x = W.make_inputs(W.custom(1, 1, h_q, 1, [L], causal=True), seed=h_q)
    out, lse, tile, splits = run_gpu(x)
    check_metadata(x, tile, splits)
    assert int(splits[1] - splits[0]) > 32
    rows = np.array([(0, 0, h) for h in range(0, h_q, max(1, h_q // 16))], dtype=np.int32)
    ro, rl = oracle.mla_decode_rows(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], rows,
                                    dv=512, softmax_scale=x["softmax_scale"], causal=True)
    o = out.double().cpu().numpy()[rows[:, 0], rows[:, 1], rows[:, 2]]
    l = lse.double().cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert np.abs(o - ro).max() <= OUT_TOL * np.abs(ro).max()
    assert (np.abs(l - rl) / np.maximum(np.abs(rl), 1.0)).max() <= LSE_RTOL
