"""GPU parity of the FP8 latent-cache decode (mla_decode_paged_fp8) against the fp64 FP8
oracle, through the C ABI.  Same tolerances as the bf16 path: max |out - ref| <= 1e-2 *
max |ref|, LSE within relative 1e-4 (against max(|ref|, 1)), rows without a visible key
exactly out = 0 and lse = -inf."""

import numpy as np
import pytest
import torch

import oracle
from paged_mla_decode_11_b200 import ops
from paged_mla_decode_11_b200 import workloads as W

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2
LSE_RTOL = 1e-4


def run_fp8(x, num_parts=None, skip_combine=False):
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    R = x["s_q"] * x["h_q"] // x["h_kv"]
    tile, splits = ops.get_mla_metadata(d["cache_seqlens"], R, x["h_kv"], num_parts=num_parts)
    b, s_q, h_q, _ = d["q"].shape
    ws = ops.new_workspace(ops.workspace_size(b, s_q, h_q, x["h_kv"], tile.shape[0]), "cuda")
    out, lse = ops.mla_decode_paged_fp8(d["q"], d["k8"], d["k_scale"], d["block_table"], d["cache_seqlens"], 512,
                                        tile, splits, softmax_scale=x["softmax_scale"], causal=x["causal"],
                                        workspace=ws, skip_combine=skip_combine)
    torch.cuda.synchronize()
    assert ops.query_status(ws) == ops.MLA_OK, "a device-side wait timed out"
    return out, lse, tile, splits, ws


def fp8_parity(x, **kw):
    out, lse, _, splits, _ = run_fp8(x, **kw)
    ref_out, ref_lse = oracle.mla_decode_fp8(x["q"], x["k8"], x["k_scale"], x["block_table"], x["cache_seqlens"],
                                             dv=512, softmax_scale=x["softmax_scale"], causal=x["causal"])
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


FP8_CASES = [
    # (batch, s_q, h_q, h_kv, seqlens, causal)
    (2, 1, 16, 1, [37, 130], True),                 # the tiny decode shape
    (5, 1, 16, 1, [1, 31, 32, 33, 300], False),     # ragged ends around half pages
    (3, 1, 16, 1, [0, 5, 0], True),                 # empty sequences
    (2, 2, 8, 1, [1, 66], True),                    # causal multi-token, a row with no visible key
    (2, 1, 32, 2, [100, 200], False),               # two latent heads
    (3, 1, 4, 1, [500, 77, 1000], True),            # 4 rows of a 16-row tile
    (1, 1, 16, 1, [6000], False),                   # one long sequence over many splits
]


@pytest.mark.parametrize("case", FP8_CASES, ids=lambda c: f"b{c[0]}sq{c[1]}h{c[2]}kv{c[3]}")
@pytest.mark.parametrize("num_parts", [None, 3])
def test_fp8_parity_small(case, num_parts):
    b, s_q, h_q, h_kv, lens, causal = case
    x = W.make_inputs_fp8(W.custom(b, s_q, h_q, h_kv, lens, causal=causal), seed=sum(lens) % 89)
    fp8_parity(x, num_parts=num_parts)


def test_fp8_parity_outliers_and_growing_maximum():
    # rows scaled x8 (5%) change the token scales; pages scaled up from page to page make the
    # running maximum grow on most chunks
    x = W.make_inputs(W.custom(3, 1, 16, 1, [1000, 640, 129], causal=False, outlier_frac=0.05), seed=31)
    kc, bt = x["k_cache"], x["block_table"]
    for b, L in enumerate(x["cache_seqlens"].tolist()):
        for pg in range((L + 63) // 64):
            page = int(bt[b, pg])
            kc[page] = (kc[page].float() * (1 + 3 * pg)).to(torch.bfloat16)
    x["k8"], x["k_scale"] = W.to_fp8_cache(kc)
    fp8_parity(x)


@pytest.mark.parametrize("q_exp", [40, -40, 0])
def test_fp8_parity_query_magnitudes(q_exp):
    # the score path carries the query tile in f16 after a power-of-two scale: queries far from
    # unit size (scaled by 2^q_exp, exact in bf16; the softmax scale compensates so the scores
    # stay the same), and a tile whose rows differ in size by 2^20 (row 3 large, row 5 small)
    x = W.make_inputs_fp8(W.custom(2, 1, 16, 1, [700, 130], causal=True), seed=17)
    q = x["q"].float() * 2.0 ** q_exp
    q[:, :, 3] *= 2.0 ** 10
    q[:, :, 5] *= 2.0 ** -10
    x["q"] = q.to(torch.bfloat16)
    assert torch.equal(x["q"].float(), q)
    x["softmax_scale"] = 576 ** -0.5 * 2.0 ** -q_exp
    fp8_parity(x)


def test_fp8_parity_subnormal_codes():
    # codes drawn from the whole E4M3 set, subnormals (exponent field 0) included, with
    # scales of a few binades: the codes' exact widening is exercised code by code
    x = W.make_inputs(W.custom(2, 1, 16, 1, [300, 77], causal=False), seed=23)
    g = torch.Generator().manual_seed(23)
    k8 = torch.randint(0, 256, x["k_cache"].shape, generator=g, dtype=torch.int32).to(torch.uint8)
    k8[(k8 & 0x7f) == 0x7f] = 0x01           # no NaN codes; more subnormals
    sub = torch.rand(k8.shape, generator=g) < 0.3
    k8[sub] = k8[sub] & 0x87                 # exponent field 0: subnormal (or zero) codes
    x["k8"] = k8
    x["k_scale"] = (2.0 ** torch.randint(-9, -5, (1, k8.shape[0], 64), generator=g)).float()
    fp8_parity(x)


def test_fp8_separate_combine_matches_fused():
    x = W.make_inputs_fp8(W.custom(2, 1, 16, 1, [5000, 300], causal=True), seed=9)
    out_a, lse_a, tile, splits, _ = run_fp8(x)
    out_b, lse_b, _, _, ws = run_fp8(x, skip_combine=True)
    ops.mla_combine(splits.cuda(), 1, 16, 1, tile.shape[0], ws, out_b, lse_b)
    torch.cuda.synchronize()
    assert int(splits[1] - splits[0]) > 1
    assert torch.equal(out_a, out_b) and torch.equal(lse_a, lse_b)


def test_fp8_full_size_memory_bound():
    # the memory-bound workload with its cache in the FP8 format, every entry compared
    x = W.make_inputs_fp8(W.WORKLOADS["memory_bound"], seed=0)
    err = fp8_parity(x)
    print(f"memory_bound fp8: out_err_over_max_ref {err:.3e}")


def test_fp8_tail_scales_are_not_read():
    # A sequence's last page holds slots past its length.  They are not keys, so whatever
    # scales they hold (here NaN and inf) enter neither a chunk's power-of-two factor nor a
    # product with a zero probability: the result equals the oracle's on clean scales.
    x = W.make_inputs_fp8(W.custom(4, 1, 16, 1, [37, 130, 69, 64], causal=True), seed=17)
    ref_out, ref_lse = oracle.mla_decode_fp8(x["q"], x["k8"], x["k_scale"], x["block_table"], x["cache_seqlens"],
                                             dv=512, softmax_scale=x["softmax_scale"], causal=True)
    ks = x["k_scale"].clone()
    for b, L in enumerate(x["cache_seqlens"].tolist()):
        if L % 64:
            page = int(x["block_table"][b, (L - 1) // 64])
            ks[:, page, L % 64:] = float("nan") if b % 2 == 0 else float("inf")
    out, lse, _, _, _ = run_fp8(dict(x, k_scale=ks))
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.isfinite(o).all() and np.isfinite(l).all()
    assert np.abs(o - ref_out).max() <= OUT_TOL * np.abs(ref_out).max()
    assert (np.abs(l - ref_lse) / np.maximum(np.abs(ref_lse), 1.0)).max() <= LSE_RTOL


def test_fp8_rejects_more_than_16_rows():
    x = W.make_inputs_fp8(W.custom(2, 1, 64, 1, [100, 10]), seed=1)
    with pytest.raises(ops.MlaError) as e:
        run_fp8(x)
    assert e.value.code == -2
