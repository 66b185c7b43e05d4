"""GPU parity of the absorption products (mla_absorb_query / mla_absorb_output) against the
fp64 oracle, through the C ABI, and of the whole absorbed chain (absorb -> latent decode ->
output projection) at the decode shapes.

Tolerance, from the arithmetic: bf16 inputs are exact in fp32; the kernel accumulates in
fp32 (K = 128 or 512 terms, each rounding error <= 2^-24 of the running sum, so the sum is off
by at most K * 2^-24 * sum_k |a_k b_k|) and rounds the result once to bf16 (<= 2^-9 relative).
The test allows |got - ref| <= 2^-8 |ref| + 2^-14 * sum_k |a_k b_k| element by element, about
twice the bound.  The rope columns of q' are copies and must be bit-equal.
"""

import numpy as np
import pytest
import torch

import oracle
from paged_mla_decode_11_b200 import ops
from paged_mla_decode_11_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _np(t):
    return t.double().cpu().numpy()


def _check(got, ref, mag):
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -14 * mag
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} elements out of bound; worst excess {(err - bound).max():.3e}"


@pytest.mark.parametrize("T,H", [(1, 1), (37, 16), (64, 128), (130, 16), (256, 128), (1000, 3)])
def test_absorb_query_parity(T, H):
    x = W.make_absorb_inputs(T, H, seed=T + H)
    d = {k: v.cuda() for k, v in x.items()}
    q = ops.absorb_query(d["q_nope"], d["q_rope"], d["w_uk"])
    torch.cuda.synchronize()
    ref = oracle.absorb_query(_np(x["q_nope"]), _np(x["q_rope"]), _np(x["w_uk"]))
    mag = oracle.absorb_query(np.abs(_np(x["q_nope"])), np.abs(_np(x["q_rope"])), np.abs(_np(x["w_uk"])))
    got = _np(q)
    np.testing.assert_array_equal(got[..., 512:], ref[..., 512:])
    _check(got[..., :512], ref[..., :512], mag[..., :512])


@pytest.mark.parametrize("T,H", [(1, 1), (37, 16), (64, 128), (130, 16), (256, 128), (1000, 3)])
def test_absorb_output_parity(T, H):
    x = W.make_absorb_inputs(T, H, seed=7 * T + H)
    o = ops.absorb_output(x["o_latent"].cuda(), x["w_uv"].cuda())
    torch.cuda.synchronize()
    ref = oracle.absorb_output(_np(x["o_latent"]), _np(x["w_uv"]))
    mag = oracle.absorb_output(np.abs(_np(x["o_latent"])), np.abs(_np(x["w_uv"])))
    _check(_np(o), ref, mag)


def test_absorb_output_reads_a_strided_latent():
    # the decode's out [b, s_q, h_q, 512] viewed with a token stride larger than H * 512
    T, H = 40, 8
    x = W.make_absorb_inputs(T, H, seed=5)
    big = torch.zeros(T, H + 2, 512, dtype=torch.bfloat16)
    big[:, 1:H + 1] = x["o_latent"]
    view = big.cuda()[:, 1:H + 1]
    o = ops.absorb_output(view, x["w_uv"].cuda())
    torch.cuda.synchronize()
    ref = oracle.absorb_output(_np(x["o_latent"]), _np(x["w_uv"]))
    mag = oracle.absorb_output(np.abs(_np(x["o_latent"])), np.abs(_np(x["w_uv"])))
    _check(_np(o), ref, mag)


@pytest.mark.parametrize("batch,s_q,H,lens", [(4, 1, 16, [1, 64, 300, 1000]), (2, 2, 128, [70, 500])])
def test_absorbed_chain_matches_the_oracle_chain(batch, s_q, H, lens):
    # GPU: absorb -> decode -> output projection; oracle: the same three steps in fp64, fed the
    # GPU's bf16 absorbed query (the decode's input type) so each side's decode sees one input
    T = batch * s_q
    x = W.make_absorb_inputs(T, H, seed=11)
    wk = W.make_inputs(W.custom(batch, s_q, H, 1, lens, causal=True), seed=3)
    qn, qr = x["q_nope"].cuda(), x["q_rope"].cuda()
    q_abs = ops.absorb_query(qn, qr, x["w_uk"].cuda()).view(batch, s_q, H, 576)
    dev = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in wk.items()}
    scale = 192 ** -0.5
    tile, splits = ops.get_mla_metadata(dev["cache_seqlens"], s_q * H, 1)
    o_lat, _ = ops.mla_decode_paged(q_abs, dev["k_cache"], dev["block_table"], dev["cache_seqlens"], 512, tile,
                                    splits, softmax_scale=scale, causal=True)
    out = ops.absorb_output(o_lat.view(T, H, 512), x["w_uv"].cuda())
    torch.cuda.synchronize()

    ref_lat, _ = oracle.mla_decode(q_abs.cpu(), wk["k_cache"], wk["block_table"], wk["cache_seqlens"], dv=512,
                                   softmax_scale=scale, causal=True)
    ref = oracle.absorb_output(ref_lat.reshape(T, H, 512), _np(x["w_uv"]))
    # decode tolerance (1e-2 of the largest latent output) carried through W^UV, plus the
    # projection's own bound
    lat_err = 1e-2 * np.abs(ref_lat).max()
    w_row = np.abs(_np(x["w_uv"])).sum(axis=2)                                   # [H, 128]
    mag = oracle.absorb_output(np.abs(ref_lat.reshape(T, H, 512)), np.abs(_np(x["w_uv"])))
    err = np.abs(_np(out) - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -14 * mag + lat_err * w_row[None]
    assert (err <= bound).all(), f"worst excess {(err - bound).max():.3e}"
