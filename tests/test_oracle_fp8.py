"""Pins of the FP8 latent-cache oracle (CPU).

The FP8 cache stores each token's latent row as OCP E4M3 codes with one fp32 scale per
token and latent head; the decode uses the dequantised rows scale * e4m3(code) (the
Baidu page on Flash MLA names FP8 storage, section 三.2, without a format; this is the
reading the oracle states).  Pins, none of which re-types the oracle's arithmetic:
  - the E4M3 decoder against torch's float8_e4m3fn conversion, on all 256 codes;
  - where every dequantised value is exactly representable in bf16 (power-of-two scales),
    the FP8 oracle equals the bf16 oracle bit for bit;
  - a common scale s on every token equals unit scales with the output times s and the
    softmax scale times s (closed form of the definition);
  - a pure-Python brute force on a tiny case.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from paged_mla_decode_11_b200 import workloads as W


def test_e4m3_decoder_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_to_float64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    np.testing.assert_array_equal(np.isnan(mine), nan)
    np.testing.assert_array_equal(mine[~nan], ref[~nan])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9 and mine[0x08] == 2.0 ** -6


def _fp8_case(seed, lens, h_q=16, h_kv=1, s_q=1, causal=True, pow2=True):
    """Inputs whose dequantised rows are exact in bf16: codes drawn from the finite E4M3
    values, scales powers of two (pow2) or arbitrary fp32."""
    x = W.make_inputs(W.custom(len(lens), s_q, h_q, h_kv, lens, causal=causal), seed=seed)
    g = torch.Generator().manual_seed(seed + 100)
    n_pages = x["k_cache"].shape[0]
    finite = torch.tensor([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=torch.uint8)
    # mostly small magnitudes (|e4m3| <= 4) so the scores stay O(1)
    small = finite[oracle.e4m3_to_float64(finite.numpy()).__abs__() <= 4.0]
    idx = torch.randint(0, small.numel(), (n_pages, 64, h_kv, 576), generator=g)
    k8 = small[idx]
    if pow2:
        k_scale = torch.pow(2.0, torch.randint(-3, 2, (h_kv, n_pages, 64), generator=g).float())
    else:
        k_scale = torch.rand(h_kv, n_pages, 64, generator=g) * 0.9 + 0.1
    return x, k8, k_scale


def _dequant_bf16(k8, k_scale):
    vals = torch.from_numpy(oracle.e4m3_to_float64(k8.numpy()))
    s = k_scale.permute(1, 2, 0).double()[..., None]          # [pages, page, h_kv, 1]
    return (vals * s).to(torch.bfloat16), vals * s


@pytest.mark.parametrize("causal,s_q,h_kv", [(True, 1, 1), (True, 2, 1), (False, 1, 2)])
def test_fp8_equals_bf16_oracle_when_values_are_bf16_exact(causal, s_q, h_kv):
    x, k8, k_scale = _fp8_case(3 + s_q + h_kv, [70, 130, 5], h_q=8 * h_kv, h_kv=h_kv, s_q=s_q, causal=causal)
    kb, kd = _dequant_bf16(k8, k_scale)
    assert torch.equal(kb.double(), kd)                      # exact in bf16
    a = oracle.mla_decode_fp8(x["q"], k8, k_scale, x["block_table"], x["cache_seqlens"], causal=causal,
                              softmax_scale=x["softmax_scale"])
    b = oracle.mla_decode(x["q"], kb, x["block_table"], x["cache_seqlens"], causal=causal,
                          softmax_scale=x["softmax_scale"])
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_common_scale_folds_into_softmax_scale_and_output():
    x, k8, _ = _fp8_case(9, [100, 64], pow2=False)
    s = float(torch.tensor(0.37, dtype=torch.float32))   # the value the fp32 scale holds
    n_pages = k8.shape[0]
    unit = torch.ones(1, n_pages, 64)
    sc = x["softmax_scale"]
    o1, l1 = oracle.mla_decode_fp8(x["q"], k8, unit * s, x["block_table"], x["cache_seqlens"], softmax_scale=sc)
    o2, l2 = oracle.mla_decode_fp8(x["q"], k8, unit, x["block_table"], x["cache_seqlens"], softmax_scale=sc * s)
    np.testing.assert_allclose(o1, s * o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=1e-12, atol=1e-12)


def test_fp8_brute_force_tiny():
    x, k8, k_scale = _fp8_case(5, [3, 7], h_q=2, pow2=False)
    q = x["q"].double().numpy()
    bt, sl = x["block_table"].numpy(), x["cache_seqlens"].numpy()
    vals = oracle.e4m3_to_float64(k8.numpy())
    ks = k_scale.double().numpy()
    sc = x["softmax_scale"]
    out, lse = oracle.mla_decode_fp8(x["q"], k8, k_scale, x["block_table"], x["cache_seqlens"], softmax_scale=sc,
                                     causal=True)
    for b in range(2):
        for h in range(2):
            keys = []
            for j in range(int(sl[b])):
                pg, sl_ = int(bt[b, j // 64]), j % 64
                keys.append([ks[0, pg, sl_] * vals[pg, sl_, 0, t] for t in range(576)])
            xs = [sc * sum(q[b, 0, h, t] * c[t] for t in range(576)) for c in keys]
            m = max(xs)
            z = sum(math.exp(v - m) for v in xs)
            ref = [sum(math.exp(xs[j] - m) / z * keys[j][t] for j in range(len(keys))) for t in range(512)]
            np.testing.assert_allclose(out[b, 0, h], ref, rtol=1e-10, atol=1e-12)
            assert abs(lse[b, h, 0] - (m + math.log(z))) < 1e-10


def test_writer_side_quantisation_is_within_e4m3_precision():
    # to_fp8_cache (input preparation) keeps every dequantised value within half an E4M3
    # step (relative 2^-4) of the bf16 source, and the per-row maximum maps to +-448
    x = W.make_inputs(W.custom(2, 1, 16, 1, [100, 30]), seed=4)
    k8, k_scale = W.to_fp8_cache(x["k_cache"])
    _, deq = _dequant_bf16(k8, k_scale)
    src = x["k_cache"].double()
    err = (deq - src).abs()
    bound = src.abs().amax(dim=-1, keepdim=True) / 448.0 * 2.0 ** -4 * 448.0 / 2
    assert bool((err <= torch.maximum(src.abs() * 2.0 ** -4, bound / 8)).all())
    vals = oracle.e4m3_to_float64(k8.numpy())
    assert np.abs(vals).max() == 448.0
