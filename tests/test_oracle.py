"""Pins of the fp64 oracle to things other than itself.

Each test ties the oracle to the definition of paged MLA decode (absorbed-query score
over the latent row, softmax, value = first dv latent columns, 64-token pages through a
block table), to closed forms, to a textbook routine, to invariants, or to hand-worked
fixtures in tests/golden.  A plausible mistake in the oracle -- a dropped scale, a
transposed operand, a wrong page index, the wrong value columns, a causal offset in the
wrong direction, a base-2 lse -- fails at least one of them.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from paged_mla_decode_11_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _inputs(batch, s_q, h_q, h_kv, seqlens, causal=True, scale=None, seed=0, outlier=0.0):
    w = W.custom(batch, s_q, h_q, h_kv, seqlens, causal=causal, scale=scale, outlier_frac=outlier)
    return W.make_inputs(w, seed=seed)


def _run(x, **kw):
    args = dict(dv=x["dv"], softmax_scale=x["softmax_scale"], causal=x["causal"])
    args.update(kw)
    return oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], **args)


# --------------------------------------------------------------------------------------
# 1. Brute force: an independent pure-Python restatement of the definition, tiny inputs.
# --------------------------------------------------------------------------------------
def _brute(x):
    q = x["q"].float().tolist()
    pool = x["k_cache"].float().tolist()
    bt = x["block_table"].tolist()
    lens = x["cache_seqlens"].tolist()
    B, S, H = len(q), len(q[0]), len(q[0][0])
    h_kv = x["h_kv"]
    g = H // h_kv
    dv, scale, causal = x["dv"], x["softmax_scale"], x["causal"]
    out = [[[None] * H for _ in range(S)] for _ in range(B)]
    lse = [[[None] * S for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for s in range(S):
            visible = lens[b] - (S - 1 - s) if causal else lens[b]
            for h in range(H):
                rows = []
                for j in range(max(visible, 0)):
                    rows.append(pool[bt[b][j // 64]][j % 64][h // g])
                scores = [scale * sum(a * c for a, c in zip(q[b][s][h], row)) for row in rows]
                if not scores:
                    out[b][s][h] = [0.0] * dv
                    lse[b][h][s] = -math.inf
                    continue
                top = max(scores)
                e = [math.exp(v - top) for v in scores]
                z = sum(e)
                out[b][s][h] = [sum(e[j] / z * rows[j][t] for j in range(len(rows))) for t in range(dv)]
                lse[b][h][s] = top + math.log(z)
    return np.array(out), np.array(lse)


@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_tiny(causal):
    x = _inputs(3, 2, 4, 2, [1, 70, 130], causal=causal, seed=3)
    out, lse = _run(x)
    bo, bl = _brute(x)
    np.testing.assert_allclose(out, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=1e-12, atol=1e-12)


def test_brute_force_empty_sequence():
    x = _inputs(2, 2, 2, 1, [0, 1], causal=True, seed=4)
    out, lse = _run(x)
    bo, bl = _brute(x)
    np.testing.assert_array_equal(out[0], 0.0)
    assert np.all(np.isneginf(lse[0]))
    # L = 1, s_q = 2, causal: row s = 0 sees no key, row s = 1 sees key 0.
    assert np.all(np.isneginf(lse[1, :, 0])) and np.all(np.isfinite(lse[1, :, 1]))
    np.testing.assert_allclose(out, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(bl))


# --------------------------------------------------------------------------------------
# 2. Textbook reduction: with h_kv = 1 and the pages gathered into one contiguous K, the
#    method is multi-query attention softmax(scale Q K^T) V with V = K[:, :dv].
# --------------------------------------------------------------------------------------
def test_textbook_mqa_reduction():
    x = _inputs(4, 1, 16, 1, [5, 64, 65, 300], causal=False, seed=5)
    out, lse = _run(x)
    q = x["q"].double()
    flat = x["k_cache"].double().reshape(-1, x["h_kv"], 576)[:, 0]
    for b in range(4):
        L = int(x["cache_seqlens"][b])
        tok = torch.arange(L)
        phys = x["block_table"][b].long()[tok // 64] * 64 + tok % 64
        K = flat.index_select(0, phys)
        V = K[:, :512]
        S = x["softmax_scale"] * q[b, 0] @ K.T
        P = torch.softmax(S, dim=-1)
        np.testing.assert_allclose(out[b, 0], (P @ V).numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(lse[b, :, 0], torch.logsumexp(S, -1).numpy(), rtol=1e-12)


# --------------------------------------------------------------------------------------
# 3. Closed forms.
# --------------------------------------------------------------------------------------
def _manual(seqlen, key_fn, q_vec, scale, h=1):
    pages = max(1, -(-seqlen // 64))
    pool = torch.zeros(pages + 1, 64, 1, 576, dtype=torch.bfloat16)
    pool[pages] = W.POISON
    for j in range(seqlen):
        pool[j // 64, j % 64, 0] = key_fn(j)
    if seqlen % 64:
        pool[(seqlen - 1) // 64, seqlen % 64:] = W.POISON
    q = torch.zeros(1, 1, h, 576, dtype=torch.bfloat16)
    q[0, 0, :] = q_vec
    bt = torch.arange(pages, dtype=torch.int32)[None]
    sl = torch.tensor([seqlen], dtype=torch.int32)
    return oracle.mla_decode(q, pool, bt, sl, dv=512, softmax_scale=scale, causal=True)


def test_identical_keys_give_that_row():
    g = torch.Generator().manual_seed(7)
    row = torch.randn(576, generator=g).to(torch.bfloat16)
    qv = torch.randn(576, generator=g).to(torch.bfloat16)
    n = 150
    out, lse = _manual(n, lambda j: row, qv, 0.05)
    xval = 0.05 * float((qv.double() * row.double()).sum())
    np.testing.assert_allclose(out[0, 0, 0], row.double()[:512].numpy(), rtol=1e-12, atol=1e-13)
    assert lse[0, 0, 0] == pytest.approx(xval + math.log(n), rel=1e-12)


def test_zero_query_gives_column_mean():
    g = torch.Generator().manual_seed(8)
    keys = torch.randn(97, 576, generator=g).to(torch.bfloat16)
    out, lse = _manual(97, lambda j: keys[j], torch.zeros(576, dtype=torch.bfloat16), 0.7)
    np.testing.assert_allclose(out[0, 0, 0], keys.double()[:, :512].mean(0).numpy(), rtol=1e-11, atol=1e-13)
    assert lse[0, 0, 0] == pytest.approx(math.log(97), rel=1e-14)


def test_single_key():
    g = torch.Generator().manual_seed(9)
    key = torch.randn(576, generator=g).to(torch.bfloat16)
    qv = torch.randn(576, generator=g).to(torch.bfloat16)
    out, lse = _manual(1, lambda j: key, qv, 0.3)
    np.testing.assert_allclose(out[0, 0, 0], key.double()[:512].numpy(), rtol=0, atol=0)
    assert lse[0, 0, 0] == pytest.approx(0.3 * float((qv.double() * key.double()).sum()), rel=1e-13)


def test_rope_columns_score_but_are_not_values():
    # Keys that differ only in the 64 rope columns: the scores differ, the values do not.
    base = torch.zeros(576, dtype=torch.bfloat16)
    base[:512] = 1.0
    qv = torch.zeros(576, dtype=torch.bfloat16)
    qv[512] = 1.0

    def key(j):
        k = base.clone()
        k[512] = float(j)
        return k

    out, lse = _manual(3, key, qv, math.log(2.0))
    np.testing.assert_allclose(out[0, 0, 0], np.ones(512), rtol=1e-14)
    assert lse[0, 0, 0] == pytest.approx(math.log(7.0), rel=1e-14)


# --------------------------------------------------------------------------------------
# 4. Hand-worked fixtures.
# --------------------------------------------------------------------------------------
def _frac(s):
    return float(Fraction(s))


def _ln(s):
    s = s.strip()
    if s == "ln 15":
        return math.log(15.0)
    if s == "8 ln 2":
        return 8 * math.log(2.0)
    raise ValueError(s)


def test_golden_two_power_weights():
    spec = json.load(open(os.path.join(GOLDEN, "two_power_weights.json")))
    for case in spec["cases"]:
        L = case["seqlen"]
        npg = case["num_pages"]
        pool = torch.zeros(npg + 1, 64, 1, 576, dtype=torch.bfloat16)
        pool[npg] = W.POISON
        bt = torch.tensor([case["block_table"]], dtype=torch.int32)
        if "keys" in case:
            for j, cols in case["keys"].items():
                j = int(j)
                for c, v in cols.items():
                    pool[int(bt[0, j // 64]), j % 64, 0, int(c)] = float(v)
        else:
            for j in range(64):
                pool[1, j, 0, 3] = 1.0
            pool[0, 0, 0, 0] = 6.0
            pool[0, 1, 0, 0] = 7.0
            pool[0, 2:] = W.POISON
        q = torch.zeros(1, 1, 1, 576, dtype=torch.bfloat16)
        for c, v in case["q_nonzero"].items():
            q[0, 0, 0, int(c)] = v
        sl = torch.tensor([L], dtype=torch.int32)
        out, lse = oracle.mla_decode(q, pool, bt, sl, dv=512, softmax_scale=math.log(2.0), causal=True)
        want = np.zeros(512)
        for c, v in case["expect_out_nonzero"].items():
            want[int(c)] = _frac(v)
        np.testing.assert_allclose(out[0, 0, 0], want, rtol=1e-13, atol=1e-14)
        assert lse[0, 0, 0] == pytest.approx(_ln(case["expect_lse"]), rel=1e-14)


# --------------------------------------------------------------------------------------
# 5. Invariants named by the method.
# --------------------------------------------------------------------------------------
def test_page_permutation_invariance():
    x = _inputs(3, 1, 8, 1, [64, 129, 200], causal=False, seed=11)
    out0, lse0 = _run(x)
    npg = x["num_pages"]
    perm = torch.randperm(npg, generator=torch.Generator().manual_seed(12))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(npg)
    pool2 = x["k_cache"].clone()
    pool2[:npg] = x["k_cache"][:npg][inv]          # physical page p moves to slot perm[p]
    bt2 = x["block_table"].clone()
    real = bt2 < npg
    bt2[real] = perm[bt2[real].long()].to(torch.int32)
    out1, lse1 = oracle.mla_decode(x["q"], pool2, bt2, x["cache_seqlens"], dv=512,
                                   softmax_scale=x["softmax_scale"], causal=False)
    np.testing.assert_array_equal(out0, out1)
    np.testing.assert_array_equal(lse0, lse1)


@pytest.mark.parametrize("cuts", [[0, 64, 192, 300], [0, 1, 2, 300], [0, 300, 300, 300]])
def test_split_merge_equals_unsplit(cuts):
    x = _inputs(1, 1, 16, 1, [300], causal=False, seed=13)
    out, lse = _run(x)
    parts_o, parts_l = [], []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        o, l = _run(x, kv_begin=[lo], kv_end=[hi])
        parts_o.append(o)
        parts_l.append(l)
    lp = np.stack(parts_l)                                         # [k, b, h, s]
    op = np.stack([o.transpose(0, 2, 1, 3) for o in parts_o])      # [k, b, h, s, dv]
    mo, ml = oracle.combine(lp, op)
    np.testing.assert_allclose(mo.transpose(0, 2, 1, 3), out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(ml, lse, rtol=1e-13)


def test_combine_all_empty_partials():
    o, l = oracle.combine(np.array([-np.inf, -np.inf]), np.ones((2, 4)))
    assert np.isneginf(l)
    np.testing.assert_array_equal(o, 0.0)


def test_causal_equals_per_row_truncation():
    x = _inputs(3, 2, 4, 1, [2, 65, 129], causal=True, seed=14)
    out, lse = _run(x)
    for s in range(2):
        trunc = x["cache_seqlens"] - (2 - 1 - s)
        o, l = oracle.mla_decode(x["q"][:, s:s + 1], x["k_cache"], x["block_table"], trunc,
                                 dv=512, softmax_scale=x["softmax_scale"], causal=False)
        np.testing.assert_array_equal(out[:, s], o[:, 0])
        np.testing.assert_array_equal(lse[:, :, s], l[:, :, 0])


def test_kv_head_grouping():
    # h_kv = 2: heads 0..g-1 read latent head 0, heads g..2g-1 read latent head 1.
    x = _inputs(1, 1, 4, 2, [70], causal=False, seed=15)
    out, _ = _run(x)
    x2 = dict(x)
    x2["k_cache"] = x["k_cache"].flip(2).contiguous()        # swap the two latent heads
    q2 = x["q"].clone()
    q2[:, :, [0, 1, 2, 3]] = x["q"][:, :, [2, 3, 0, 1]]      # and the two head groups
    o2, _ = oracle.mla_decode(q2, x2["k_cache"], x["block_table"], x["cache_seqlens"], dv=512,
                              softmax_scale=x["softmax_scale"], causal=False)
    np.testing.assert_array_equal(out[:, :, [2, 3, 0, 1]], o2)
