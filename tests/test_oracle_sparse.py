"""Pins for the oracle's token-level sparse decode (mla_decode_sparse).

Reading (Baidu page on Flash MLA, section 三.3: only the Top-K key connections are kept, the
pattern is stored in CSR form): query token (b, s) attends to the listed key positions that
it may see.  Each pin reduces the sparse decode to the dense decode (itself pinned in
test_oracle.py) on a differently built cache, or to a closed form, so a wrong list offset,
block-table lookup, causal limit or pruning rule fails one of them.
"""

import math

import numpy as np
import torch

import oracle
from paged_mla_decode_11_b200 import workloads as W


def _inputs(lens, s_q=1, h_q=4, seed=0):
    return W.make_inputs(W.custom(len(lens), s_q, h_q, 1, lens, causal=True), seed=seed)


def _csr(lists):
    row_ptr = np.zeros(len(lists) + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum([len(x) for x in lists])
    col = np.concatenate([np.asarray(x, dtype=np.int32) for x in lists]) if row_ptr[-1] else np.zeros(0, np.int32)
    return row_ptr, col


def _sparse(x, lists, causal=True):
    rp, ci = _csr(lists)
    return oracle.mla_decode_sparse(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], rp, ci, dv=512,
                                    softmax_scale=x["softmax_scale"], causal=causal)


def _dense(x, causal=True):
    return oracle.mla_decode(x["q"], x["k_cache"], x["block_table"], x["cache_seqlens"], dv=512,
                             softmax_scale=x["softmax_scale"], causal=causal)


def _cache_row(x, b, j):
    return x["k_cache"][int(x["block_table"][b, j // 64]), j % 64]


def test_full_lists_equal_the_dense_decode():
    lens = [37, 130, 64]
    x = _inputs(lens, s_q=2, seed=1)
    lists = [list(range(L)) for L in lens for _ in range(2)]
    for causal in (True, False):
        o, l = _sparse(x, lists, causal)
        od, ld = _dense(x, causal)
        np.testing.assert_array_equal(o, od)
        np.testing.assert_array_equal(l, ld)


def test_a_list_equals_the_dense_decode_of_its_compacted_keys():
    # the listed keys copied, in list order, into a fresh contiguous sequence: the dense
    # decode of that sequence (no causal limit) is the sparse decode of the list
    lens = [300, 90]
    x = _inputs(lens, seed=2)
    rng = np.random.default_rng(2)
    lists = [list(rng.choice(300, 70, replace=False)), [5, 89, 0, 5, 44]]   # a duplicate in the second
    o, l = _sparse(x, lists, causal=False)
    for b, lst in enumerate(lists):
        n = len(lst)
        pages = (n + 63) // 64
        cache = torch.zeros(pages, 64, 1, 576, dtype=torch.bfloat16)
        for k, j in enumerate(lst):
            cache.view(-1, 1, 576)[k] = _cache_row(x, b, j)
        od, ld = oracle.mla_decode(x["q"][b:b + 1], cache, np.arange(pages, dtype=np.int32)[None], np.array([n]),
                                   dv=512, softmax_scale=x["softmax_scale"], causal=False)
        np.testing.assert_allclose(o[b:b + 1], od, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[b:b + 1], ld, rtol=1e-14, atol=0)


def test_padding_and_invisible_positions_are_pruned():
    lens = [200]
    x = _inputs(lens, s_q=2, seed=3)
    base = [[3, 150, 60], [3, 150, 60, 199]]
    # -1 padding, a position past the sequence, and (row s = 0 only) the last position,
    # which the causal rule hides from the first of the two query tokens
    padded = [[-1, 3, 150, 200, 60, 199, -1], [3, -5, 150, 60, 199, 4096]]
    o1, l1 = _sparse(x, base)
    o2, l2 = _sparse(x, padded)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_list_order_does_not_matter():
    x = _inputs([500], seed=4)
    rng = np.random.default_rng(4)
    lst = list(rng.choice(500, 120, replace=False))
    o1, l1 = _sparse(x, [lst])
    o2, l2 = _sparse(x, [list(reversed(lst))])
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-15, atol=0)


def test_a_repeated_entry_doubles_its_weight():
    # one key listed twice: the same softmax with that key's exponential doubled; with a
    # single distinct key, out = its value row and lse = its score + ln 2
    x = _inputs([90], h_q=2, seed=5)
    o, l = _sparse(x, [[17, 17]])
    row = _cache_row(x, 0, 17).double()[0]
    q = x["q"][0, 0].double()
    for h in range(2):
        score = float(x["softmax_scale"] * (q[h] @ row))
        np.testing.assert_allclose(o[0, 0, h], row[:512].numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(l[0, h, 0], score + math.log(2.0), rtol=1e-14)


def test_empty_lists_give_zero_and_minus_infinity():
    x = _inputs([64, 10], seed=6)
    o, l = _sparse(x, [[], [-1, 10, 11]])
    assert (o == 0).all() and np.isneginf(l).all()


def test_causal_limit_per_query_token():
    # s_q = 3: token s sees positions < L - 2 + s; the list [L-3, L-2, L-1] therefore gives
    # 1, 2 and 3 keys, which must match the dense decode of the compacted keys
    L = 130
    x = _inputs([L], s_q=3, h_q=2, seed=7)
    lst = [L - 3, L - 2, L - 1]
    o, l = _sparse(x, [lst, lst, lst])
    for s in range(3):
        o1, l1 = _sparse(x, [lst[:s + 1]] * 3, causal=False)
        np.testing.assert_allclose(o[:, s], o1[:, s], rtol=0, atol=1e-13)
        np.testing.assert_allclose(l[:, :, s], l1[:, :, s], rtol=1e-15)
