"""Pins for the oracle's weight-absorption products (absorb_query, absorb_output).

The absorption notes ("DeepSeek FlashMLA ... practitioner notes", dpshk.com, section 2.1)
fix what the two products must achieve: attention over per-head keys k_h = [W^UK_h c ; k_rope]
and values v_h = W^UV_h c materialised from the latent rows c equals latent attention with the
absorbed query, followed by the output up-projection.  The textbook side below builds those
keys and values explicitly and runs plain softmax attention, so a transposed weight, a wrong
head index or a dropped rope term on the oracle's side fails it.
"""

import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from paged_mla_decode_11_b200 import workloads as wl  # noqa: E402


def test_identity_projection_keeps_the_query():
    # W^UK_h = [I_128 | 0]: the absorbed query is q_nope in the first 128 latent columns,
    # zeros up to 512, then q_rope
    T, H = 3, 2
    rng = np.random.default_rng(1)
    qn, qr = rng.standard_normal((T, H, 128)), rng.standard_normal((T, H, 64))
    w = np.zeros((H, 128, 512))
    w[:, np.arange(128), np.arange(128)] = 1.0
    q = oracle.absorb_query(qn, qr, w)
    assert q.shape == (T, H, 576)
    np.testing.assert_array_equal(q[..., :128], qn)
    np.testing.assert_array_equal(q[..., 128:512], 0.0)
    np.testing.assert_array_equal(q[..., 512:], qr)


def test_output_projection_selects_latent_columns():
    # W^UV_h with a single 1 at (d, perm_h[d]) picks latent column perm_h[d] for output d,
    # a different permutation per head
    T, H = 4, 3
    rng = np.random.default_rng(2)
    o = rng.standard_normal((T, H, 512))
    w = np.zeros((H, 128, 512))
    perms = [rng.permutation(512)[:128] for _ in range(H)]
    for h in range(H):
        w[h, np.arange(128), perms[h]] = 1.0
    out = oracle.absorb_output(o, w)
    for h in range(H):
        np.testing.assert_array_equal(out[:, h, :], o[:, h, perms[h]])


def _textbook_attention(q_nope, q_rope, latent, k_rope, w_uk, w_uv, scale):
    """Per-head attention with explicitly materialised keys and values (the "traditional"
    form that expands the cache per head): k_h[j] = [W^UK_h c_j ; k_rope_j],
    v_h[j] = W^UV_h c_j, out = softmax(scale q k^T) v."""
    T, H, _ = q_nope.shape
    out = np.zeros((T, H, 128))
    for h in range(H):
        keys = np.concatenate([latent @ w_uk[h].T, k_rope], axis=1)      # [n, 192]
        vals = latent @ w_uv[h].T                                        # [n, 128]
        for t in range(T):
            qv = np.concatenate([q_nope[t, h], q_rope[t, h]])
            x = scale * (keys @ qv)
            p = np.exp(x - x.max())
            out[t, h] = (p / p.sum()) @ vals
    return out


def test_absorbed_decode_equals_textbook_attention():
    # small integers times powers of two keep the absorbed query exact in bf16, so the
    # bf16-input decode oracle sees exactly the fp64 absorbed query
    T, H, n = 2, 3, 70
    rng = np.random.default_rng(3)
    q_nope = rng.integers(-2, 3, (T, H, 128)) / 4.0
    q_rope = rng.integers(-3, 4, (T, H, 64)) / 4.0
    w_uk = rng.integers(-1, 2, (H, 128, 512)) * (rng.random((H, 128, 512)) < 0.05) / 2.0
    w_uv = rng.standard_normal((H, 128, 512))
    latent = rng.integers(-3, 4, (n, 512)) / 8.0
    k_rope = rng.integers(-3, 4, (n, 64)) / 8.0
    scale = 192 ** -0.5

    q_abs = oracle.absorb_query(q_nope, q_rope, w_uk)                   # [T, H, 576]
    assert np.array_equal(torch.tensor(q_abs).to(torch.bfloat16).double().numpy(), q_abs)
    # one sequence of n tokens over two pages; the query rows are the T tokens' heads
    cache = torch.zeros(2, 64, 1, 576, dtype=torch.float64)
    rows = np.concatenate([latent, k_rope], axis=1)
    cache.view(128, 1, 576)[:n, 0] = torch.tensor(rows)
    q = torch.tensor(q_abs).reshape(1, T, H, 576).to(torch.bfloat16)
    o_lat, _ = oracle.mla_decode(q, cache.to(torch.bfloat16), np.array([[0, 1]]), np.array([n]),
                                 dv=512, softmax_scale=scale, causal=False)
    got = oracle.absorb_output(o_lat.reshape(T, H, 512), w_uv)
    want = _textbook_attention(q_nope, q_rope, latent, k_rope, w_uk, w_uv, scale)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_absorb_inputs_are_two_views_of_one_projection():
    x = wl.make_absorb_inputs(5, 4, seed=0)
    assert x["q_nope"].shape == (5, 4, 128) and x["q_rope"].shape == (5, 4, 64)
    assert x["q_nope"].stride() == (4 * 192, 192, 1)
    assert x["q_rope"].data_ptr() - x["q_nope"].data_ptr() == 128 * 2
    assert x["w_uk"].shape == (4, 128, 512) and x["w_uv"].shape == (4, 128, 512)
    y = wl.make_absorb_inputs(5, 4, seed=0)
    for k in x:
        assert torch.equal(x[k], y[k])
