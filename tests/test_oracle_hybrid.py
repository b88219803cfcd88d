"""Pins of the oracle's decode attention with the pages' own assignment (STAR-KV technical
summary, Methodology §2: keys head-wise, values joint):

* at full rank without quantisation it equals standard attention with K = x W_k, V = x W_v;
* at truncated ranks it equals standard attention on the rank-r projections of W_k per head
  and of W_v as a whole;
* with every head's query equal, the heads of one KV head give equal outputs, and a
  one-hot-in-position query of a single-token context returns that token's value row.
"""
import numpy as np
import pytest

import oracle as O

from test_oracle_attention import _layer, _sdpa_reference


@pytest.mark.parametrize("H,n_kv", [(4, 4), (8, 2)])
def test_full_rank_hybrid_equals_standard_attention(H, n_kv):
    d_model, d, L = 256, 64, 200
    Wk, Wv = _layer(d_model, n_kv, d, 16.0, 11)
    g = np.random.default_rng(12)
    x = g.standard_normal((L, d_model))
    q = g.standard_normal((H, d))
    kparts = O.headwise_factors(Wk, n_kv, d, [d] * n_kv)
    Av, Bv, _ = O.joint_factors(Wv, min(d_model, n_kv * d))
    got = O.decode_attention_hybrid(q, [O.project(x, a) for a, _, _ in kparts], O.project(x, Av),
                                    [b for _, b, _ in kparts], Bv, 10000.0, n_kv)
    want = _sdpa_reference(q, x @ Wk, x @ Wv, 10000.0, n_kv)
    assert np.max(np.abs(got - want)) <= 1e-12 * max(1.0, np.max(np.abs(want)))


def test_truncated_hybrid_equals_attention_on_rank_r_projections():
    d_model, n_kv, d, L, H = 256, 4, 64, 150, 8
    Wk, Wv = _layer(d_model, n_kv, d, 16.0, 13)
    g = np.random.default_rng(14)
    x = g.standard_normal((L, d_model))
    q = g.standard_normal((H, d))
    kparts = O.headwise_factors(Wk, n_kv, d, [9, 30, 64, 2])
    Av, Bv, _ = O.joint_factors(Wv, 70)
    got = O.decode_attention_hybrid(q, [O.project(x, a) for a, _, _ in kparts], O.project(x, Av),
                                    [b for _, b, _ in kparts], Bv, 500000.0, n_kv)
    Wk_r = np.concatenate([a @ b for a, b, _ in kparts], axis=1)
    want = _sdpa_reference(q, x @ Wk_r, x @ (Av @ Bv), 500000.0, n_kv)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_gqa_heads_share_keys_and_single_token_returns_its_value():
    d, n_kv, H = 16, 2, 6
    g = np.random.default_rng(15)
    C_k = [g.standard_normal((1, 5)), g.standard_normal((1, 3))]
    B_k = [g.standard_normal((5, d)), g.standard_normal((3, d))]
    C_v = g.standard_normal((1, 7))
    B_v = g.standard_normal((7, n_kv * d))
    q = np.repeat(g.standard_normal((1, d)), H, axis=0)
    out = O.decode_attention_hybrid(q, C_k, C_v, B_k, B_v, 10000.0, n_kv)
    G = H // n_kv
    for h in range(H):
        kv = h // G
        # one token: softmax weight 1, so o_h is the token's value row of head kv
        np.testing.assert_allclose(out[h], (C_v @ B_v)[0, kv * d:(kv + 1) * d], rtol=1e-12)
