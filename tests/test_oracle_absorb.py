"""Pins of the oracle's weight absorption (STAR-KV technical summary, Methodology §2: the
value up-projection folded into the attention output projection).

* With W_o = I (d_out = H d) the absorbed output is the concatenation of the per-head
  outputs of decode_attention (a special case that reduces to the pinned path).
* For any W_o it equals the unabsorbed evaluation (concat_h o_h) W_o: the other association
  of the same product, computed from decode_attention's outputs.
* A W_o that is zero outside the rows of one head h makes the output depend on head h alone.
"""
import numpy as np

import oracle as O


def _case(seed, H=8, H_kv=4, d=16, L=37, r_k=24, ranks=(5, 9, 3, 7)):
    g = np.random.default_rng(seed)
    q = g.standard_normal((H, d))
    C_k = g.standard_normal((L, r_k))
    C_v = [g.standard_normal((L, r)) for r in ranks]
    B_k = g.standard_normal((r_k, H_kv * d)) / np.sqrt(r_k)
    B_v = [g.standard_normal((r, d)) for r in ranks]
    return q, C_k, C_v, B_k, B_v, H, H_kv, d


def test_identity_output_projection_gives_the_concatenated_head_outputs():
    q, C_k, C_v, B_k, B_v, H, H_kv, d = _case(1)
    W_o = np.eye(H * d)
    M = O.absorb_output_weights(B_v, W_o, H)
    y = O.decode_attention_absorbed(q, C_k, C_v, B_k, M, 10000.0, H_kv)
    o = O.decode_attention(q, C_k, C_v, B_k, B_v, 10000.0, H_kv)
    np.testing.assert_allclose(y, o.reshape(-1), rtol=1e-12, atol=1e-12)


def test_absorbed_equals_unabsorbed_output_projection():
    q, C_k, C_v, B_k, B_v, H, H_kv, d = _case(2)
    d_out = 50
    W_o = np.random.default_rng(3).standard_normal((H * d, d_out))
    M = O.absorb_output_weights(B_v, W_o, H)
    assert [m.shape for m in M] == [(B_v[h // (H // H_kv)].shape[0], d_out) for h in range(H)]
    y = O.decode_attention_absorbed(q, C_k, C_v, B_k, M, 500000.0, H_kv)
    o = O.decode_attention(q, C_k, C_v, B_k, B_v, 500000.0, H_kv)
    np.testing.assert_allclose(y, o.reshape(-1) @ W_o, rtol=1e-10, atol=1e-10)


def test_output_rows_of_one_head_select_that_head():
    q, C_k, C_v, B_k, B_v, H, H_kv, d = _case(4)
    d_out = 11
    for h in (0, 5):
        W_o = np.zeros((H * d, d_out))
        W_o[h * d:(h + 1) * d] = np.random.default_rng(h).standard_normal((d, d_out))
        M = O.absorb_output_weights(B_v, W_o, H)
        y = O.decode_attention_absorbed(q, C_k, C_v, B_k, M, 10000.0, H_kv)
        o_h = O.decode_attention(q, C_k, C_v, B_k, B_v, 10000.0, H_kv, heads=[h])[0]
        np.testing.assert_allclose(y, o_h @ W_o[h * d:(h + 1) * d], rtol=1e-12, atol=1e-12)
        # the other heads' absorbed factors are zero
        assert all(np.count_nonzero(M[k]) == 0 for k in range(H) if k != h)
