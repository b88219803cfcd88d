"""Pins of the oracle's RoPE and decode attention (no GPU): closed forms, an independent
complex-number formulation of RoPE, the relative-position property, and equality with
standard attention (torch's scaled_dot_product_attention in fp64) when the rank is full
and nothing is quantised."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from rank_quantized_kv_decode_b200 import synth


def test_rope_d2_closed_form():
    # d = 2: one pair, theta_0 = base^0 = 1, so position t rotates by t radians
    v = np.array([1.0, 0.0])
    np.testing.assert_allclose(O.apply_rope(v, math.pi / 2, 10000.0), [0.0, 1.0], atol=1e-15)
    np.testing.assert_allclose(O.apply_rope(np.array([0.3, -0.4]), 1.0, 500000.0),
                               [0.3 * math.cos(1) + 0.4 * math.sin(1), -0.4 * math.cos(1) + 0.3 * math.sin(1)],
                               atol=1e-15)


def test_rope_half_split_pairs_d4():
    # d = 4, base 100: pairs (0, 2) at frequency 1 and (1, 3) at frequency 100^(-1/2) = 0.1
    v = np.array([1.0, 2.0, 3.0, 4.0])
    t = 2.0
    a0, a1 = t * 1.0, t * 0.1
    want = [1 * math.cos(a0) - 3 * math.sin(a0), 2 * math.cos(a1) - 4 * math.sin(a1),
            3 * math.cos(a0) + 1 * math.sin(a0), 4 * math.cos(a1) + 2 * math.sin(a1)]
    np.testing.assert_allclose(O.apply_rope(v, t, 100.0), want, atol=1e-14)


@pytest.mark.parametrize("d,theta", [(64, 10000.0), (128, 500000.0)])
def test_rope_matches_complex_formulation(d, theta):
    g = np.random.default_rng(d)
    v = g.standard_normal((5, d))
    pos = np.array([0, 1, 77, 4095, 131071])
    z = v[:, :d // 2] + 1j * v[:, d // 2:]
    freqs = np.array([theta ** (-(2.0 * j) / d) for j in range(d // 2)])
    zr = z * np.exp(1j * pos[:, None] * freqs[None, :])
    want = np.concatenate([zr.real, zr.imag], axis=1)
    # angles reach 1.3e5 rad; fp64 rounding of pos*freq is ~1.3e5 * 2^-52 per formulation
    np.testing.assert_allclose(O.apply_rope(v, pos, theta), want, rtol=0, atol=5e-10)


def test_rope_relative_position_and_norm():
    g = np.random.default_rng(1)
    q, k = g.standard_normal(128), g.standard_normal(128)
    m, n = 4000, 17
    a = O.apply_rope(q, m, 10000.0) @ O.apply_rope(k, n, 10000.0)
    b = O.apply_rope(q, m + 321, 10000.0) @ O.apply_rope(k, n + 321, 10000.0)
    assert abs(a - b) < 1e-10
    assert abs(np.linalg.norm(O.apply_rope(q, 99999, 10000.0)) - np.linalg.norm(q)) < 1e-12


def _sdpa_reference(q, K, V, theta, n_kv):
    """Standard attention with explicit keys and values: torch SDPA in fp64."""
    H, d = q.shape
    L = K.shape[0]
    G = H // n_kv
    Kh = np.stack([O.apply_rope(K[:, g * d:(g + 1) * d], np.arange(L), theta) for g in range(n_kv)])
    Vh = np.stack([V[:, g * d:(g + 1) * d] for g in range(n_kv)])
    qh = np.stack([O.apply_rope(q[h], L - 1, theta) for h in range(H)])
    Kt = torch.from_numpy(Kh).repeat_interleave(G, dim=0)[None]
    Vt = torch.from_numpy(Vh).repeat_interleave(G, dim=0)[None]
    qt = torch.from_numpy(qh)[None, :, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)
    return o[0, :, 0, :].numpy()


def _layer(d_model, n_kv, d, scale, seed):
    g = np.random.default_rng(seed)
    n = n_kv * d
    k = min(d_model, n)
    s = synth.spectrum(k, scale)
    Wk = (synth.haar_frame(g, d_model, k) * s) @ synth.haar_frame(g, n, k).T
    Wv = (synth.haar_frame(g, d_model, k) * s) @ synth.haar_frame(g, n, k).T
    return Wk, Wv


@pytest.mark.parametrize("H,n_kv", [(4, 4), (8, 2)])
def test_full_rank_unquantised_equals_standard_attention(H, n_kv):
    d_model, d, L = 256, 64, 256
    Wk, Wv = _layer(d_model, n_kv, d, 16.0, 7)
    g = np.random.default_rng(8)
    x = g.standard_normal((L, d_model))
    q = g.standard_normal((H, d))
    r_full = min(d_model, n_kv * d)
    Ak, Bk, _ = O.joint_factors(Wk, r_full)
    parts = O.headwise_factors(Wv, n_kv, d, [d] * n_kv)
    Ck = O.project(x, Ak)
    Cv = [O.project(x, a) for a, _, _ in parts]
    Bv = [b for _, b, _ in parts]
    got = O.decode_attention(q, Ck, Cv, Bk, Bv, 10000.0, n_kv)
    want = _sdpa_reference(q, x @ Wk, x @ Wv, 10000.0, n_kv)
    assert np.max(np.abs(got - want)) <= 1e-12 * max(1.0, np.max(np.abs(want)))


def test_truncated_rank_equals_attention_on_rank_r_projection():
    # at rank r the keys/values are exactly those of the best rank-r projections W_r
    d_model, n_kv, d, L, H = 256, 4, 64, 200, 4
    Wk, Wv = _layer(d_model, n_kv, d, 16.0, 9)
    g = np.random.default_rng(10)
    x = g.standard_normal((L, d_model))
    q = g.standard_normal((H, d))
    Ak, Bk, _ = O.joint_factors(Wk, 40)
    ranks = [5, 17, 33, 64]
    parts = O.headwise_factors(Wv, n_kv, d, ranks)
    got = O.decode_attention(q, O.project(x, Ak), [O.project(x, a) for a, _, _ in parts],
                             Bk, [b for _, b, _ in parts], 10000.0, n_kv)
    Wv_r = np.concatenate([a @ b for a, b, _ in parts], axis=1)
    want = _sdpa_reference(q, x @ (Ak @ Bk), x @ Wv_r, 10000.0, n_kv)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_zero_query_gives_mean_of_values():
    g = np.random.default_rng(2)
    L, r_k, H, n_kv, d = 50, 12, 4, 2, 16
    Ck = g.standard_normal((L, r_k))
    Bk = g.standard_normal((r_k, n_kv * d))
    Cv = [g.standard_normal((L, 5)), g.standard_normal((L, 7))]
    Bv = [g.standard_normal((5, d)), g.standard_normal((7, d))]
    out = O.decode_attention(np.zeros((H, d)), Ck, Cv, Bk, Bv, 10000.0, n_kv)
    for h in range(H):
        gg = h // 2
        np.testing.assert_allclose(out[h], Cv[gg].mean(0) @ Bv[gg], rtol=1e-12)


def test_sharp_query_selects_one_token_and_gqa_mapping():
    # one key row aligned with the (rotated) query dominates the softmax
    L, n_kv, d, H = 30, 2, 8, 4
    Ck = np.eye(L)[:, :L]  # latent t is e_t, r_k = L
    g = np.random.default_rng(3)
    Bk = np.zeros((L, n_kv * d))
    Bk[11, 0:d] = 1.0   # only token 11 has a key in KV head 0
    Bk[23, d:2 * d] = 1.0  # only token 23 has a key in KV head 1
    Cv = [np.eye(L), np.eye(L)]
    Bv = [g.standard_normal((L, d)), g.standard_normal((L, d))]
    q = np.zeros((H, d))
    for h in range(H):
        gg = h // 2
        t = 11 if gg == 0 else 23
        k_rot = O.apply_rope(np.ones(d), t, 10000.0)
        q[h] = 200.0 * O.apply_rope(k_rot, -(L - 1), 10000.0)  # undo the query's rotation
    out = O.decode_attention(q, Ck, Cv, Bk, Bv, 10000.0, n_kv)
    np.testing.assert_allclose(out[0], Bv[0][11], atol=1e-9)
    np.testing.assert_allclose(out[1], Bv[0][11], atol=1e-9)
    np.testing.assert_allclose(out[2], Bv[1][23], atol=1e-9)
    np.testing.assert_allclose(out[3], Bv[1][23], atol=1e-9)


def test_single_token_context():
    g = np.random.default_rng(4)
    Ck = g.standard_normal((1, 6))
    Bk = g.standard_normal((6, 16))
    Cv = [g.standard_normal((1, 3))]
    Bv = [g.standard_normal((3, 16))]
    out = O.decode_attention(g.standard_normal((2, 16)), Ck, Cv, Bk, Bv, 10000.0, 1)
    np.testing.assert_allclose(out, np.stack([Cv[0][0] @ Bv[0]] * 2), rtol=1e-12)


def _tiny_latents(seed, L, H, Hkv, d, rk, ranks):
    g = np.random.default_rng(seed)
    q = g.standard_normal((H, d))
    Ck = g.standard_normal((L, rk))
    Cv = [g.standard_normal((L, r)) for r in ranks]
    Bk = g.standard_normal((rk, Hkv * d)) / math.sqrt(rk)
    return q, Ck, Cv, Bk


@pytest.mark.parametrize("L,tile", [(1, 128), (5, 2), (300, 128), (256, 128), (7, 7)])
def test_tile_partials_merge_to_latent_attention(L, tile):
    """The log-sum-exp merge of the per-block records is the whole-sequence softmax output."""
    H, Hkv, d = 4, 2, 8
    q, Ck, Cv, Bk = _tiny_latents(L, L, H, Hkv, d, 6, [3, 5])
    want = O.latent_attention(q, Ck, Cv, Bk, 10000.0, Hkv)
    parts = O.tile_partials(q, Ck, Cv, Bk, 10000.0, Hkv, tile=tile)
    for h in range(H):
        blocks = parts[h]
        assert len(blocks) == -(-L // tile)
        M = max(m for m, _, _ in blocks)
        num = sum(2.0 ** (m - M) * a for m, _, a in blocks)
        den = sum(2.0 ** (m - M) * l for m, l, _ in blocks)
        np.testing.assert_allclose(num / den, want[h], rtol=1e-12, atol=1e-14)
        for m, l, a in blocks:
            # the block's own maximum term is 2^0 = 1: 1 <= l <= block length
            assert 1.0 - 1e-12 <= l <= tile + 1e-12


def test_tile_partials_hand_worked():
    """d = 2 (one RoPE pair, frequency 1), one KV head, keys reconstructed by an identity B:
    the scores are q'.k'_t / sqrt(2) with q' rotated by (L-1) and k_t by t radians."""
    q = np.array([[1.0, 0.0]])
    Ck = np.array([[1.0, 0.0], [0.0, 1.0], [2.0, 0.0]])  # L = 3
    Cv = [np.array([[1.0], [10.0], [100.0]])]
    Bk = np.eye(2)
    parts = O.tile_partials(q, Ck, Cv, Bk, 10000.0, 1, tile=2)
    # q' = (cos 2, sin 2); k'_0 = (1, 0); k'_1 = rot(1)(0, 1) = (-sin 1, cos 1);
    # k'_2 = rot(2)(2, 0) = (2 cos 2, 2 sin 2)
    s = np.array([math.cos(2),
                  -math.cos(2) * math.sin(1) + math.sin(2) * math.cos(1),
                  2.0]) / math.sqrt(2) / math.log(2)
    (m0, l0, a0), (m1, l1, a1) = parts[0]
    assert m0 == pytest.approx(max(s[0], s[1]), abs=1e-14)
    assert l0 == pytest.approx(2 ** (s[0] - m0) + 2 ** (s[1] - m0), abs=1e-14)
    assert a0[0] == pytest.approx(2 ** (s[0] - m0) * 1 + 2 ** (s[1] - m0) * 10, abs=1e-12)
    assert (m1, l1) == (pytest.approx(s[2], abs=1e-14), pytest.approx(1.0, abs=1e-15))
    assert a1[0] == pytest.approx(100.0, abs=1e-12)
