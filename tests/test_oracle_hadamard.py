"""Pins of the oracle's version of the pages' own quantiser (STAR-KV technical summary,
Methodology §3: block-wise Hadamard rotation of an outlier and an inlier block, 4-bit and
3-bit codes, the rotation folded into the factors):

* the Sylvester matrices and the block transforms are orthogonal, with the closed form at
  order 2 and the block sizes of the binary decomposition;
* folding the transform into the factors leaves their product unchanged;
* a single spike in a block of 2^k channels is spread to 2^-k/2 of its height (the
  smoothing the rotation is there for);
* the 3-bit packing: a hand-worked word, every code at every position, random lengths;
* hand-worked 3-bit groups (tests/golden/quant_groups_3bit.txt): ties to even, a scale that
  rounds down to an fp16 subnormal, saturation, the zero group;
* quantisation error at most half a scale step per channel, groups restarting at the block
  boundary, and the format's average of 3.2 bits per channel (scales excluded) at the
  pages' 20 % / 80 % split.
"""
import math
import os

import numpy as np
import pytest

import oracle as O


def test_sylvester_closed_form_and_orthogonality():
    np.testing.assert_allclose(O.sylvester_hadamard(2), np.array([[1, 1], [1, -1]]) / math.sqrt(2))
    for n in (1, 2, 4, 8, 16, 64):
        H = O.sylvester_hadamard(n)
        np.testing.assert_allclose(H @ H.T, np.eye(n), atol=1e-13)
        np.testing.assert_allclose(np.abs(H), np.full((n, n), 1 / math.sqrt(n)), atol=1e-15)


@pytest.mark.parametrize("n", [1, 3, 5, 13, 20, 51, 64, 80])
def test_block_transform_is_orthogonal_with_binary_blocks(n):
    T = O.block_hadamard(n)
    np.testing.assert_allclose(T @ T.T, np.eye(n), atol=1e-13)
    # block sizes: the set bits of n, largest first, down the diagonal
    at = 0
    for k in reversed(range(n.bit_length())):
        if n & (1 << k):
            size = 1 << k
            np.testing.assert_allclose(T[at:at + size, at:at + size], O.sylvester_hadamard(size))
            assert np.count_nonzero(T[at:at + size, at + size:]) == 0
            at += size
    assert at == n


def test_split_and_transform_blocks():
    sp = O.hadamard_split(100)
    assert (sp["n_hi"], sp["n_lo"]) == (20, 80)
    assert O.hadamard_split(7)["n_hi"] == 2  # rounded up
    T = O.hadamard_transform(37)
    n_hi = O.hadamard_split(37)["n_hi"]
    assert np.count_nonzero(T[:n_hi, n_hi:]) == 0 and np.count_nonzero(T[n_hi:, :n_hi]) == 0
    np.testing.assert_allclose(T @ T.T, np.eye(37), atol=1e-13)


def test_folding_into_the_factors_keeps_the_product():
    g = np.random.default_rng(5)
    A = g.standard_normal((96, 45))
    B = g.standard_normal((45, 128))
    A2, B2 = O.rotate_factors(A, B)
    np.testing.assert_allclose(A2 @ B2, A @ B, rtol=1e-12, atol=1e-12)
    # the latents of the rotated factors are the rotated latents
    x = g.standard_normal((3, 96))
    np.testing.assert_allclose(x @ A2, (x @ A) @ O.hadamard_transform(45), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("k", [2, 4, 6])
def test_a_spike_is_spread_over_its_block(k):
    n = 1 << k
    c = np.zeros(n)
    c[3] = 100.0
    rotated = c @ O.block_hadamard(n)
    np.testing.assert_allclose(np.abs(rotated), np.full(n, 100.0 / math.sqrt(n)), rtol=1e-13)


def test_pack_int3_hand_worked_word():
    # codes 0,1,2,3,-4,-3,-2,-1 are the 3-bit patterns 0..7; the word is
    # sum_i v_i * 8^i = 0o76543210 = 0xFAC688, stored low byte first
    assert O.pack_int3([0, 1, 2, 3, -4, -3, -2, -1]).tolist() == [0x88, 0xC6, 0xFA]


def test_pack_int3_every_code_at_every_position_and_random_lengths():
    for pos in range(8):
        for v in range(-4, 4):
            codes = np.zeros(8, np.int64)
            codes[pos] = v
            packed = O.pack_int3(codes)
            assert packed.size == 3
            np.testing.assert_array_equal(O.unpack_int3(packed, 8), codes)
    g = np.random.default_rng(6)
    for n in range(1, 41):
        codes = g.integers(-4, 4, size=n)
        packed = O.pack_int3(codes)
        assert packed.size == 3 * -(-n // 8)
        np.testing.assert_array_equal(O.unpack_int3(packed, n), codes)


def test_quantisation_error_and_block_groups():
    r = 77
    g = np.random.default_rng(7)
    sigma = np.exp(-np.arange(r) / 16.0)
    c = (g.standard_normal(r) * sigma).astype(np.float32)
    rotated = (c.astype(np.float64) @ O.hadamard_transform(r)).astype(np.float32)
    qh, ql, sc = O.quantize_hadamard_latent(rotated, r)
    sp = O.hadamard_split(r)
    assert qh.size == sp["n_hi"] and ql.size == sp["n_lo"]
    assert sc.size == sp["g_hi"] + sp["g_lo"]
    assert np.abs(qh).max() <= 7 and np.abs(ql).max() <= 3
    back = O.dequantize_hadamard_latent(qh, ql, sc, r)
    step = np.concatenate([np.repeat(sc[:sp["g_hi"]].astype(np.float64), 32)[:sp["n_hi"]],
                           np.repeat(sc[sp["g_hi"]:].astype(np.float64), 32)[:sp["n_lo"]]])
    assert np.all(np.abs(back - rotated) <= step / 2 * (1 + 1e-6) + 1e-12)
    # the inlier block's first group starts at the block boundary: its scale comes from
    # channels [n_hi, n_hi + 32) only
    s_first = O.fp16_scale(np.max(np.abs(rotated[sp["n_hi"]:sp["n_hi"] + 32])), 3)
    assert sc[sp["g_hi"]] == s_first


def test_average_bits_at_the_pages_split():
    r = 1000
    sp = O.hadamard_split(r)
    bits = (4 * sp["n_hi"] + 3 * sp["n_lo"]) / r
    assert bits == O.two_level_bits(0.2, 4, 3) == pytest.approx(3.2)


def test_page_layout_of_the_hadamard_format():
    L = O.page_layout(O.HAD43, 100, [40, 13])
    k = L["segs"][0]
    # rank 100: 20 outlier channels (10 bytes of 4-bit codes), 80 inlier channels (30 bytes
    # of 3-bit codes), 1 + 3 fp16 scales
    assert (k["nb_hi"], k["nb_lo"], k["g_hi"] + k["g_lo"]) == (10, 30, 4)
    assert L["token_bytes"] == (10 + 30 + 8) + (4 + 12 + 4) + (2 + 6 + 4)
    for seg in L["segs"]:
        for key in ("hi", "lo", "sc"):
            assert seg[key] % 16 == 0


def test_page_roundtrip_of_the_hadamard_format():
    g = np.random.default_rng(8)
    ranks = [100, 40, 13]
    L = O.page_layout(O.HAD43, ranks[0], ranks[1:])
    page = np.zeros(L["page_bytes"], np.uint8)
    for slot in (0, 17, 63):
        for li, r in enumerate(ranks):
            c = (g.standard_normal(r) * np.exp(-np.arange(r) / 16.0)).astype(np.float32)
            rot = (c.astype(np.float64) @ O.hadamard_transform(r)).astype(np.float32)
            O.encode_token(page, L, li, slot, rot)
            want = O.dequantize_hadamard_latent(*O.quantize_hadamard_latent(rot, r), r)
            np.testing.assert_array_equal(O.decode_token(page, L, li, slot), want)


def _golden_3bit():
    rows = []
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "quant_groups_3bit.txt")
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, vals, s16, codes = [p.strip() for p in line.split(";")]
            vals = [float.fromhex(v) if "0x" in v else float(v) for v in vals.split()]
            rows.append((int(bits), np.array(vals, np.float32), int(s16, 16), [int(c) for c in codes.split()]))
    return rows


@pytest.mark.parametrize("row", _golden_3bit())
def test_quantize_3bit_group_golden(row):
    bits, vals, s16_bits, codes = row
    assert bits == 3
    s16, q = O.quantize_group(vals, bits)
    assert int(np.array(s16, np.float16).view(np.uint16)) == s16_bits
    assert q.tolist() == codes
    # the same group placed at the start of a rank-40 latent's inlier block, behind an
    # all-zero outlier block (scale 0), comes out of the format's quantiser unchanged
    sp = O.hadamard_split(40)
    c = np.zeros(40, np.float32)
    c[sp["n_hi"]:sp["n_hi"] + len(vals)] = vals
    qh, ql, sc = O.quantize_hadamard_latent(c, 40)
    assert not qh.any() and not sc[:sp["g_hi"]].view(np.uint16).any()
    assert ql[:len(vals)].tolist() == codes
    assert int(sc[sp["g_hi"]:sp["g_hi"] + 1].view(np.uint16)[0]) == s16_bits


def test_vector_quantiser_matches_per_token_definition():
    g = np.random.default_rng(10)
    for r in [1, 8, 17, 37, 64, 256, 1000]:
        C = (g.standard_normal((40, r)) * np.exp(-np.arange(r) / 20)).astype(np.float32)
        C = (C.astype(np.float64) @ O.hadamard_transform(r)).astype(np.float32)
        C[3] = 0.0
        C[5, 0] = 1e7                 # a saturated scale in the first group
        C[6] *= np.float32(1e-9)      # subnormal (or zero) scales in every group
        C[7, -1] = 2.5
        qh, ql, sc = O.quantize_hadamard_rows(C, r)
        for n in range(C.shape[0]):
            ah, al, asc = O.quantize_hadamard_latent(C[n], r)
            assert qh[n].tolist() == ah.tolist()
            assert ql[n].tolist() == al.tolist()
            assert sc[n].view(np.uint16).tolist() == asc.view(np.uint16).tolist()
        want = np.stack([O.dequantize_hadamard_latent(*O.quantize_hadamard_latent(c, r), r) for c in C])
        np.testing.assert_array_equal(O.dequantize_hadamard_rows(qh, ql, sc, r), want)
        np.testing.assert_array_equal(O.stored_rows(C, r, O.HAD43), want)
