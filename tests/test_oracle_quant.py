"""Pins of the oracle's quantiser, int4 packing, page layout and compression accounting
(no GPU)."""
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_float(tok):
    return float.fromhex(tok) if "0x" in tok else float(tok)


def _golden_groups():
    rows = []
    with open(os.path.join(GOLDEN, "quant_groups.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, vals, s16, codes = [p.strip() for p in line.split(";")]
            rows.append((int(bits), np.array([_parse_float(v) for v in vals.split()], np.float32),
                         int(s16, 16), [int(c) for c in codes.split()]))
    return rows


@pytest.mark.parametrize("row", _golden_groups())
def test_quantize_group_golden(row):
    bits, vals, s16_bits, codes = row
    s16, q = O.quantize_group(vals, bits)
    assert int(np.array(s16, np.float16).view(np.uint16)) == s16_bits
    assert q.tolist() == codes


def test_int4_pack_exhaustive():
    for a in range(-8, 8):
        for b in range(-8, 8):
            packed = O.pack_int4([a, b])
            assert packed.shape == (1,)
            assert O.unpack_int4(packed, 2).tolist() == [a, b]
    for byte in range(256):
        codes = O.unpack_int4(np.array([byte], np.uint8), 2)
        assert int(O.pack_int4(codes)[0]) == byte
    # odd count: the unused high nibble is zero
    assert O.pack_int4([-1]).tolist() == [0x0F]
    assert O.pack_int4([3, -2, 5]).tolist() == [0xE3, 0x05]


def test_int8_codes_roundtrip_through_page():
    lay = O.page_layout(O.MIXED, 128, [], page_tokens=4)
    page = np.zeros(lay["page_bytes"], np.uint8)
    # channel values chosen so that every int8 code -127..127 appears with scale 1
    sp = O.mixed_split(128)
    assert sp["n8"] == 32
    for start in range(-127, 128, 32):
        c = np.zeros(128, np.float32)
        codes8 = np.arange(start, start + 32).clip(-127, 127)
        c[:32] = codes8
        c[0] = 127.0  # group absmax 127 -> scale exactly 1
        c[32:] = np.tile(np.arange(-7, 8), 7)[:96]
        c[32] = 7.0
        c[64] = 7.0
        c[96] = 7.0
        O.encode_token(page, lay, 0, 1, c)
        back = O.decode_token(page, lay, 0, 1)
        np.testing.assert_array_equal(back, c.astype(np.float64))


def test_dequantisation_is_exact_and_error_bounded():
    g = np.random.default_rng(0)
    for r in [8, 17, 37, 64, 256]:
        for trial in range(20):
            c = (g.standard_normal(r) * np.exp(-np.arange(r) / 16)).astype(np.float32)
            q8, q4, sc = O.quantize_latent(c, r)
            chat = O.dequantize_latent(q8, q4, sc, r)
            sp = O.mixed_split(r)
            # exact in fp32: the fp32 product equals the fp64 product
            s_of = np.array([float(sc[i // 32]) for i in range(sp["n8"])] +
                            [float(sc[sp["g8"] + i // 32]) for i in range(sp["n4"])])
            codes = np.concatenate([q8, q4]).astype(np.float64)
            np.testing.assert_array_equal((s_of.astype(np.float32) * codes.astype(np.float32)),
                                          chat.astype(np.float32))
            np.testing.assert_array_equal(s_of * codes, chat)
            # rounding error at most half a step where the code is not clamped
            qmax = np.array([127.0] * sp["n8"] + [7.0] * sp["n4"])
            free = np.abs(codes) < qmax
            assert np.all(np.abs(c.astype(np.float64) - chat)[free] <= s_of[free] / 2 * (1 + 1e-6))
            # clamped codes only occur where the scale was rounded down
            assert np.all(np.abs(codes) <= qmax)


def test_quantize_latent_group_boundaries():
    # r = 37: n8 = 10 (one int8 group), n4 = 27 (one int4 group starting at channel 10)
    sp = O.mixed_split(37)
    assert (sp["n8"], sp["n4"], sp["g8"], sp["g4"], sp["nb4"]) == (10, 27, 1, 1, 14)
    c = np.zeros(37, np.float32)
    c[:10] = 127.0
    c[10:] = 7.0
    c[9] = -254.0  # int8 group amax 254 -> scale 2
    q8, q4, sc = O.quantize_latent(c, 37)
    assert float(sc[0]) == 2.0 and float(sc[1]) == 1.0
    assert q8.tolist() == [64] * 9 + [-127]  # 127/2 = 63.5 -> 64 (half to even)
    assert q4.tolist() == [7] * 27
    # r = 256: groups of 32 restart at the int4 part
    sp = O.mixed_split(256)
    assert (sp["n8"], sp["n4"], sp["g8"], sp["g4"], sp["nb4"]) == (64, 192, 2, 6, 96)


def test_bf16_rne():
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -3.14159, 65504.0], np.float32)
    got = O.bf16_rne(vals)
    # 1+2^-8 is a tie between 1 and 1+2^-7 -> even (1.0); 1+3*2^-8 ties to 1+2^-6 (even)
    assert got.tolist()[:4] == [1.0, 1.0, 1.0 + 2 ** -6, 1.0]
    assert got[4] == np.float32(-3.140625)
    assert got[5] == 65536.0


def test_page_layout_sizes():
    lay = O.page_layout(O.MIXED, 256, [32] * 8, page_tokens=64)
    k = lay["segs"][0]
    # K latent of rank 256: 64 int8 + 96 packed int4 + 8 fp16 scales = 176 bytes per token
    assert k["n8"] + k["nb4"] + 2 * (k["g8"] + k["g4"]) == 176
    # V latent of rank 32: 8 int8 + 12 packed + 2 scales = 24 bytes
    v = lay["segs"][1]
    assert v["n8"] + v["nb4"] + 2 * (v["g8"] + v["g4"]) == 24
    assert lay["token_bytes"] == 176 + 8 * 24
    assert lay["page_bytes"] == 64 * (176 + 8 * 24)
    # blocks are 16-byte aligned and do not overlap
    spans = []
    for s in lay["segs"]:
        for key, w in (("i8", s["n8"]), ("i4", s["nb4"]), ("sc", 2 * (s["g8"] + s["g4"]))):
            assert s[key] % 16 == 0
            spans.append((s[key], s[key] + 64 * w))
    spans.sort()
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    lay2 = O.page_layout(O.BF16, 1024, [32] * 32)
    assert lay2["page_bytes"] == 64 * 2 * 2048
    assert lay2["token_bytes"] == 4096


def test_mixed_format_bits_closed_form():
    # 0.25*8 + 0.75*4 + 16/32 = 5.5 bits per channel when r is a multiple of 128
    for r in [128, 256, 1024]:
        assert O.mixed_bits_per_channel(r) == 5.5


def _accounting():
    out = {}
    with open(os.path.join(GOLDEN, "compression_accounting.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, args, val = [p.strip() for p in line.split(";")]
            out[key] = ([float(a) for a in args.split()], float(val))
    return out


def test_pages_compression_accounting():
    acc = _accounting()
    args, want = acc["avg_bits"]
    assert abs(O.two_level_bits(args[0], int(args[1]), int(args[2])) - want) < 1e-12
    args, want = acc["total_reduction"]
    assert abs(O.total_reduction(args[0], args[1], int(args[2])) - want) < 1e-9


def test_paged_encode_read_roundtrip_with_permuted_table():
    g = np.random.default_rng(6)
    ranks_v = [5, 9]
    for fmt in (O.F32, O.BF16, O.MIXED):
        lay = O.page_layout(fmt, 12, ranks_v, page_tokens=4)
        num_pages, B, maxp = 10, 2, 5
        cache = np.zeros((num_pages, lay["page_bytes"]), np.uint8)
        table = g.permutation(num_pages).astype(np.int32)[:B * maxp].reshape(B, maxp)
        L = [7, 13]
        seq = np.concatenate([[b] * L[b] for b in range(B)])
        pos = np.concatenate([np.arange(L[b]) for b in range(B)])
        lat = g.standard_normal((len(seq), 12 + sum(ranks_v))).astype(np.float32)
        O.encode_tokens(cache, lay, table, seq, pos, lat)
        n = 0
        for b in range(B):
            Ck, Cv = O.read_sequence(cache, lay, table[b], L[b])
            rows = lat[n:n + L[b]]
            n += L[b]
            if fmt == O.MIXED:
                want_k = np.stack([O.dequantize_latent(*O.quantize_latent(r[:12], 12), 12) for r in rows])
            else:
                want_k = O.store_latents(rows[:, :12], fmt)
            np.testing.assert_array_equal(Ck, want_k)
            off = 12
            for gi, r in enumerate(ranks_v):
                if fmt == O.MIXED:
                    want = np.stack([O.dequantize_latent(*O.quantize_latent(x[off:off + r], r), r)
                                     for x in rows])
                else:
                    want = O.store_latents(rows[:, off:off + r], fmt)
                np.testing.assert_array_equal(Cv[gi], want)
                off += r


def test_vector_quantiser_matches_per_token_definition():
    g = np.random.default_rng(9)
    for r in [8, 17, 37, 64, 256]:
        C = (g.standard_normal((40, r)) * np.exp(-np.arange(r) / 20)).astype(np.float32)
        C[3] = 0.0
        C[5, :4] = [1e7, -3e-7, 0, 0]
        q8, q4, sc = O.quantize_rows(C, r)
        for n in range(C.shape[0]):
            a8, a4, asc = O.quantize_latent(C[n], r)
            assert q8[n].tolist() == a8.tolist()
            assert q4[n].tolist() == a4.tolist()
            assert sc[n].view(np.uint16).tolist() == asc.view(np.uint16).tolist()
        np.testing.assert_array_equal(O.dequantize_rows(q8, q4, sc, r),
                                      np.stack([O.dequantize_latent(*O.quantize_latent(c, r), r) for c in C]))
