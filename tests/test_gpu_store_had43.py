"""GPU parity of the store and read-back of the pages' own 4-bit/3-bit format (STAR-KV
technical summary, Methodology §3: block-wise Hadamard rotation folded into the factors, the
leading fifth of a latent's channels as 4-bit codes, the rest as 3-bit codes, fp16 group
scales): bit-exact against the oracle on the same fp32 latents, the hand-worked groups, and
the write path with rotated down-projection factors."""
import os

import numpy as np
import pytest
import torch

import oracle as O
from rank_quantized_kv_decode_b200 import api

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _layout(key_rank, value_ranks, d=128, d_model=256):
    Hkv = len(value_ranks)
    return api.layout_init(api.make_config(Hkv, Hkv, d, d_model, key_rank, value_ranks, "had43",
                                           10000.0))


def _rotated_latents(g, n, ranks):
    """Latents with singular-value decay, rotated per latent by the format's transform."""
    cols = []
    for r in ranks:
        c = g.standard_normal((n, r)) * np.exp(-np.arange(r) / max(r / 4, 1.0)) * 3.0
        cols.append(c @ O.hadamard_transform(r))
    lat = np.concatenate(cols, axis=1).astype(np.float32)
    lat[::17] = 0.0                      # all-zero tokens
    lat[5::23, :4] = np.float32(2.5)     # ties after scaling
    return lat


@pytest.mark.parametrize("key_rank,value_ranks", [
    (256, [8, 48, 37, 17, 32, 29, 40, 45]),
    (1024, [16, 64, 23, 41]),
    (16, [1, 2, 3, 5]),
    (48, [128, 100, 7, 64]),
])
def test_quant_pack_bit_exact(key_rank, value_ranks):
    g = np.random.default_rng(key_rank * 31 + len(value_ranks))
    lay = _layout(key_rank, value_ranks)
    batch, max_pages, num_pages = 3, 6, 23
    n_tok = 700
    table = g.permutation(num_pages).astype(np.int32)[:batch * max_pages].reshape(batch, max_pages)
    pairs = g.choice(batch * max_pages * 64, size=n_tok, replace=False)
    seq = (pairs // (max_pages * 64)).astype(np.int32)
    pos = (pairs % (max_pages * 64)).astype(np.int32)
    lat = _rotated_latents(g, n_tok, [key_rank] + value_ranks)
    dev = "cuda"
    cache = torch.zeros(num_pages * lay.page_bytes, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    t_table = torch.from_numpy(table).to(dev)
    t_seq, t_pos = torch.from_numpy(seq).to(dev), torch.from_numpy(pos).to(dev)
    api.quant_pack(lay, torch.from_numpy(lat).to(dev), t_seq, t_pos, t_table, cache, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref_layout = O.page_layout(O.HAD43, key_rank, value_ranks, page_tokens=64)
    assert ref_layout["page_bytes"] == lay.page_bytes
    ref = np.zeros((num_pages, lay.page_bytes), np.uint8)
    O.encode_tokens(ref, ref_layout, table, seq, pos, lat)
    got = cache.cpu().numpy().reshape(num_pages, lay.page_bytes)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at page/byte {bad[:5].tolist()}"
    out = torch.empty(n_tok, lay.proj_cols, dtype=torch.float32, device=dev)
    api.dequant(lay, cache, t_seq, t_pos, t_table, out, status)
    torch.cuda.synchronize()
    want = np.concatenate(
        [np.stack([O.decode_token(ref[table[s, p // 64]], ref_layout, li, p % 64)
                   for s, p in zip(seq[:64], pos[:64])]) for li in range(1 + len(value_ranks))], axis=1)
    np.testing.assert_array_equal(out.cpu().numpy()[:64].astype(np.float64), want)


def _golden(name, bits):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            b, vals, s16, codes = [p.strip() for p in line.split(";")]
            if int(b) == bits:
                rows.append(([float.fromhex(v) if "0x" in v else float(v) for v in vals.split()],
                             int(s16, 16), [int(c) for c in codes.split()]))
    return rows


@pytest.mark.parametrize("bits,case", [(4, c) for c in _golden("quant_groups.txt", 4)]
                         + [(3, c) for c in _golden("quant_groups_3bit.txt", 3)])
def test_golden_groups_on_gpu(bits, case):
    """The hand-worked 4-bit groups at the start of the outlier block and the 3-bit groups at
    the start of the inlier block of a rank-48 key latent (10 outlier channels); the other
    channels are zero."""
    vals, s16_bits, codes = case
    lay = _layout(48, [1])
    seg = lay.seg[0]
    assert (seg.n8, seg.n4) == (10, 38)
    lat = np.zeros((1, lay.proj_cols), np.float32)
    start = 0 if bits == 4 else seg.n8
    lat[0, start:start + len(vals)] = vals
    dev = "cuda"
    cache = torch.zeros(lay.page_bytes, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    table = torch.zeros(1, 1, dtype=torch.int32, device=dev)
    api.quant_pack(lay, torch.from_numpy(lat).to(dev), zero, zero, table, cache, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    page = cache.cpu().numpy()
    scales = page[seg.off_sc:seg.off_sc + 2 * (seg.g8 + seg.g4)].view(np.uint16)
    if bits == 4:
        got = O.unpack_int4(page[seg.off_i8:seg.off_i8 + seg.pitch], seg.n8)[:len(vals)].tolist()
        assert int(scales[0]) == s16_bits
    else:
        got = O.unpack_int3(page[seg.off_i4:seg.off_i4 + seg.nb4], seg.n4)[:len(vals)].tolist()
        assert int(scales[seg.g8]) == s16_bits
    assert got == codes


def test_append_with_rotated_factors():
    """x A' on the tensor cores (bf16 operands, fp32 accumulation) with A' = A T folded per
    latent, then the 4-bit/3-bit store: the projection within 1e-4 of the row scale of the
    oracle's, the stored values within one quantisation step of the oracle's storage of its
    own latents, and rarely different."""
    g = np.random.default_rng(43)
    key_rank, value_ranks, d_model = 256, [8, 48, 37, 17, 32, 29, 40, 45], 512
    lay = _layout(key_rank, value_ranks, d_model=d_model)
    ranks = [key_rank] + value_ranks
    blocks = []
    for r in ranks:
        A = g.standard_normal((d_model, r)) * np.exp(-np.arange(r) / max(r / 4, 1.0)) / np.sqrt(d_model)
        A_rot, _ = O.rotate_factors(A, np.eye(r))
        blocks.append(A_rot)
    A_bf = torch.from_numpy(np.concatenate(blocks, axis=1).astype(np.float32)).to(torch.bfloat16)
    n_tok, batch, max_pages = 333, 2, 8
    x_bf = torch.from_numpy(g.standard_normal((n_tok, d_model)).astype(np.float32)).to(torch.bfloat16)
    dev = "cuda"
    lc = api.LatentCache.create(lay, batch * max_pages, batch, max_pages, n_tok, dev)
    lc.cache.zero_()
    pairs = g.choice(batch * max_pages * 64, size=n_tok, replace=False)
    seq = torch.from_numpy((pairs // (max_pages * 64)).astype(np.int32)).to(dev)
    pos = torch.from_numpy((pairs % (max_pages * 64)).astype(np.int32)).to(dev)
    table = torch.arange(batch * max_pages, dtype=torch.int32, device=dev).reshape(batch, max_pages)
    A_t = A_bf.t().contiguous().to(dev)
    lat_out = torch.empty(n_tok, lay.proj_cols, dtype=torch.float32, device=dev)
    api.append(lay, x_bf.to(dev), A_t, seq, pos, table, lc.cache, lc.append_ws, lc.status,
               latents_out=lat_out)
    torch.cuda.synchronize()
    assert lc.status.item() == 0
    want = O.project(x_bf.float().numpy(), A_bf.float().numpy())
    got = lat_out.cpu().numpy().astype(np.float64)
    scale = np.linalg.norm(want, axis=1, keepdims=True) / np.sqrt(want.shape[1])
    assert np.max(np.abs(got - want) / scale) < 1e-4
    back = torch.empty_like(lat_out)
    api.dequant(lay, lc.cache, seq, pos, table, back, lc.status)
    torch.cuda.synchronize()
    stored_gpu = back.cpu().numpy().astype(np.float64)
    cols = np.concatenate([[0], np.cumsum(ranks)])
    want32 = want.astype(np.float32)
    diff_frac = []
    for li, r in enumerate(ranks):
        for n in range(n_tok):
            qh, ql, sc = O.quantize_hadamard_latent(want32[n, cols[li]:cols[li + 1]], r)
            ref = O.dequantize_hadamard_latent(qh, ql, sc, r)
            diff = np.abs(stored_gpu[n, cols[li]:cols[li + 1]] - ref)
            assert np.all(diff <= 1.01 * float(sc.astype(np.float64).max()) + 1e-12)
            diff_frac.append(np.mean(diff > 0))
    assert np.mean(diff_frac) < 1e-2, f"{np.mean(diff_frac):.2e} of stored values differ"
