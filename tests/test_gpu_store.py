"""GPU parity of the latent store (quantise + pack + scatter into pages) and of the
read-back: bit-exact against the oracle on the same fp32 latents."""
import os

import numpy as np
import pytest
import torch

import oracle as O
from rank_quantized_kv_decode_b200 import _lib as L
from rank_quantized_kv_decode_b200 import api

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _layout(fmt, key_rank, value_ranks, H=None):
    Hkv = len(value_ranks)
    return api.layout_init(api.make_config(H or Hkv, Hkv, 128, 256, key_rank, value_ranks, fmt, 10000.0))


def _scatter(g, n_tok, batch, max_pages, num_pages):
    table = g.permutation(num_pages).astype(np.int32)[:batch * max_pages].reshape(batch, max_pages)
    # distinct (seq, pos) pairs, in random order
    pairs = g.choice(batch * max_pages * 64, size=n_tok, replace=False)
    seq = (pairs // (max_pages * 64)).astype(np.int32)
    pos = (pairs % (max_pages * 64)).astype(np.int32)
    return table, seq, pos


def _latents(g, n, ranks):
    cols = []
    for r in ranks:
        std = np.exp(-np.arange(r) / max(r / 4, 1.0))
        cols.append(g.standard_normal((n, r)) * std * 3.0)
    lat = np.concatenate(cols, axis=1).astype(np.float32)
    lat[::17] = 0.0                      # all-zero tokens
    lat[5::23, :8] = np.float32(2.5)     # exact ties after scaling in the int8 part
    return lat


@pytest.mark.parametrize("fmt,key_rank,value_ranks", [
    ("f32", 64, [40, 44, 47, 50]),
    ("bf16", 128, [16, 64, 33, 20]),
    ("mixed", 256, [8, 48, 37, 17, 32, 29, 40, 45]),
    ("mixed", 1024, [16, 64, 23, 41]),
    ("mixed", 48, [1, 2, 3, 127 // 2]),
])
def test_quant_pack_bit_exact(fmt, key_rank, value_ranks):
    g = np.random.default_rng(hash((fmt, key_rank)) % 2**32)
    lay = _layout(fmt, key_rank, value_ranks)
    batch, max_pages, num_pages = 3, 6, 23
    n_tok = 700
    table, seq, pos = _scatter(g, n_tok, batch, max_pages, num_pages)
    lat = _latents(g, n_tok, [key_rank] + value_ranks)
    dev = "cuda"
    cache = torch.zeros(num_pages * lay.page_bytes, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    t_table = torch.from_numpy(table).to(dev)
    t_seq, t_pos = torch.from_numpy(seq).to(dev), torch.from_numpy(pos).to(dev)
    api.quant_pack(lay, torch.from_numpy(lat).to(dev), t_seq, t_pos, t_table, cache, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref_layout = O.page_layout(fmt, key_rank, value_ranks, page_tokens=64)
    ref = np.zeros((num_pages, ref_layout["page_bytes"]), np.uint8)
    O.encode_tokens(ref, ref_layout, table, seq, pos, lat)
    got = cache.cpu().numpy().reshape(num_pages, lay.page_bytes)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at page/byte {bad[:5].tolist()}"
    # read-back: dequantised values exactly equal the oracle's stored values
    out = torch.empty(n_tok, lay.proj_cols, dtype=torch.float32, device=dev)
    api.dequant(lay, cache, t_seq, t_pos, t_table, out, status)
    torch.cuda.synchronize()
    want = np.concatenate(
        [np.stack([O.decode_token(ref[table[s, p // 64]], ref_layout, li, p % 64)
                   for s, p in zip(seq[:64], pos[:64])]) for li in range(1 + len(value_ranks))], axis=1)
    np.testing.assert_array_equal(out.cpu().numpy()[:64].astype(np.float64), want)


def _golden_groups():
    rows = []
    with open(os.path.join(GOLDEN, "quant_groups.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, vals, s16, codes = [p.strip() for p in line.split(";")]
            rows.append((int(bits), [float.fromhex(v) if "0x" in v else float(v) for v in vals.split()],
                         int(s16, 16), [int(c) for c in codes.split()]))
    return rows


@pytest.mark.parametrize("case", _golden_groups())
def test_golden_groups_on_gpu(case):
    """The hand-worked groups, placed in the first int8 group (bits 8) or the first int4
    group (bits 4) of a rank-128 latent; the other channels are zero (no effect on amax)."""
    bits, vals, s16_bits, codes = case
    lay = _layout("mixed", 128, [1])
    lat = np.zeros((1, lay.proj_cols), np.float32)
    start = 0 if bits == 8 else 32  # n8 = 32 for r = 128
    lat[0, start:start + len(vals)] = vals
    dev = "cuda"
    cache = torch.zeros(lay.page_bytes, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    one = torch.zeros(1, dtype=torch.int32, device=dev)
    table = torch.zeros(1, 1, dtype=torch.int32, device=dev)
    api.quant_pack(lay, torch.from_numpy(lat).to(dev), one, one, table, cache, status)
    page = cache.cpu().numpy()
    seg = lay.seg[0]
    scales = page[seg.off_sc:seg.off_sc + 2 * (seg.g8 + seg.g4)].view(np.uint16)
    if bits == 8:
        got_codes = page[seg.off_i8:seg.off_i8 + len(vals)].view(np.int8).tolist()
        assert int(scales[0]) == s16_bits
    else:
        got_codes = O.unpack_int4(page[seg.off_i4:seg.off_i4 + seg.nb4], seg.n4)[:len(vals)].tolist()
        assert int(scales[1]) == s16_bits
    assert got_codes == codes


def test_bad_page_and_position_flagged_not_written():
    lay = _layout("mixed", 64, [8, 8])
    dev = "cuda"
    num_pages = 2
    cache = torch.zeros(num_pages * lay.page_bytes, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    table = torch.tensor([[0, 7], [1, -1]], dtype=torch.int32, device=dev)  # 7, -1 invalid
    seq = torch.tensor([0, 1, 0, 1], dtype=torch.int32, device=dev)
    pos = torch.tensor([64, 70, 128, 3], dtype=torch.int32, device=dev)  # page 7, page -1, past table, ok
    lat = torch.ones(4, lay.proj_cols, dtype=torch.float32, device=dev)
    api.quant_pack(lay, lat, seq, pos, table, cache, status)
    torch.cuda.synchronize()
    assert status.item() & L.DEV_BOUNDS
    data = cache.cpu().numpy().reshape(num_pages, lay.page_bytes)
    assert data[0].max() == 0           # nothing reached page 0
    assert data[1].max() > 0            # the valid token (seq 1, pos 3) landed in page 1
