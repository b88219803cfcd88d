"""Host-side checks of the C ABI (no GPU): the library loads, exports every entry point the
header declares, and its pure host calls (layout, sizes, validation) agree with the oracle's
independent layout definition."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle as O
from rank_quantized_kv_decode_b200 import _lib as L
from rank_quantized_kv_decode_b200 import api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from rank_quantized_kv_decode_b200 import build
    build.build()
    return L.load()


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "starkv.h")).read()
    return re.findall(r"STARKV_API\s+[\w\s\*]+?\b(starkv_\w+)\s*\(", src)


def test_header_declares_the_abi():
    names = declared_entry_points()
    assert set(names) == set(L.EXPORTS), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_entry_points():
        assert hasattr(lib, name), name
    assert lib.starkv_version() == 100


def test_struct_sizes_match_c(lib):
    # the C side checks that a layout equals starkv_layout_init's output byte for byte,
    # so a ctypes struct of the wrong size would be rejected
    assert ctypes.sizeof(L.Config) == 296
    assert ctypes.sizeof(L.Segment) == 64
    assert ctypes.sizeof(L.HybridConfig) == 296
    assert ctypes.sizeof(L.Layout) == 296 + 16 + 16 + 65 * 64 + 8 + 296


CASES = [
    ("f32", 4, 4, 64, 256, 64, [40, 44, 47, 50]),
    ("bf16", 32, 32, 128, 4096, 1024, [16 + (g * 7) % 49 for g in range(32)]),
    ("mixed", 32, 32, 128, 4096, 1024, [16 + (g * 5) % 49 for g in range(32)]),
    ("mixed", 32, 8, 128, 4096, 256, [8, 48, 37, 17, 32, 29, 40, 45]),
    ("had43", 32, 8, 128, 4096, 256, [8, 48, 37, 17, 32, 29, 40, 45]),
    ("had43", 4, 4, 64, 256, 64, [1, 2, 13, 64]),
]


@pytest.mark.parametrize("fmt,H,Hkv,d,dm,rk,rv", CASES)
def test_layout_matches_oracle(lib, fmt, H, Hkv, d, dm, rk, rv):
    lay = api.layout_init(api.make_config(H, Hkv, d, dm, rk, rv, fmt, 10000.0))
    ref = O.page_layout(fmt, rk, rv, page_tokens=64)
    assert lay.page_bytes == ref["page_bytes"]
    assert lay.token_bytes == ref["token_bytes"]
    assert lay.n_latents == 1 + Hkv
    assert lay.proj_cols == rk + sum(rv)
    col = 0
    for li, s in enumerate(ref["segs"]):
        seg = lay.seg[li]
        assert seg.rank == s["rank"] and seg.col == col
        col += s["rank"]
        if fmt == "mixed":
            assert (seg.n8, seg.n4, seg.g8, seg.g4, seg.nb4) == (s["n8"], s["n4"], s["g8"], s["g4"], s["nb4"])
            assert (seg.off_i8, seg.off_i4, seg.off_sc) == (s["i8"], s["i4"], s["sc"])
            assert seg.off_plain == -1
        elif fmt == "had43":
            # the 4-bit outlier block and the 3-bit inlier block in the int8/int4 fields
            assert (seg.n8, seg.n4, seg.g8, seg.g4) == (s["n_hi"], s["n_lo"], s["g_hi"], s["g_lo"])
            assert (seg.pitch, seg.nb4) == (s["nb_hi"], s["nb_lo"])
            assert (seg.off_i8, seg.off_i4, seg.off_sc) == (s["hi"], s["lo"], s["sc"])
            assert seg.off_plain == -1
        else:
            assert seg.off_plain == s["plain"] and seg.pitch == s["pitch"]


def test_alloc_sizes(lib):
    rv = [8, 48, 37, 17, 32, 29, 40, 45]
    lay = api.layout_init(api.make_config(32, 8, 128, 4096, 256, rv, "mixed", 500000.0))
    s = api.alloc(lay, 1000, 4, 16, 8192)
    assert s.cache_bytes == 1000 * lay.page_bytes
    # RoPE table: 128 in-tile offsets + one row per 128-token tile, d/2 (cos, sin) pairs each
    assert s.rope_table_bytes == (128 + 8) * 64 * 8
    # partial records: 2 + max rank floats, rounded up to 4
    assert s.decode_workspace_bytes == 4 * 32 * 8 * 52 * 4
    assert s.append_workspace_bytes >= 8192 * lay.proj_cols * 4


def test_absorbed_sizes(lib):
    rv = [8, 48, 37, 17, 32, 29, 40, 45]
    lay = api.layout_init(api.make_config(32, 8, 128, 4096, 256, rv, "mixed", 500000.0))
    rows, nbytes = api.absorbed_sizes(lay, 3, 4096)
    # four query heads per KV head, each with the r_g rows of its group
    assert rows == 4 * sum(rv)
    # the latent outputs of every (sequence, head), then at least one split of [3][4096] partials
    assert nbytes >= 3 * rows * 4 + 3 * 4096 * 4
    with pytest.raises(L.StarkvError):
        api.absorbed_sizes(lay, 3, 0)


def test_absorbed_combine_rejects_small_scratch_before_touching_the_device(lib):
    lay = api.layout_init(api.make_config(32, 8, 128, 4096, 256, [32] * 8, "mixed", 500000.0))
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check comes first
    st = lib.starkv_decode_combine_absorbed(ctypes.byref(lay), fake, 2, 4, fake, 64, fake, 1 << 30,
                                            fake, 16, fake, None)
    assert st == L.ERR_WORKSPACE


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, L.ERR_UNSUPPORTED),
    ("n_kv_heads", 0, L.ERR_INVALID_ARG),
    ("n_q_heads", 12, L.ERR_INVALID_ARG),
    ("key_rank", 100, L.ERR_INVALID_ARG),
    ("page_tokens", 32, L.ERR_UNSUPPORTED),
    ("fmt", 7, L.ERR_INVALID_ARG),
    ("rope_theta", float("nan"), L.ERR_INVALID_ARG),
])
def test_layout_rejects(lib, field, value, status):
    cfg = api.make_config(32, 8, 128, 4096, 256, [32] * 8, "mixed", 500000.0)
    setattr(cfg, field, value)
    lay = L.Layout()
    assert lib.starkv_layout_init(ctypes.byref(cfg), ctypes.byref(lay)) == status
    assert lib.starkv_last_error()


def test_value_rank_out_of_range_rejected(lib):
    cfg = api.make_config(4, 4, 64, 256, 64, [40, 65, 3, 3], "f32", 10000.0)
    lay = L.Layout()
    assert lib.starkv_layout_init(ctypes.byref(cfg), ctypes.byref(lay)) == L.ERR_INVALID_ARG


def test_tampered_layout_rejected(lib):
    lay = api.layout_init(api.make_config(4, 4, 64, 256, 64, [40, 44, 47, 50], "f32", 10000.0))
    lay.page_bytes += 16
    s = L.Sizes()
    assert lib.starkv_alloc(ctypes.byref(lay), 4, 1, 4, 0, ctypes.byref(s)) == L.ERR_INVALID_ARG


def test_store_rejects_token_counts_past_32_bit_warp_numbering(lib):
    # key rank 2048 int8/int4: 64 chunks per token for the key alone, so ~33.5 M tokens would
    # number warps past 2^31; refused before any device call (the pointers are never used)
    lay = api.layout_init(api.make_config(8, 1, 128, 4096, 2048, [128], "mixed", 10000.0))
    fake = ctypes.c_void_p(1 << 20)
    st = lib.starkv_quant_pack(ctypes.byref(lay), fake, 40_000_000, fake, fake, fake, 1, 1, fake,
                               1, fake, None)
    assert st == L.ERR_INVALID_ARG and b"split the tokens" in lib.starkv_last_error()
    st = lib.starkv_dequant(ctypes.byref(lay), fake, 1, fake, fake, 40_000_000, fake, 1, 1, fake,
                            fake, None)
    assert st == L.ERR_INVALID_ARG


def test_had43_decode_plans_like_int8_int4(lib):
    """The pages' own format decodes through the int8/int4 machinery: the same key modes
    (resident operand at rank <= 256, staged codes above), CTA pairs and chunking."""
    for rk, rv, batch, pages, mode, cg in [(256, [32] * 8, 32, 512, 1, 2),
                                           (1024, [32] * 32, 16, 256, 2, 1)]:
        hkv = len(rv)
        lay_m = api.layout_init(api.make_config(32, hkv, 128, 4096, rk, rv, "mixed", 1e4))
        lay_h = api.layout_init(api.make_config(32, hkv, 128, 4096, rk, rv, "had43", 1e4))
        pm = api.decode_plan(lay_m, batch, pages)
        ph = api.decode_plan(lay_h, batch, pages)
        assert (ph.key_mode, ph.cta_group) == (mode, cg)
        assert (ph.chunk_cols, ph.n_chunks, ph.n_ranges, ph.grid) == \
            (pm.chunk_cols, pm.n_chunks, pm.n_ranges, pm.grid)
        assert 120 * 1024 <= ph.smem_bytes <= 232448


def test_alloc_rejects_a_cache_size_past_size_t(lib):
    lay = api.layout_init(api.make_config(32, 8, 128, 4096, 256, [32] * 8, "mixed", 500000.0))
    s = L.Sizes()
    huge = (1 << 64) // lay.page_bytes + 1
    assert huge < (1 << 63)
    assert lib.starkv_alloc(ctypes.byref(lay), huge, 1, 4, 0, ctypes.byref(s)) == L.ERR_INVALID_ARG
    assert lib.starkv_alloc(ctypes.byref(lay), huge - 2, 1, 4, 0, ctypes.byref(s)) == L.OK


def test_decode_workspace_size_is_checked_for_overflow(lib):
    """batch * n_q_heads * tiles * record floats * 4 must not wrap: a wrapped size could pass
    both the caller-workspace check and the no-allocation entry point's scratch check."""
    lay = api.layout_init(api.make_config(512, 64, 128, 4096, 256, [128] * 64, "mixed", 1e4))
    s = L.Sizes()
    # 2^31 - 1 sequences x 512 heads: above the combine's grid limit (and past 2^64 bytes)
    assert lib.starkv_alloc(ctypes.byref(lay), 1, (1 << 31) - 1, 1 << 24, 0,
                            ctypes.byref(s)) == L.ERR_INVALID_ARG
    assert b"2^31" in lib.starkv_last_error()
    # the largest batch the grid allows: the size is exact (below 2^64, no wrap)
    b = ((1 << 31) - 1) // 512
    assert lib.starkv_alloc(ctypes.byref(lay), 1, b, 1 << 24, 0, ctypes.byref(s)) == L.OK
    assert s.decode_workspace_bytes == b * 512 * (1 << 23) * 132 * 4
    # and the no-allocation entry point refuses the oversized batch before touching a device
    rc = lib.starkv_decode_attention_noalloc(
        ctypes.byref(lay), None, None, 1, None, 1 << 24, None, (1 << 31) - 1, None, None, None,
        0, None, None, None, None)
    assert rc == L.ERR_INVALID_ARG
    # an ordinary size is exact
    assert lib.starkv_alloc(ctypes.byref(lay), 1, 3, 10, 0, ctypes.byref(s)) == L.OK
    assert s.decode_workspace_bytes == 3 * 512 * 5 * (4 * ((2 + 128 + 3) // 4)) * 4


def test_binding_refuses_host_tensors_instead_of_passing_host_pointers(lib):
    # every device argument goes through the same marshalling; a CPU tensor never reaches the
    # library as if it were device memory
    lay = api.layout_init(api.make_config(4, 4, 64, 256, 64, [40, 44, 47, 50], "f32", 10000.0))
    cpu = torch.zeros(16, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.quant_pack(lay, torch.zeros(1, lay.proj_cols), cpu[:1], cpu[:1], cpu[:1].reshape(1, 1),
                       torch.zeros(lay.page_bytes, dtype=torch.uint8), cpu[:1])
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.decode_combine(lay, cpu[:1], 1, torch.zeros(lay.value_rank_total, 64), torch.zeros(64),
                           torch.zeros(4, 64))


def test_binding_checks_dtype_and_size_before_the_library_sees_a_pointer(lib):
    # the library sees only pointers: a tensor of the wrong dtype or too few elements is
    # refused in the binding (checked before the device check, so this runs on the CPU)
    lay = api.layout_init(api.make_config(4, 4, 64, 256, 64, [40, 44, 47, 50], "f32", 10000.0))
    i32 = torch.zeros(4, dtype=torch.int32)
    table = torch.zeros(2, 4, dtype=torch.int32)
    cache = torch.zeros(lay.page_bytes, dtype=torch.uint8)
    with pytest.raises(ValueError, match="latents: expected dtype"):
        api.quant_pack(lay, torch.zeros(2, lay.proj_cols, dtype=torch.float64), i32, i32, table,
                       cache, i32)
    with pytest.raises(ValueError, match="tok_pos: 1 elements"):
        api.quant_pack(lay, torch.zeros(2, lay.proj_cols), i32, i32[:1], table, cache, i32)
    with pytest.raises(ValueError, match="block_table: expected 2 dimensions"):
        api.quant_pack(lay, torch.zeros(2, lay.proj_cols), i32, i32, table.reshape(-1), cache, i32)
    with pytest.raises(ValueError, match="x: expected dtype"):
        api.append(lay, torch.zeros(2, 256, dtype=torch.bfloat16),
                   torch.zeros(lay.proj_cols, 256), i32, i32, table, cache, cache, i32)
    H, d = 4, 64
    q = torch.zeros(2, H, d)
    Bk_t = torch.zeros(4 * d, 64)
    Bv = torch.zeros(lay.value_rank_total, d)
    out = torch.zeros(2, H, d)
    seq_lens = i32[:2]
    with pytest.raises(ValueError, match="q: 256 elements"):
        api.decode_attention(lay, q[:1], cache, table, seq_lens, Bk_t, Bv, cache, out, cache, i32)
    with pytest.raises(ValueError, match="Bk_t: expected dtype"):
        api.decode_attention(lay, q, cache, table, seq_lens, Bk_t.half(), Bv, cache, out, cache, i32)
    with pytest.raises(ValueError, match="out: "):
        api.decode_attention(lay, q, cache, table, seq_lens, Bk_t, Bv, cache, out[:1], cache, i32)
    with pytest.raises(ValueError, match="block_table: 1 rows for 2 sequences"):
        api.decode_partials(lay, q, cache, table[:1], seq_lens, Bk_t, cache, cache, i32)
    # well-formed arguments pass the checks and stop at the device check
    with pytest.raises(ValueError, match="CUDA tensor"):
        api.decode_attention(lay, q, cache, table, seq_lens, Bk_t, Bv, cache, out, cache, i32)


# ---- the hybrid assignment (keys head-wise, values joint)
HYBRID_CASES = [
    ("mixed", 32, 8, 128, 4096, [32, 16, 48, 32, 32, 16, 48, 32], 256),
    ("mixed", 8, 2, 64, 256, [64, 16], 48),
    ("bf16", 32, 32, 128, 4096, [16 * (1 + g % 8) for g in range(32)], 1024),
    ("had43", 32, 8, 128, 4096, [32] * 8, 256),
    ("f32", 4, 4, 64, 256, [16, 32, 48, 64], 128),
]


@pytest.mark.parametrize("fmt,H,Hkv,d,dm,kr,rv", HYBRID_CASES)
def test_hybrid_layout_matches_oracle(lib, fmt, H, Hkv, d, dm, kr, rv):
    lay = api.hybrid_layout_init(api.make_hybrid_config(H, Hkv, d, dm, kr, rv, fmt, 500000.0))
    ref = O.hybrid_page_layout(fmt, kr, rv, page_tokens=64)
    assert lay.assignment == L.ASSIGN_HYBRID
    assert lay.page_bytes == ref["page_bytes"] and lay.token_bytes == ref["token_bytes"]
    assert lay.n_latents == Hkv + 1
    assert lay.proj_cols == sum(kr) + rv
    assert lay.value_rank_total == rv and lay.value_rank_max == rv
    assert lay.cfg.key_rank == 0 and all(lay.cfg.value_rank[g] == 0 for g in range(L.MAX_KV_HEADS))
    assert (lay.cfg.n_q_heads, lay.cfg.n_kv_heads, lay.cfg.head_dim) == (H, Hkv, d)
    assert [lay.hybrid.key_rank[g] for g in range(Hkv)] == kr and lay.hybrid.value_rank == rv
    col = 0
    for li, s in enumerate(ref["segs"]):
        seg = lay.seg[li]
        assert seg.rank == (kr[li] if li < Hkv else rv) == s["rank"] and seg.col == col
        col += s["rank"]
        if fmt == "mixed":
            assert (seg.off_i8, seg.off_i4, seg.off_sc) == (s["i8"], s["i4"], s["sc"])
            assert (seg.n8, seg.nb4, seg.g8, seg.g4) == (s["n8"], s["nb4"], s["g8"], s["g4"])
        elif fmt == "had43":
            assert (seg.off_i8, seg.off_i4, seg.off_sc) == (s["hi"], s["lo"], s["sc"])
        else:
            assert seg.off_plain == s["plain"] and seg.pitch == s["pitch"]


@pytest.mark.parametrize("field,value", [("value_rank", 24), ("value_rank", 0), ("value_rank", 4096),
                                         ("head_dim", 96), ("page_tokens", 32)])
def test_hybrid_layout_rejects(lib, field, value):
    cfg = api.make_hybrid_config(32, 8, 128, 4096, [32] * 8, 256, "mixed", 10000.0)
    setattr(cfg, field, value)
    lay = L.Layout()
    assert lib.starkv_hybrid_layout_init(ctypes.byref(cfg), ctypes.byref(lay)) != L.OK


@pytest.mark.parametrize("rank", [0, 8, 20, 144])
def test_hybrid_layout_rejects_key_ranks_off_the_16_grid(lib, rank):
    cfg = api.make_hybrid_config(32, 8, 128, 4096, [32] * 7 + [rank], 256, "mixed", 10000.0)
    lay = L.Layout()
    assert lib.starkv_hybrid_layout_init(ctypes.byref(cfg), ctypes.byref(lay)) == L.ERR_INVALID_ARG


def test_hybrid_workspace_holds_one_record_per_page_range_and_head(lib):
    lay = api.hybrid_layout_init(api.make_hybrid_config(32, 8, 128, 4096, [32] * 8, 256, "mixed",
                                                        500000.0))
    for batch, max_pages in [(32, 512), (1, 2048), (3, 17), (1000, 4)]:
        s = api.alloc(lay, 10, batch, max_pages, 0)
        want = -(-1184 // batch)
        want = max(1, min(want, max_pages))
        pps = -(-max_pages // want)
        nsplit = -(-max_pages // pps)
        assert nsplit * pps >= max_pages and (nsplit - 1) * pps < max_pages
        rec = (2 + 256 + 3) // 4 * 4
        assert s.decode_workspace_bytes == batch * 32 * nsplit * rec * 4


def test_joint_key_calls_refuse_a_hybrid_layout_before_touching_the_device(lib):
    lay = api.hybrid_layout_init(api.make_hybrid_config(32, 8, 128, 4096, [32] * 8, 256, "mixed",
                                                        500000.0))
    plan = L.DecodePlan()
    assert lib.starkv_decode_plan_query(ctypes.byref(lay), 4, 16, None, 148, 232448,
                                        ctypes.byref(plan)) == L.ERR_UNSUPPORTED
    rows, scratch = ctypes.c_int64(0), ctypes.c_size_t(0)
    assert lib.starkv_absorbed_sizes(ctypes.byref(lay), 4, 4096, ctypes.byref(rows),
                                     ctypes.byref(scratch)) == L.ERR_UNSUPPORTED
    # the decode call itself, with host dummies that it must not dereference
    assert lib.starkv_decode_attention(ctypes.byref(lay), 16, 16, 4, 16, 16, 16, 1, 16, 16, 16,
                                       1 << 20, 16, 16, 1 << 30, None, 16, None) == L.ERR_UNSUPPORTED


def test_hybrid_decode_refuses_before_touching_the_device(lib):
    joint = api.layout_init(api.make_config(32, 8, 128, 4096, 256, [32] * 8, "mixed", 500000.0))
    args = (16, 16, 4, 16, 16, 16, 1, 16, 16, 16, 1 << 20, 16, 16, 1 << 30, 16, None)
    assert lib.starkv_hybrid_decode(ctypes.byref(joint), *args) == L.ERR_INVALID_ARG
    bf16 = api.hybrid_layout_init(api.make_hybrid_config(32, 8, 128, 4096, [32] * 8, 256, "bf16",
                                                         500000.0))
    assert lib.starkv_hybrid_decode(ctypes.byref(bf16), *args) == L.ERR_UNSUPPORTED
    wide = api.hybrid_layout_init(api.make_hybrid_config(64, 32, 128, 4096, [32] * 32, 256,
                                                         "mixed", 500000.0))
    assert lib.starkv_hybrid_decode(ctypes.byref(wide), *args) == L.ERR_UNSUPPORTED  # H_kv > 16
    big = api.hybrid_layout_init(api.make_hybrid_config(64, 8, 128, 4096, [32] * 8, 512, "mixed",
                                                        500000.0))
    assert lib.starkv_hybrid_decode(ctypes.byref(big), *args) == L.ERR_UNSUPPORTED  # 4 x 8 tiles


def test_tampered_hybrid_layout_rejected(lib):
    lay = api.hybrid_layout_init(api.make_hybrid_config(32, 8, 128, 4096, [32] * 8, 256, "mixed",
                                                        500000.0))
    lay.seg[8].off_sc += 16
    s = L.Sizes()
    assert lib.starkv_alloc(ctypes.byref(lay), 10, 1, 4, 0, ctypes.byref(s)) == L.ERR_INVALID_ARG
    lay2 = api.hybrid_layout_init(api.make_hybrid_config(32, 8, 128, 4096, [32] * 8, 256, "mixed",
                                                         500000.0))
    lay2.assignment = 7
    assert lib.starkv_alloc(ctypes.byref(lay2), 10, 1, 4, 0, ctypes.byref(s)) == L.ERR_INVALID_ARG
