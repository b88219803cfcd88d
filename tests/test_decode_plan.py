"""Host-side checks of the decode launch planner (no GPU): ``starkv_decode_plan_query`` gives
the launch shape the decode calls choose, from the layout, batch and block-table width and a
device's SM count and opt-in shared memory.

* The five workloads get the kernel variants that were profiled on a B200: bf16 MHA on CTA
  pairs with the TMA ring, int8/int4 keys of rank 1024 on single CTAs with staged codes,
  int8/int4 GQA keys of rank 256 on CTA pairs with the resident operand.
* Over the configuration space that ``starkv_layout_init`` accepts, every plan fits the
  device's shared memory and its work-unit arithmetic is consistent; a configuration that
  cannot be planned is refused with STARKV_ERR_UNSUPPORTED (nothing else), and the bf16 and
  int8/int4 formats at head_dim 128 always plan.
"""
import pytest

from rank_quantized_kv_decode_b200 import _lib as L
from rank_quantized_kv_decode_b200 import api

SMEM = 232448  # opt-in shared memory per block of a B200
SMS = 148


@pytest.fixture(scope="module", autouse=True)
def lib():
    from rank_quantized_kv_decode_b200 import build
    build.build()
    return L.load()


def _layout(fmt, H, Hkv, d, rk, rv, dm=256):
    return api.layout_init(api.make_config(H, Hkv, d, dm, rk, rv, fmt, 10000.0))


RV32 = [16 + (g * 7) % 49 for g in range(32)]
RV8 = [8, 48, 37, 17, 32, 29, 40, 45]


@pytest.mark.parametrize("name,fmt,H,Hkv,rk,rv,batch,ctx,cg,mode", [
    ("llama2 bf16 b8 ctx4096", "bf16", 32, 32, 1024, RV32, 8, 4096, 2, 0),
    ("llama2 int8/int4 b16 ctx16384", "mixed", 32, 32, 1024, RV32, 16, 16384, 1, 2),
    ("llama3 int8/int4 b32 ctx32768", "mixed", 32, 8, 256, RV8, 32, 32768, 2, 1),
    ("llama3 int8/int4 b1 ctx131072", "mixed", 32, 8, 256, RV8, 1, 131072, 2, 1),
])
def test_workload_plans(name, fmt, H, Hkv, rk, rv, batch, ctx, cg, mode):
    lay = _layout(fmt, H, Hkv, 128, rk, rv, dm=4096)
    pl = api.decode_plan(lay, batch, ctx // 64)
    assert (pl.cta_group, pl.key_mode, pl.chunk_cols) == (cg, mode, 256)
    assert pl.n_chunks == Hkv * 128 // 256
    assert 120 * 1024 <= pl.smem_bytes <= SMEM
    assert pl.grid == SMS  # enough work units for a persistent CTA on every SM


def test_small_fp32_workload_plan():
    lay = _layout("f32", 4, 4, 64, 64, [40, 44, 47, 50])
    pl = api.decode_plan(lay, 1, 4)
    # fp32 latents: 128-column chunks (hi/lo tf32 copies), single CTAs, one unit per chunk
    assert (pl.cta_group, pl.key_mode, pl.chunk_cols, pl.n_chunks) == (1, 0, 128, 2)
    assert pl.work_units == 2 * 1 * pl.n_ranges and pl.grid == pl.work_units


def test_cta_group_request():
    lay = _layout("bf16", 32, 32, 128, 1024, RV32)
    assert api.decode_plan(lay, 8, 64, cta_group=1).cta_group == 1
    assert api.decode_plan(lay, 8, 64, cta_group=2).cta_group == 2
    f32 = _layout("f32", 4, 4, 64, 64, [40, 44, 47, 50])
    with pytest.raises(L.StarkvError) as e:
        api.decode_plan(f32, 1, 4, cta_group=2)
    assert e.value.status == 2


def test_max_ctas_caps_the_grid_in_whole_pairs():
    lay = _layout("bf16", 32, 32, 128, 1024, RV32)
    for cap in (1, 2, 3, 17, 64):
        pl = api.decode_plan(lay, 8, 64, max_ctas=cap)
        assert pl.grid <= max(cap, pl.cta_group) and pl.grid % pl.cta_group == 0


def _sweep():
    for fmt in ("f32", "bf16", "mixed"):
        for d in (64, 128):
            for G in (1, 2, 4, 8):
                for Hkv in (1, 3, 8, 33, 64):
                    for rk in (16, 256, 272, 1024, 2048):
                        for rvk in ("1", "d", "mix"):
                            yield fmt, d, G, Hkv, rk, rvk


def test_every_accepted_configuration_plans_or_is_refused():
    refused = []
    for fmt, d, G, Hkv, rk, rvk in _sweep():
        rv = ([1] * Hkv if rvk == "1" else [d] * Hkv if rvk == "d"
              else [1 + (g * 37) % d for g in range(Hkv)])
        lay = _layout(fmt, G * Hkv, Hkv, d, rk, rv)
        for batch, max_pages in ((1, 1), (64, 2048)):
            try:
                pl = api.decode_plan(lay, batch, max_pages)
            except L.StarkvError as e:
                assert e.status == 2, (fmt, d, G, Hkv, rk, rvk, str(e))
                refused.append((fmt, d, G, Hkv, rk, rvk))
                continue
            ncols = Hkv * d
            nc = (128 if fmt == "f32" else 256) if ncols >= 256 else ncols
            assert pl.chunk_cols == nc and pl.n_chunks == -(-ncols // nc)
            assert 1 <= pl.n_ranges <= pl.n_chunks
            tiles = -(-max_pages * 64 // 128)
            assert pl.work_units == -(-tiles // pl.cta_group) * batch * pl.n_ranges
            assert pl.grid == min(pl.work_units * pl.cta_group, SMS // pl.cta_group * pl.cta_group)
            assert 120 * 1024 <= pl.smem_bytes <= SMEM
            assert 2 <= pl.stages <= 6 and pl.value_buffers in (1, 2)
            if fmt == "mixed":
                assert pl.key_mode == 1 if rk <= 256 else pl.key_mode in (0, 2)
            else:
                assert pl.key_mode == 0
            if fmt == "f32":
                assert pl.cta_group == 1
    # the production formats at head_dim 128 always plan
    assert not [r for r in refused if r[0] != "f32" and r[1] == 128]
    assert not [r for r in refused if r[0] == "bf16"]
