"""GPU parity of decode attention read from the compressed cache, against the fp64 oracle:
every workload at reduced batch/context with ragged lengths, launch-shape invariance, a
sharp softmax, empty sequences and bad block-table entries."""
import numpy as np
import pytest
import torch

from rank_quantized_kv_decode_b200 import _lib as L
from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import ref_for, tolerance_check

pytestmark = pytest.mark.gpu

# (workload, overrides, per-sequence lengths): several tiles and a ragged tail per case
CASES = {
    1: (dict(batch=3), [256, 1, 130]),
    2: (dict(batch=2, context=640), [640, 65]),
    3: (dict(batch=2, context=520), [129, 520]),
    4: (dict(batch=3, context=1000), [1000, 1, 333]),
    5: (dict(batch=1, context=1500, prefill_tokens=512), [1500]),
}

_built = {}


def built(index):
    if index not in _built:
        ov, lens = CASES[index]
        _built[index] = W.build(index, seq_lens=lens, **ov)
    return _built[index]


def need_down(index):
    w = CASES[index][0]
    return index in (1, 5)


def check_all(index, wl, q=None):
    ov, lens = CASES[index]
    ref = ref_for(index, need_down(index), **ov)
    out = wl.out.cpu().numpy()
    assert wl.lc.status.item() == 0
    for b, Lb in enumerate(lens):
        want = ref.expected(b, Lb, q=q)
        tolerance_check(out[b], want)


@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
def test_decode_matches_oracle(index):
    wl = built(index)
    W.decode(wl)
    torch.cuda.synchronize()
    check_all(index, wl)


@pytest.mark.parametrize("index", [2, 4])
@pytest.mark.parametrize("cta_group", [1, 2])
@pytest.mark.parametrize("max_ctas,n_ranges", [(2, 1), (8, 2), (0, 4), (6, 0)])
def test_launch_shape_does_not_change_result(index, cta_group, max_ctas, n_ranges):
    wl = built(index)
    W.decode(wl, cta_group=cta_group)
    torch.cuda.synchronize()
    base = wl.out.clone()
    W.decode(wl, cta_group=cta_group, max_ctas=max_ctas, n_ranges=n_ranges)
    torch.cuda.synchronize()
    assert wl.lc.status.item() == 0
    # each tile's partial is computed the same way whatever the grid: bit-identical
    assert torch.equal(base, wl.out)


@pytest.mark.parametrize("index", [2, 3, 4, 5])
@pytest.mark.parametrize("cta_group", [1, 2])
def test_single_and_paired_ctas_match_oracle(index, cta_group):
    wl = built(index)
    W.decode(wl, cta_group=cta_group)
    torch.cuda.synchronize()
    check_all(index, wl)


@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("scale", [8.0, 32.0])
def test_sharp_softmax(index, scale):
    """At the stated spectra the softmax is nearly uniform; scaling the query by 8 or 32 (a
    power of two: exact in bf16 and fp32) makes a few tokens dominate, so an error in a score
    shows in the output instead of averaging out."""
    wl = built(index)
    q0 = wl.q.clone()
    try:
        wl.q.mul_(scale)
        W.decode(wl)
        torch.cuda.synchronize()
        qs = (q0.float() * scale).cpu().numpy()
        check_all(index, wl, q=qs)
    finally:
        wl.q.copy_(q0)


def test_empty_sequence_gives_zeros():
    wl = built(4)
    lens0 = wl.seq_lens.clone()
    try:
        wl.seq_lens[1] = 0
        W.decode(wl)
        torch.cuda.synchronize()
        assert wl.lc.status.item() == 0
        assert torch.count_nonzero(wl.out[1]) == 0
        ref = ref_for(4, False, **CASES[4][0])
        tolerance_check(wl.out[0].cpu().numpy(), ref.expected(0, CASES[4][1][0]))
    finally:
        wl.seq_lens.copy_(lens0)


def test_bad_block_table_entry_is_flagged():
    wl = built(4)
    saved = wl.block_table.clone()
    try:
        wl.block_table[0, 3] = wl.lc.num_pages + 5
        wl.block_table[2, 0] = -1
        wl.lc.status.zero_()
        W.decode(wl)
        torch.cuda.synchronize()
        assert wl.lc.status.item() & L.DEV_BOUNDS
        assert torch.isfinite(wl.out).all()
    finally:
        wl.block_table.copy_(saved)
        wl.lc.status.zero_()


def test_key_codes_too_large_to_stage_read_from_global_memory():
    """int8/int4 keys of rank 2048: a 128-token tile's codes (2 x 90 KB) do not fit in shared
    memory next to the ring, so the dequantisers read them from the pages in global memory;
    ranks up to ~1024 stage them (the other cases of this file)."""
    from oracle.workloads import Ref
    from rank_quantized_kv_decode_b200 import synth

    ov = dict(key_rank=2048, batch=1, context=200)
    wl = W.build(3, seq_lens=[200], **ov)
    W.decode(wl)
    torch.cuda.synchronize()
    assert wl.lc.status.item() == 0
    ref = Ref(synth.workload(3, **ov), False)
    tolerance_check(wl.out[0].cpu().numpy(), ref.expected(0, 200))
