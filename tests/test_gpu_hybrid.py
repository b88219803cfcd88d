"""GPU parity of decode attention with the hybrid assignment (keys head-wise, values joint;
STAR-KV technical summary, Methodology §2) against the fp64 oracle's decode_attention_hybrid:
ragged lengths (an empty sequence, a single token, a page boundary, tails), page ranges of
several pages, d = 64 and G = 1 / 8, a sharp softmax, the full workload-size cache sampled,
and a bad block-table entry."""
import numpy as np
import pytest
import torch

from rank_quantized_kv_decode_b200 import _lib as L
from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import HybridRef, tolerance_check

pytestmark = pytest.mark.gpu

CASES = {
    # workload shape (GQA 32/8, d 128), reduced context: one page per range
    "gqa": (dict(batch=4, context=1000), [1000, 0, 333, 64]),
    # enough sequences that a range holds two pages
    "ranges": (dict(batch=20, context=4096), [4096, 4000, 130, 0, 1] + [4096 - 97 * i for i in range(15)]),
    # d 64, one query head per KV head, ranks up to head_dim, value rank 128
    "d64": (dict(batch=2, context=700, n_q_heads=4, n_kv_heads=4, head_dim=64,
                 key_ranks=(16, 32, 48, 64), value_rank=128), [700, 129]),
    # eight query heads per KV head
    "g8": (dict(batch=2, context=520, n_q_heads=16, n_kv_heads=2, key_ranks=(32, 64), value_rank=64),
           [520, 65]),
}

_built = {}


def built(name):
    if name not in _built:
        ov, lens = CASES[name]
        _built[name] = (W.build_hybrid(seq_lens=lens, **ov), HybridRef(**ov))
    return _built[name]


def check(name, seqs=None, q=None):
    hw, ref = built(name)
    lens = CASES[name][1]
    out = hw.out.cpu().numpy()
    assert hw.lc.status.item() == 0
    for b in (range(len(lens)) if seqs is None else seqs):
        tolerance_check(out[b], ref.expected(b, lens[b], q=q))


@pytest.mark.parametrize("name", ["gqa", "d64", "g8"])
def test_hybrid_decode_matches_oracle(name):
    hw, _ = built(name)
    W.decode_hybrid(hw)
    torch.cuda.synchronize()
    check(name)


def test_page_ranges_of_several_pages():
    hw, _ = built("ranges")
    assert hw.lay.n_latents == 9
    W.decode_hybrid(hw)
    torch.cuda.synchronize()
    check("ranges", seqs=[0, 1, 2, 3, 4, 9, 19])


def test_repeat_is_bit_identical():
    hw, _ = built("gqa")
    W.decode_hybrid(hw)
    torch.cuda.synchronize()
    first = hw.out.clone()
    W.decode_hybrid(hw)
    torch.cuda.synchronize()
    assert torch.equal(first, hw.out)


@pytest.mark.parametrize("name,scale", [("gqa", 8.0), ("gqa", 32.0), ("g8", 8.0)])
def test_sharp_softmax(name, scale):
    hw, ref = built(name)
    q0 = hw.q.clone()
    try:
        # exact in bf16: a power-of-two scale of bf16 values
        hw.q.mul_(scale)
        W.decode_hybrid(hw)
        torch.cuda.synchronize()
        check(name, q=ref.queries() * scale)
    finally:
        hw.q.copy_(q0)


def test_bad_block_table_entry_is_flagged_and_skipped():
    hw, _ = built("gqa")
    bt0 = hw.block_table.clone()
    try:
        hw.block_table[2, 1] = -5
        hw.lc.status.zero_()
        W.decode_hybrid(hw)
        torch.cuda.synchronize()
        assert hw.lc.status.item() & L.DEV_BOUNDS
        assert torch.isfinite(hw.out).all()
    finally:
        hw.block_table.copy_(bt0)
        hw.lc.status.zero_()


def test_full_size_cache_sampled():
    # 32 sequences x 32768 tokens (the workload's cache, 386 MB), two sequences sampled
    hw = W.build_hybrid()
    W.decode_hybrid(hw)
    torch.cuda.synchronize()
    assert hw.lc.status.item() == 0
    ref = HybridRef()
    out = hw.out.cpu().numpy()
    L_ = hw.w["context"]
    for b, heads in [(0, [0, 13, 31]), (31, [5, 22])]:
        tolerance_check(out[b, heads], ref.expected(b, L_, heads=heads))
    assert np.isfinite(out).all()
