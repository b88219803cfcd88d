"""Decode parity at the full workload sizes, in the launch configuration the benchmark uses
(default grid and work split), on sampled (sequence, query head) outputs the oracle computes
one by one."""
import numpy as np
import pytest
import torch

from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import ref_for, tolerance_check

pytestmark = pytest.mark.gpu

# workload -> [(sequence, query heads)]
SAMPLES = {
    1: [(0, [0, 1, 2, 3])],
    2: [(0, [0, 31]), (5, [7, 18])],
    3: [(9, [2, 30])],
    4: [(0, [0, 5]), (17, [13, 31])],
    5: [(0, [0, 9, 31])],
}


@pytest.mark.parametrize("index", [1, 2, 3, 4, 5])
def test_full_size_sampled(index):
    wl = W.build(index)
    W.decode(wl)
    torch.cuda.synchronize()
    assert wl.lc.status.item() == 0
    out = wl.out.cpu().numpy()
    ref = ref_for(index, index in (1, 5))
    L = wl.w["context"]
    for b, heads in SAMPLES[index]:
        want = ref.expected(b, L, heads=heads)
        tolerance_check(out[b, heads], want)
    # every output finite, and the sequences not sampled are not all zero
    assert np.isfinite(out).all()
    assert np.abs(out).sum(axis=(1, 2)).min() > 0
    del wl
    torch.cuda.empty_cache()
