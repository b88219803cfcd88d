"""The allocation-free decode entry point (built-in scratch instead of a caller workspace),
for callers that cannot allocate device memory.  Its output must match the workspace entry
point's, within the decode tolerance, on two calls in a row (the scratch keeps the previous
call's contents).  Collected last, so a failure here leaves every other test already run."""
import ctypes

import numpy as np
import pytest
import torch

from rank_quantized_kv_decode_b200 import _lib as L
from rank_quantized_kv_decode_b200 import api
from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import tolerance_check


@pytest.mark.gpu
@pytest.mark.parametrize("index,ov,lens", [
    (4, dict(batch=3, context=1000), [1000, 1, 333]),
    (2, dict(batch=2, context=640), [640, 65]),
])
def test_noalloc_matches_workspace_entry_point(index, ov, lens):
    wl = W.build(index, seq_lens=lens, **ov)
    W.decode(wl)
    torch.cuda.synchronize()
    assert wl.lc.status.item() == 0
    want = wl.out.cpu().numpy().copy()
    out = torch.empty_like(wl.out)
    for call in range(2):
        out.fill_(float("nan"))
        api.decode_attention_noalloc(wl.lay, wl.q, wl.lc.cache, wl.block_table, wl.seq_lens,
                                     wl.Bk_t, wl.Bv, wl.lc.rope, out, wl.lc.status)
        torch.cuda.synchronize()
        assert wl.lc.status.item() == 0
        got = out.cpu().numpy()
        for b in range(len(lens)):
            tolerance_check(got[b], want[b])


def test_noalloc_rejects_calls_above_its_scratch():
    # batch 64 x 32 heads x 256 tiles x 36 floats (75 MiB) is above the 16 MiB scratch: refused
    # before anything touches a device
    from rank_quantized_kv_decode_b200 import build
    build.build()
    lay = api.layout_init(api.make_config(32, 8, 128, 4096, 256, [32] * 8, "mixed", 500000.0))
    lib = L.load()
    rc = lib.starkv_decode_attention_noalloc(
        ctypes.byref(lay), None, None, 1, None, 512, None, 64, None, None, None, 0, None, None,
        None, None)
    assert rc == L.ERR_WORKSPACE
    assert b"16777216" in lib.starkv_last_error()
