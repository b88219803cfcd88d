"""The allocation-free decode entry point (built-in scratch instead of a caller workspace),
for callers that cannot allocate device memory.  Its output must match the workspace entry
point's, within the decode tolerance, on calls in a row: the scratch keeps the previous
call's partial records, and each call must write every record it reads.  Between two calls of
one workload a call of another (other lengths, batch and values) leaves different records
behind, so a record the split kernel skipped would show up as a wrong output.  Collected
last, so a failure here leaves every other test already run."""
import ctypes

import pytest
import torch

from rank_quantized_kv_decode_b200 import _lib as L
from rank_quantized_kv_decode_b200 import api
from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import tolerance_check

CASES = [
    (4, dict(batch=3, context=1000), [1000, 1, 333]),
    (2, dict(batch=2, context=640), [640, 65]),
]
# a different workload run between the calls of the one under test
OTHER = {
    4: (4, dict(batch=5, context=1500, shuffle_pages=False), [700, 1500, 64, 1, 1281]),
    2: (3, dict(batch=3, context=900), [900, 129, 17]),
}


def _reference(wl):
    """Output of the workspace entry point (caller-allocated workspace)."""
    W.decode(wl)
    torch.cuda.synchronize()
    assert wl.lc.status.item() == 0
    return wl.out.cpu().numpy().copy()


def _noalloc(wl, out):
    out.fill_(float("nan"))
    api.decode_attention_noalloc(wl.lay, wl.q, wl.lc.cache, wl.block_table, wl.seq_lens,
                                 wl.Bk_t, wl.Bv, wl.lc.rope, out, wl.lc.status)
    torch.cuda.synchronize()
    assert wl.lc.status.item() == 0
    return out.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("index,ov,lens", CASES)
def test_noalloc_matches_workspace_entry_point(index, ov, lens):
    wl = W.build(index, seq_lens=lens, **ov)
    want = _reference(wl)
    oi, oov, olens = OTHER[index]
    other = W.build(oi, seq_lens=olens, **oov)
    other_want = _reference(other)
    out = torch.empty_like(wl.out)
    other_out = torch.empty_like(other.out)
    for call in range(2):
        got = _noalloc(wl, out)
        for b in range(len(lens)):
            tolerance_check(got[b], want[b])
        # the other workload's records now replace part of this one's in the scratch
        got_o = _noalloc(other, other_out)
        for b in range(len(olens)):
            tolerance_check(got_o[b], other_want[b])


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
