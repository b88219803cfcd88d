"""Failure detection without a GPU fault: a bounded in-kernel wait that nothing completes
runs out, reports STARKV_DEV_TIMEOUT, releases its resources, and the context keeps working."""
import time

import pytest
import torch

from rank_quantized_kv_decode_b200 import _lib as L
from rank_quantized_kv_decode_b200 import api
from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import ref_for, tolerance_check

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    api.diag_bounded_wait(50, status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert status.item() & L.DEV_TIMEOUT
    assert 0.04 < dt < 5.0
    # the same process goes on decoding correctly
    wl = W.build(1, batch=1)
    W.decode(wl)
    torch.cuda.synchronize()
    assert wl.lc.status.item() == 0
    ref = ref_for(1, True, batch=1)
    tolerance_check(wl.out[0].cpu().numpy(), ref.expected(0, 256))


def test_bad_timeout_rejected():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(L.StarkvError):
        api.diag_bounded_wait(0, status)
