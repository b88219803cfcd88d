"""GPU parity of the per-tile partial records of the split step (starkv_decode_partials)
against the oracle's tile_partials: for every (sequence, query head, 128-token tile) inside
the sequence, the tile's largest score m (log2 units), its weight sum l and its latent sum a.
These records are the only direct view of the scores and the softmax: an error in q.k that
the final output would average away shows here tile by tile."""
import numpy as np
import pytest
import torch

import oracle.starkv_oracle as O
from rank_quantized_kv_decode_b200 import api
from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import ref_for

pytestmark = pytest.mark.gpu

# (workload, overrides, per-sequence lengths): several tiles and a ragged tail
CASES = {
    1: (dict(batch=2), [256, 130]),
    2: (dict(batch=2, context=640), [640, 65]),
    3: (dict(batch=2, context=520), [129, 520]),
    4: (dict(batch=2, context=1000), [1000, 333]),
}

# Bars per record.  The kernel's scores carry the fp32 SFU sine/cosine of the RoPE angles
# (~5e-5 rad at the angles here), fp32 accumulation and, for int8/int4 latents, the fp16
# rounding of the dequantised key operand (2^-12 relative per element); at the stated spectra
# the scores have a standard deviation below 1, so their absolute error stays below 1e-4 (in
# log2 units).  The bars are 20x that: m within 2e-3, l and a within 2e-3 relative.
M_TOL, REL_TOL = 2e-3, 2e-3


@pytest.mark.parametrize("index", [1, 2, 3, 4])
def test_partials_match_oracle_tile_by_tile(index):
    ov, lens = CASES[index]
    wl = W.build(index, seq_lens=lens, **ov)
    lay, lc = wl.lay, wl.lc
    lc.decode_ws.zero_()
    api.decode_partials(lay, wl.q, lc.cache, wl.block_table, wl.seq_lens, wl.Bk_t, lc.rope,
                        lc.decode_ws, lc.status)
    torch.cuda.synchronize()
    assert lc.status.item() == 0
    H = wl.w["n_q_heads"]
    T = (lc.max_pages * 64 + 127) // 128
    R = 4 * ((2 + lay.value_rank_max + 3) // 4)
    ws = lc.decode_ws.view(torch.float32)[:len(lens) * H * T * R].cpu().numpy()
    ws = ws.reshape(len(lens), H, T, R)
    ref = ref_for(index, index in (1, 5), **ov)
    q = ref.queries()
    G = H // wl.w["n_kv_heads"]
    n_checked = 0
    for b, Lb in enumerate(lens):
        Ck, Cv = ref.stored(ref.sequence_latents(b)[:Lb])
        parts = O.tile_partials(q[b], Ck, Cv, ref.Bk_s, wl.w["rope_theta"], wl.w["n_kv_heads"])
        for h in range(H):
            r = ref.ranks[h // G]
            assert len(parts[h]) == -(-Lb // 128)
            for t, (m, l, a) in enumerate(parts[h]):
                gm, gl, ga = ws[b, h, t, 0], ws[b, h, t, 1], ws[b, h, t, 2:2 + r]
                assert abs(gm - m) <= M_TOL, (b, h, t, gm, m)
                assert abs(gl - l) <= REL_TOL * l, (b, h, t, gl, l)
                assert np.linalg.norm(ga - a) <= REL_TOL * np.linalg.norm(a) + 1e-6, (b, h, t)
                n_checked += 1
    assert n_checked == H * sum(-(-Lb // 128) for Lb in lens)
