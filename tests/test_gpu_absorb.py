"""GPU parity of the weight-absorbed output (STAR-KV technical summary, Methodology §2: the
value up-projection folded into the attention output projection) against the fp64 oracle:
y_b = sum_h a_b,h (B_v,g(h) W_o,h) for a seeded W_o, on the reduced GQA and MHA workloads,
with a ragged tail and an empty sequence."""
import numpy as np
import pytest
import torch

import oracle as O
from rank_quantized_kv_decode_b200 import api
from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import ref_for, tolerance_check

pytestmark = pytest.mark.gpu

CASES = {
    2: (dict(batch=2, context=640), [640, 65]),
    4: (dict(batch=3, context=1000), [1000, 1, 333]),
}


@pytest.mark.parametrize("index", [2, 4])
def test_absorbed_output_matches_oracle(index):
    ov, lens = CASES[index]
    wl = W.build(index, seq_lens=lens, **ov)
    ref = ref_for(index, False, **ov)
    w = wl.w
    H, d = w["n_q_heads"], w["head_dim"]
    d_out = w["d_model"]
    g = np.random.default_rng(1000 + index)
    Wo = (g.standard_normal((H * d, d_out)) / np.sqrt(H * d)).astype(np.float32)
    Wo_t = torch.from_numpy(Wo).cuda()
    rows, nbytes = api.absorbed_sizes(wl.lay, len(lens), d_out)
    assert rows == (H // w["n_kv_heads"]) * sum(wl.st.value_ranks)
    M = torch.empty(rows, d_out, dtype=torch.float32, device="cuda")
    api.absorb_output_weights(wl.lay, wl.Bv, Wo_t, M)
    scratch = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty(len(lens), d_out, dtype=torch.float32, device="cuda")
    lc = wl.lc
    api.decode_partials(wl.lay, wl.q, lc.cache, wl.block_table, wl.seq_lens, wl.Bk_t, lc.rope,
                        lc.decode_ws, lc.status)
    api.decode_combine_absorbed(wl.lay, wl.seq_lens, lc.max_pages, M, lc.decode_ws, scratch, out)
    torch.cuda.synchronize()
    assert lc.status.item() == 0
    M_ref = O.absorb_output_weights(ref.Bv_s, Wo.astype(np.float64), H)
    # the absorbed factors themselves (fp32 products of the stored B_v and W_o)
    got_M = M.cpu().numpy().astype(np.float64)
    want_M = np.concatenate(M_ref, axis=0)
    assert np.max(np.abs(got_M - want_M)) <= 1e-5 * max(np.max(np.abs(want_M)), 1e-30)
    q = ref.queries()
    for b, Lb in enumerate(lens):
        lat = ref.sequence_latents(b)[:Lb]
        Ck, Cv = ref.stored(lat)
        want = O.decode_attention_absorbed(q[b], Ck, Cv, ref.Bk_s, M_ref, w["rope_theta"],
                                           w["n_kv_heads"])
        tolerance_check(out[b].cpu().numpy(), want)


def test_absorbed_output_of_an_empty_sequence_is_zero():
    ov, lens = CASES[4]
    wl = W.build(4, seq_lens=lens, **ov)
    w = wl.w
    H, d, d_out = w["n_q_heads"], w["head_dim"], 256
    Wo_t = torch.randn(H * d, d_out, dtype=torch.float32, device="cuda")
    rows, nbytes = api.absorbed_sizes(wl.lay, len(lens), d_out)
    M = torch.empty(rows, d_out, dtype=torch.float32, device="cuda")
    api.absorb_output_weights(wl.lay, wl.Bv, Wo_t, M)
    scratch = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.full((len(lens), d_out), 7.0, dtype=torch.float32, device="cuda")
    wl.seq_lens[1] = 0
    lc = wl.lc
    api.decode_partials(wl.lay, wl.q, lc.cache, wl.block_table, wl.seq_lens, wl.Bk_t, lc.rope,
                        lc.decode_ws, lc.status)
    api.decode_combine_absorbed(wl.lay, wl.seq_lens, lc.max_pages, M, lc.decode_ws, scratch, out)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out[1]) == 0
    assert torch.count_nonzero(out[0]) > 0
