"""GPU parity of the latent write path: projection c = x A on the tensor cores (fp32
accumulation) against the fp64 oracle, then the stored values (codes may differ from the
oracle's only where the fp32 projection crossed a rounding boundary of the quantiser)."""
import numpy as np
import pytest
import torch

import oracle as O
from rank_quantized_kv_decode_b200 import api
from rank_quantized_kv_decode_b200 import workload as W

from oracle.workloads import ref_for

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("index,n_tok", [(1, 300), (5, 8), (5, 333), (2, 8), (3, 16), (3, 200), (4, 32)])
def test_append_projection_and_store(index, n_tok):
    ref = ref_for(index, True)
    w = ref.w
    fmt = w["fmt"]
    st = W.setup(dict(w), need_down=True)
    assert st.value_ranks == ref.ranks
    cfg = api.make_config(w["n_q_heads"], w["n_kv_heads"], w["head_dim"], w["d_model"],
                          st.key_rank, st.value_ranks, fmt, w["rope_theta"])
    lay = api.layout_init(cfg)
    dev = "cuda"
    batch, max_pages = 2, 8
    lc = api.LatentCache.create(lay, batch * max_pages, batch, max_pages, n_tok, dev)
    lc.cache.zero_()
    g = np.random.default_rng(index * 1000 + n_tok)
    pairs = g.choice(batch * max_pages * 64, size=n_tok, replace=False)
    seq = torch.from_numpy((pairs // (max_pages * 64)).astype(np.int32)).to(dev)
    pos = torch.from_numpy((pairs % (max_pages * 64)).astype(np.int32)).to(dev)
    table = torch.arange(batch * max_pages, dtype=torch.int32, device=dev).reshape(batch, max_pages)
    x_np = ref.hidden("append-test", n_tok)
    x = torch.from_numpy(x_np).to(W.x_dtype(fmt)).to(dev)
    A = np.concatenate([st.Ak] + st.Av, axis=1)
    A_t = torch.from_numpy(np.ascontiguousarray(A.T, dtype=np.float32)).to(W.x_dtype(fmt)).to(dev)
    lat_out = torch.empty(n_tok, lay.proj_cols, dtype=torch.float32, device=dev)
    api.append(lay, x, A_t, seq, pos, table, lc.cache, lc.append_ws, lc.status, latents_out=lat_out)
    torch.cuda.synchronize()
    assert lc.status.item() == 0
    got = lat_out.cpu().numpy().astype(np.float64)
    want = O.project(x_np, ref.A_s)
    # bf16 operands: exact products, fp32 accumulation -> far below 1e-4 of the row scale;
    # fp32 operands run as 3xTF32 (hi*hi + hi*lo + lo*hi): about 2^-20 per product
    scale = np.linalg.norm(want, axis=1, keepdims=True) / np.sqrt(want.shape[1])
    proj_tol = 1e-4
    proj_err = np.abs(got - want)
    assert np.max(proj_err / scale) < proj_tol
    # stored values: read back and compare with the oracle's storage of its own latents
    back = torch.empty_like(lat_out)
    api.dequant(lay, lc.cache, seq, pos, table, back, lc.status)
    torch.cuda.synchronize()
    stored_gpu = back.cpu().numpy().astype(np.float64)
    Ck, Cv = ref.stored(want.astype(np.float32))
    stored_ref = np.concatenate([Ck] + Cv, axis=1)
    diff = np.abs(stored_gpu - stored_ref)
    if fmt == "mixed":
        # one quantisation step at most, and rarely
        cols = np.concatenate([[0], np.cumsum([st.key_rank] + st.value_ranks)])
        frac = np.mean(diff > 0)
        assert frac < 2e-3, f"{frac:.2e} of stored values differ"
        for li in range(len(cols) - 1):
            part = want[:, cols[li]:cols[li + 1]].astype(np.float32)
            _, _, sc = O.quantize_rows(part, part.shape[1])
            step = sc.astype(np.float64).max(axis=1, keepdims=True)
            assert np.all(diff[:, cols[li]:cols[li + 1]] <= 1.01 * step + 1e-12)
    else:
        # the store itself is exact (f32) or one rounding (bf16): the difference is the
        # projection error plus at most one storage ulp
        ulp = np.abs(stored_ref) * (2.0 ** -8 if fmt == "bf16" else 2.0 ** -23)
        assert np.all(diff <= proj_err * (1 + 1e-6) + ulp)
