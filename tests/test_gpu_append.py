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
    # stored values, read back: (1) bit-exact against the oracle's storage of the GPU's own
    # fp32 latents (the quantiser and the packing are exact functions of their input)
    back = torch.empty_like(lat_out)
    api.dequant(lay, lc.cache, seq, pos, table, back, lc.status)
    torch.cuda.synchronize()
    assert lc.status.item() == 0
    stored_gpu = back.cpu().numpy().astype(np.float64)
    Ck_g, Cv_g = ref.stored(lat_out.cpu().numpy())
    np.testing.assert_array_equal(stored_gpu, np.concatenate([Ck_g] + Cv_g, axis=1))
    # (2) against the oracle's storage of its own fp64 latents: the projections differ by the
    # fp32 rounding above, and the quantiser is discontinuous (a group's absmax near an fp16
    # rounding boundary of its scale moves the whole group to the neighbouring scale), so each
    # stored value may differ by at most one quantisation step of either scale (mixed), or by
    # the projection error plus one bf16 spacing (bf16), or the projection error (f32)
    Ck, Cv = ref.stored(want.astype(np.float32))
    stored_ref = np.concatenate([Ck] + Cv, axis=1)
    diff = np.abs(stored_gpu - stored_ref)
    if fmt == "mixed":
        cols = np.concatenate([[0], np.cumsum([st.key_rank] + st.value_ranks)])
        for li in range(len(cols) - 1):
            sl = slice(cols[li], cols[li + 1])
            _, _, sc_ref = O.quantize_rows(want[:, sl].astype(np.float32), cols[li + 1] - cols[li])
            _, _, sc_gpu = O.quantize_rows(got[:, sl].astype(np.float32), cols[li + 1] - cols[li])
            step = np.maximum(sc_ref.astype(np.float64), sc_gpu.astype(np.float64)).max(axis=1, keepdims=True)
            assert np.all(diff[:, sl] <= 1.01 * step + 1e-12)
        print(f"values differing from the storage of the fp64 latents: {np.mean(diff > 0):.2e}")
    else:
        mag = np.maximum(np.abs(stored_ref), np.abs(stored_gpu))
        spacing = np.exp2(np.floor(np.log2(np.maximum(mag, 1e-30))) - (7 if fmt == "bf16" else 23))
        assert np.all(diff <= proj_err * (1 + 1e-6) + spacing)
