"""GPU parity of the latent write with the hybrid layout (keys head-wise, values joint; STAR-KV
technical summary, Methodology §2): c = x [A_k,0 | ... | A_k,H_kv-1 | A_v] on the decode-step
path (one fused launch, <= 32 tokens) and on the prefill path (projection + store), against
the fp64 oracle's projection; the stored pages read back bit-exactly as the oracle stores the
GPU's own fp32 latents."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle.workloads import stored_factor
from rank_quantized_kv_decode_b200 import api

pytestmark = pytest.mark.gpu

H, HKV, D, DM = 32, 8, 128, 4096
KR = [32, 16, 48, 32, 32, 16, 48, 32]
RV = 256


@pytest.mark.parametrize("n_tok", [8, 32, 200])
def test_hybrid_append_projection_and_store(n_tok):
    lay = api.hybrid_layout_init(api.make_hybrid_config(H, HKV, D, DM, KR, RV, "mixed", 500000.0))
    dev = "cuda"
    batch, max_pages = 2, 8
    lc = api.LatentCache.create(lay, batch * max_pages, batch, max_pages, n_tok, dev)
    lc.cache.zero_()
    g = np.random.default_rng(4242 + n_tok)
    pairs = g.choice(batch * max_pages * 64, size=n_tok, replace=False)
    seq = torch.from_numpy((pairs // (max_pages * 64)).astype(np.int32)).to(dev)
    pos = torch.from_numpy((pairs % (max_pages * 64)).astype(np.int32)).to(dev)
    table = torch.from_numpy(g.permutation(batch * max_pages).astype(np.int32).reshape(batch, max_pages)).to(dev)
    # inputs in their storage precision (bf16), as fp32 arrays both sides start from
    x_np = O.bf16_rne(g.standard_normal((n_tok, DM)).astype(np.float32)).reshape(n_tok, DM)
    A_np = stored_factor(g.standard_normal((DM, lay.proj_cols)) / np.sqrt(DM), O.BF16)
    x = torch.from_numpy(x_np.astype(np.float32)).to(torch.bfloat16).to(dev)
    A_t = torch.from_numpy(np.ascontiguousarray(A_np.T, dtype=np.float32)).to(torch.bfloat16).to(dev)
    lat_out = torch.empty(n_tok, lay.proj_cols, dtype=torch.float32, device=dev)
    api.append(lay, x, A_t, seq, pos, table, lc.cache, lc.append_ws, lc.status, latents_out=lat_out)
    torch.cuda.synchronize()
    assert lc.status.item() == 0
    got = lat_out.cpu().numpy().astype(np.float64)
    want = O.project(x_np, A_np)
    scale = np.linalg.norm(want, axis=1, keepdims=True) / np.sqrt(want.shape[1])
    assert np.max(np.abs(got - want) / scale) < 1e-4
    # read-back, bit-exact against the oracle's storage of the GPU's fp32 latents, per latent
    back = torch.empty_like(lat_out)
    api.dequant(lay, lc.cache, seq, pos, table, back, lc.status)
    torch.cuda.synchronize()
    assert lc.status.item() == 0
    lat32 = lat_out.cpu().numpy()
    ranks = KR + [RV]
    cols = np.concatenate([[0], np.cumsum(ranks)])
    want_stored = np.concatenate(
        [O.stored_rows(lat32[:, cols[i]:cols[i + 1]], ranks[i], O.MIXED) for i in range(len(ranks))],
        axis=1)
    np.testing.assert_array_equal(back.cpu().numpy().astype(np.float64), want_stored)
    # the pages themselves, byte for byte, against the oracle's encoding of those latents
    layout = O.hybrid_page_layout(O.MIXED, KR, RV)
    cache = np.zeros((batch * max_pages, layout["page_bytes"]), dtype=np.uint8)
    O.encode_tokens(cache, layout, table.cpu().numpy(), seq.cpu().numpy(), pos.cpu().numpy(), lat32)
    gpu_pages = lc.cache[: batch * max_pages * lay.page_bytes].cpu().numpy().reshape(batch * max_pages, -1)
    np.testing.assert_array_equal(gpu_pages, cache)
