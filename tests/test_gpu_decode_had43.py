"""GPU parity of decode attention read from pages in the pages' own 4-bit/3-bit format
(STAR-KV technical summary, Methodology §3: a block-wise Hadamard rotation folded into the
factors, the leading fifth of a latent's channels as 4-bit codes, the rest as 3-bit codes,
fp16 group scales) against the fp64 oracle.

Inputs: the stated GQA and MHA layers' factors and drawn latents; each latent is rotated by its
block transform and each factor by the transposed transform (K = c B = (c T)(T^T B)), as the
offline setup folds it.  The rotated fp32 latents are stored by starkv_quant_pack; the oracle
stores the same fp32 latents with its own quantiser and decodes its own pages."""
import numpy as np
import pytest
import torch

import oracle.starkv_oracle as O
from oracle.workloads import Ref, tolerance_check
from rank_quantized_kv_decode_b200 import api, synth

pytestmark = pytest.mark.gpu


def _case(index, overrides, lens, key_rank=None):
    w = synth.workload(index, **overrides)
    if key_rank is not None:
        w["key_rank"] = key_rank
    ref = Ref(w, False)
    Tk = O.hadamard_transform(w["key_rank"])
    Tv = [O.hadamard_transform(r) for r in ref.ranks]
    Bk = Tk.T @ ref.Bk                              # rotated factors (fp64)
    Bv = [t.T @ b for t, b in zip(Tv, ref.Bv)]
    ranks = [w["key_rank"]] + ref.ranks
    cols = np.concatenate([[0], np.cumsum(ranks)])
    lat = []
    for b, Lb in enumerate(lens):
        raw = ref.drawn_latents(b)[:Lb].astype(np.float64)
        parts = [raw[:, cols[i]:cols[i + 1]] @ (Tk if i == 0 else Tv[i - 1])
                 for i in range(len(ranks))]
        lat.append(np.concatenate(parts, axis=1).astype(np.float32))
    return w, ref, Bk, Bv, ranks, cols, lat


def _run(index, overrides, lens, key_rank=None, **decode_kw):
    w, ref, Bk, Bv, ranks, cols, lat = _case(index, overrides, lens, key_rank)
    dev = "cuda"
    H, Hkv, d = w["n_q_heads"], w["n_kv_heads"], w["head_dim"]
    lay = api.layout_init(api.make_config(H, Hkv, d, w["d_model"], w["key_rank"], ref.ranks,
                                          "had43", w["rope_theta"]))
    B = len(lens)
    max_pages = (max(lens) + 63) // 64
    max_pages += max_pages & 1
    lc = api.LatentCache.create(lay, B * max_pages, B, max_pages, 0, dev)
    g = np.random.default_rng(index * 7 + B)
    table = torch.from_numpy(g.permutation(B * max_pages).astype(np.int32).reshape(B, max_pages)).to(dev)
    for b, Lb in enumerate(lens):
        if Lb == 0:
            continue
        seq = torch.full((Lb,), b, dtype=torch.int32, device=dev)
        pos = torch.arange(Lb, dtype=torch.int32, device=dev)
        api.quant_pack(lay, torch.from_numpy(lat[b]).to(dev), seq, pos, table, lc.cache, lc.status)
    q = torch.from_numpy(ref.queries()[:B]).to(torch.bfloat16).to(dev).contiguous()
    Bk_t = torch.from_numpy(np.ascontiguousarray(Bk.T, dtype=np.float32)).to(torch.float16).to(dev)
    Bv_d = torch.from_numpy(np.concatenate(Bv, axis=0).astype(np.float32)).to(dev)
    out = torch.empty(B, H, d, dtype=torch.float32, device=dev)
    seq_lens = torch.tensor(lens, dtype=torch.int32, device=dev)
    api.decode_attention(lay, q, lc.cache, table, seq_lens, Bk_t, Bv_d, lc.rope, out, lc.decode_ws,
                         lc.status, **decode_kw)
    torch.cuda.synchronize()
    assert lc.status.item() == 0
    got = out.cpu().numpy()
    # oracle: its own storage of the same rotated latents, the stored factors
    Bk_s = np.asarray(Bk, np.float32).astype(np.float16).astype(np.float64)
    Bv_s = [np.asarray(b, np.float32).astype(np.float64) for b in Bv]
    qs = ref.queries()
    for b, Lb in enumerate(lens):
        if Lb == 0:
            assert np.count_nonzero(got[b]) == 0
            continue
        stored = [O.stored_rows(lat[b][:, cols[i]:cols[i + 1]], ranks[i], O.HAD43)
                  for i in range(len(ranks))]
        want = O.decode_attention(qs[b], stored[0], stored[1:], Bk_s, Bv_s, w["rope_theta"], Hkv)
        tolerance_check(got[b], want)


@pytest.mark.parametrize("cta_group", [0, 1])
def test_had43_gqa_rank256_resident_operand(cta_group):
    # the GQA layer: key rank 256 (resident operand), value ranks ~32; ragged lengths and an
    # empty sequence; 4-bit blocks of 52 channels (the 8-channel groups straddle both the
    # 4-bit/3-bit boundary and the 32-channel scale groups)
    _run(4, dict(batch=4, context=1000), [1000, 1, 333, 0], cta_group=cta_group)


def test_had43_mha_rank1024_staged_codes():
    # the MHA layer: key rank 1024 (codes staged per tile, operand streamed through the ring)
    _run(3, dict(batch=2, context=520), [520, 129])


def test_had43_rank2048_codes_from_global_memory():
    # key rank 2048: the tile's codes do not fit in shared memory; read from the pages
    _run(3, dict(batch=1, context=200), [200], key_rank=2048)


def test_had43_tiny_fp_ranks():
    # the tiny layer's shapes (d = 64, 4 heads, value ranks from thresholding)
    _run(1, dict(batch=2, fmt="bf16", latents_from_x=False), [256, 77])


def test_had43_sharp_softmax():
    # query x 8: a few tokens dominate, so an error in a score shows in the output
    orig = Ref.queries

    def sharp(self):
        return orig(self) * 8.0
    Ref.queries = sharp
    try:
        _run(4, dict(batch=1, context=700), [700])
    finally:
        Ref.queries = orig
