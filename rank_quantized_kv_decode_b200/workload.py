"""Synthetic workloads of the stated shapes, prepared on the device for the CUDA path.

Raw random material comes from ``synth`` (shared with the oracle); the offline setup
(factorisation, rank selection) is ``factorize``; storage of the context latents and the
prefill append go through the CUDA library.  Used by the benchmark, the smoke check and
the GPU tests.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from . import api, factorize, synth

STORE_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "mixed": torch.float16}


def stored_factor(a: np.ndarray, fmt: str, device) -> torch.Tensor:
    """Factor in its storage dtype: fp64 -> fp32 (nearest) -> storage dtype (nearest)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(STORE_DTYPE[fmt]).to(device).contiguous()


@dataclass
class Setup:
    """Offline factors of one layer (host, fp64)."""
    w: dict
    sigma: np.ndarray          # key spectrum
    key_rank: int
    value_ranks: list
    Bk: np.ndarray             # (r_k, H_kv*d)
    Bv: list                   # [(r_g, d)]
    Ak: np.ndarray | None      # (d_model, r_k) when latents are projected from x
    Av: list | None            # [(d_model, r_g)]
    value_stds: list           # [s_g[:r_g]]


def setup(w: dict, need_down: bool) -> Setup:
    """Factor W_k = U_k S V_k^T (JD) and W_v = U_v S V_v^T (HD per KV head), S the stated
    spectrum.  The key factors follow from the construction; the value factors from the SVD
    of each head's slice, ranks from the threshold rule of the workload."""
    idx = w["index"]
    H_kv, d, dm = w["n_kv_heads"], w["head_dim"], w["d_model"]
    n = H_kv * d
    m = min(dm, n)
    sigma = synth.spectrum(m, w["spectrum_scale"])
    r_k = w["key_rank"]
    Vk = synth.haar_frame(synth.rng(idx, "Vk"), n, r_k)
    Ak = None
    if need_down:
        Uk = synth.haar_frame(synth.rng(idx, "Uk"), dm, r_k)
        Ak = Uk * sigma[:r_k]
    Ak, Bk = factorize.fix_signs(Ak, Vk.T)
    Bk = np.ascontiguousarray(Bk)
    # values: slice g of W_v = U_v (S V_v^T)[:, g]; its singular values and right vectors are
    # those of M_g = S V_v[g rows]^T, and the left vectors are U_v times those of M_g.
    Vv = synth.haar_frame(synth.rng(idx, "Vv"), n, m)
    Uv = synth.haar_frame(synth.rng(idx, "Uv"), dm, m) if need_down else None
    svds = []
    for g in range(H_kv):
        Mg = sigma[:, None] * Vv[g * d:(g + 1) * d, :].T
        svds.append(np.linalg.svd(Mg, full_matrices=False))
    spectra = [s for _, s, _ in svds]
    if w["value_tau"] is not None:
        ranks = [max(1, factorize.rank_at(s, w["value_tau"])) for s in spectra]
    else:
        lo, hi = w["value_clip"]
        ranks = factorize.ranks_for_target_mean(spectra, lo, hi, w["value_mean"])
    Bv, Av, stds = [], [] if need_down else None, []
    for g, (Ug, sg, Vtg) in enumerate(svds):
        r = ranks[g]
        A_g, B_g = factorize.fix_signs(Ug[:, :r] * sg[:r], Vtg[:r])
        Bv.append(np.ascontiguousarray(B_g))
        stds.append(sg[:r].copy())
        if need_down:
            Av.append(Uv @ A_g)
    return Setup(w, sigma, r_k, ranks, Bk, Bv, Ak, Av, stds)


@dataclass
class Workload:
    w: dict
    st: Setup
    lay: object
    lc: api.LatentCache
    block_table: torch.Tensor   # int32 [B, max_pages]
    seq_lens: torch.Tensor      # int32 [B]
    q: torch.Tensor             # [B, H, d] bf16 / f32
    Bk_t: torch.Tensor          # [H_kv*d, r_k] storage dtype
    Bv: torch.Tensor            # [R_v, d] fp32
    A_t: torch.Tensor | None    # [proj_cols, d_model] bf16 / f32
    out: torch.Tensor           # [B, H, d] fp32
    extra: dict = field(default_factory=dict)


def x_dtype(fmt: str) -> torch.dtype:
    return torch.float32 if fmt == "f32" else torch.bfloat16


def context_latents(w: dict, st: Setup, b0: int, b1: int, t0: int, t1: int) -> np.ndarray:
    """fp32 context latents [K | V_0 | ...] of sequences b0..b1-1, positions t0..t1-1, drawn
    with the per-channel spectra (one generator stream per sequence and latent)."""
    rows = []
    for b in range(b0, b1):
        parts = [synth.latent_draw(synth.rng(w["index"], f"ck:{b}"), w["context"], st.sigma[:st.key_rank])]
        for g, s in enumerate(st.value_stds):
            parts.append(synth.latent_draw(synth.rng(w["index"], f"cv{g}:{b}"), w["context"], s))
        rows.append(np.concatenate(parts, axis=1)[t0:t1])
    return np.concatenate(rows, axis=0)


def hidden_rows(w: dict, name: str, n: int) -> np.ndarray:
    """Hidden rows x ~ N(0, 1) in their storage precision (fp32 or bf16-rounded), as fp32."""
    x = synth.gaussian(synth.rng(w["index"], name), (n, w["d_model"]), np.float32)
    return x if w["fmt"] == "f32" else synth.bf16_round(x)


def queries(w: dict) -> np.ndarray:
    q = synth.gaussian(synth.rng(w["index"], "q"), (w["batch"], w["n_q_heads"], w["head_dim"]),
                       np.float32)
    return q if w["fmt"] == "f32" else synth.bf16_round(q)


def block_table(w: dict, max_pages: int) -> np.ndarray:
    B = w["batch"]
    if w["shuffle_pages"]:
        perm = synth.page_permutation(synth.rng(w["index"], "pages"), B * max_pages)
    else:
        perm = np.arange(B * max_pages, dtype=np.int32)
    return perm.reshape(B, max_pages)


def build(index: int, device="cuda", seq_lens=None, st: Setup | None = None,
          chunk_tokens: int = 1 << 16, need_down: bool = False, **overrides) -> Workload:
    """Prepare workload ``index`` on ``device``: factors, page pool, block table, queries, and
    the context written into the cache (latents drawn and stored with starkv_quant_pack, or
    projected from hidden rows with starkv_append)."""
    w = synth.workload(index, **overrides)
    from_x = w["latents_from_x"]
    prefill = w["prefill_tokens"]
    if st is None:
        st = setup(w, need_down=need_down or from_x or prefill > 0)
    B, L = w["batch"], w["context"]
    cfg = api.make_config(w["n_q_heads"], w["n_kv_heads"], w["head_dim"], w["d_model"],
                          st.key_rank, st.value_ranks, w["fmt"], w["rope_theta"])
    lay = api.layout_init(cfg)
    max_pages = (L + 63) // 64
    max_pages += max_pages & 1  # whole 128-token tiles
    lens = np.full(B, L, dtype=np.int32) if seq_lens is None else np.asarray(seq_lens, np.int32)
    append_tokens = max(prefill, min(chunk_tokens, L) if from_x else 0, B)
    lc = api.LatentCache.create(lay, B * max_pages, B, max_pages, append_tokens, device)
    bt = torch.from_numpy(block_table(w, max_pages)).to(device)
    fmt = w["fmt"]
    Bk_t = stored_factor(st.Bk.T, fmt, device)
    Bv = torch.from_numpy(np.concatenate(st.Bv, axis=0).astype(np.float32)).to(device)
    A_t = None
    if st.Ak is not None:
        A = np.concatenate([st.Ak] + st.Av, axis=1)  # (d_model, proj_cols)
        A_t = torch.from_numpy(np.ascontiguousarray(A.T, dtype=np.float32)).to(x_dtype(fmt)).to(device)
    q = torch.from_numpy(queries(w)).to(x_dtype(fmt)).to(device)
    out = torch.empty(B, w["n_q_heads"], w["head_dim"], dtype=torch.float32, device=device)
    wl = Workload(w, st, lay, lc, bt, torch.from_numpy(lens).to(device), q, Bk_t, Bv, A_t, out)
    # context: positions [0, L - prefill) of every sequence (up to its own length)
    n_ctx = L - prefill
    for b in range(B):
        lb = int(min(lens[b], n_ctx))
        for t0 in range(0, lb, chunk_tokens):
            t1 = min(lb, t0 + chunk_tokens)
            seq = torch.full((t1 - t0,), b, dtype=torch.int32, device=device)
            pos = torch.arange(t0, t1, dtype=torch.int32, device=device)
            if from_x:
                x = torch.from_numpy(hidden_rows(w, f"x:{b}", L)[t0:t1]).to(x_dtype(fmt)).to(device)
                api.append(lay, x, A_t, seq, pos, bt, lc.cache, lc.append_ws, lc.status)
            else:
                lat = torch.from_numpy(context_latents(w, st, b, b + 1, t0, t1)).to(device)
                api.quant_pack(lay, lat, seq, pos, bt, lc.cache, lc.status)
    if prefill > 0:
        # the last ``prefill`` positions of sequence 0 go through the projection path
        x = torch.from_numpy(hidden_rows(w, "prefill", prefill)).to(x_dtype(fmt)).to(device)
        seq = torch.zeros(prefill, dtype=torch.int32, device=device)
        pos = torch.arange(n_ctx, L, dtype=torch.int32, device=device)
        wl.extra.update(prefill_x=x, prefill_seq=seq, prefill_pos=pos)
        api.append(lay, x, A_t, seq, pos, bt, lc.cache, lc.append_ws, lc.status)
    torch.cuda.synchronize(device)
    return wl


def decode(wl: Workload, **kw) -> torch.Tensor:
    api.decode_attention(wl.lay, wl.q, wl.lc.cache, wl.block_table, wl.seq_lens, wl.Bk_t, wl.Bv,
                         wl.lc.rope, wl.out, wl.lc.decode_ws, wl.lc.status, **kw)
    return wl.out


@dataclass
class HybridWorkload:
    """A hybrid layer (keys head-wise, values joint) and its cache on the device."""

    w: dict
    lay: object
    lc: api.LatentCache
    block_table: torch.Tensor
    seq_lens: torch.Tensor
    q: torch.Tensor
    Bk_t: torch.Tensor
    Bv: torch.Tensor
    out: torch.Tensor


def build_hybrid(device="cuda", seq_lens=None, **overrides) -> HybridWorkload:
    """Prepare the hybrid workload: layout, page pool, block table, queries, the factors in
    their operand types (B_k,g^T fp16 blocks, B_v fp32) and the context latents stored with
    starkv_quant_pack."""
    w = synth.hybrid_workload(**overrides)
    B, L, Hkv, d = w["batch"], w["context"], w["n_kv_heads"], w["head_dim"]
    cfg = api.make_hybrid_config(w["n_q_heads"], Hkv, d, w["d_model"], list(w["key_ranks"]),
                                 w["value_rank"], w["fmt"], w["rope_theta"])
    lay = api.hybrid_layout_init(cfg)
    max_pages = (L + 63) // 64
    max_pages += max_pages & 1
    lens = np.full(B, L, dtype=np.int32) if seq_lens is None else np.asarray(seq_lens, np.int32)
    lc = api.LatentCache.create(lay, B * max_pages, B, max_pages, B, device)
    bt = torch.from_numpy(block_table(w, max_pages)).to(device)
    Bk, Bv = synth.hybrid_factors(w)
    Bk_t = torch.from_numpy(np.concatenate([np.ascontiguousarray(b.T).ravel() for b in Bk])
                            .astype(np.float32)).to(torch.float16).to(device)
    Bv_t = torch.from_numpy(np.ascontiguousarray(Bv, dtype=np.float32)).to(device)
    q = torch.from_numpy(queries(w)).to(torch.bfloat16).to(device)
    out = torch.empty(B, w["n_q_heads"], d, dtype=torch.float32, device=device)
    for b in range(B):
        lb = int(lens[b])
        if lb == 0:
            continue
        lat = torch.from_numpy(synth.hybrid_latents(w, b, 0, lb)).to(device)
        seq = torch.full((lb,), b, dtype=torch.int32, device=device)
        pos = torch.arange(0, lb, dtype=torch.int32, device=device)
        api.quant_pack(lay, lat, seq, pos, bt, lc.cache, lc.status)
    torch.cuda.synchronize(device)
    return HybridWorkload(w, lay, lc, bt, torch.from_numpy(lens).to(device), q, Bk_t, Bv_t, out)


def decode_hybrid(hw: HybridWorkload) -> torch.Tensor:
    api.hybrid_decode(hw.lay, hw.q, hw.lc.cache, hw.block_table, hw.seq_lens, hw.Bk_t, hw.Bv,
                      hw.lc.rope, hw.out, hw.lc.decode_ws, hw.lc.status)
    return hw.out
