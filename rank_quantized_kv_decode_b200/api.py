"""Python binding of the C ABI.  Argument marshalling only: every step of the hot path runs
in the CUDA library; PyTorch supplies device memory and the stream.

Names mirror include/starkv.h (``starkv_append`` -> ``append`` ...).  Tensors must be
contiguous CUDA tensors on the current device; dtypes follow the header.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib as L


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    if t.device.index is not None and t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, but the current device is "
                         f"cuda:{torch.cuda.current_device()}")
    return t.data_ptr()


def _need(t, name: str, dtype, min_numel: int = 0, ndim: int | None = None) -> None:
    """Dtype and size a device argument must have, so that the library never reads or writes
    past the end of a caller's tensor (it sees only a pointer)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name}: expected {ndim} dimensions, got shape {tuple(t.shape)}")
    if t.numel() < min_numel:
        raise ValueError(f"{name}: {t.numel()} elements, at least {min_numel} needed")


def _operand_dtype(lay) -> torch.dtype:
    """dtype of x, A_t and q: fp32 for fp32 latents, else bf16."""
    return torch.float32 if lay.cfg.fmt == L.FMT["f32"] else torch.bfloat16


def _factor_dtype(lay) -> torch.dtype:
    """dtype of Bk_t: the tensor-core operand type of the format."""
    f = lay.cfg.fmt
    return torch.float32 if f == L.FMT["f32"] else (torch.bfloat16 if f == L.FMT["bf16"] else torch.float16)


def _check_tokens(n_tok: int, tok_seq, tok_pos, block_table, status) -> None:
    _need(tok_seq, "tok_seq", torch.int32, n_tok)
    _need(tok_pos, "tok_pos", torch.int32, n_tok)
    _need(block_table, "block_table", torch.int32, ndim=2)
    _need(status, "status", torch.int32, 1)


def _check_decode(lay, q, block_table, seq_lens, Bk_t, Bv, out, status) -> None:
    c = lay.cfg
    batch = seq_lens.shape[0]
    _need(seq_lens, "seq_lens", torch.int32, ndim=1)
    _need(block_table, "block_table", torch.int32, ndim=2)
    if block_table.shape[0] < batch:
        raise ValueError(f"block_table: {block_table.shape[0]} rows for {batch} sequences")
    _need(q, "q", _operand_dtype(lay), batch * c.n_q_heads * c.head_dim)
    _need(Bk_t, "Bk_t", _factor_dtype(lay), c.n_kv_heads * c.head_dim * c.key_rank)
    _need(Bv, "Bv", torch.float32, lay.value_rank_total * c.head_dim)
    _need(out, "out", torch.float32, batch * c.n_q_heads * c.head_dim)
    _need(status, "status", torch.int32, 1)


def _stream(stream) -> int | None:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def make_config(n_q_heads: int, n_kv_heads: int, head_dim: int, d_model: int, key_rank: int,
                value_ranks, fmt: str, rope_theta: float, page_tokens: int = 64) -> L.Config:
    c = L.Config()
    c.n_q_heads, c.n_kv_heads, c.head_dim, c.d_model = n_q_heads, n_kv_heads, head_dim, d_model
    c.key_rank = key_rank
    if len(value_ranks) != n_kv_heads:
        raise ValueError("one value rank per KV head")
    for g, r in enumerate(value_ranks):
        c.value_rank[g] = int(r)
    c.fmt = L.FMT[fmt]
    c.page_tokens = page_tokens
    c.rope_theta = float(rope_theta)
    return c


def layout_init(cfg: L.Config) -> L.Layout:
    lay = L.Layout()
    L.check(L.load().starkv_layout_init(ctypes.byref(cfg), ctypes.byref(lay)), "starkv_layout_init")
    return lay


def make_hybrid_config(n_q_heads: int, n_kv_heads: int, head_dim: int, d_model: int, key_ranks,
                       value_rank: int, fmt: str, rope_theta: float,
                       page_tokens: int = 64) -> L.HybridConfig:
    """Config of the hybrid assignment: one key latent per KV head (ranks ``key_ranks``), one
    joint value latent of rank ``value_rank``."""
    c = L.HybridConfig()
    c.n_q_heads, c.n_kv_heads, c.head_dim, c.d_model = n_q_heads, n_kv_heads, head_dim, d_model
    if len(key_ranks) != n_kv_heads:
        raise ValueError("one key rank per KV head")
    for g, r in enumerate(key_ranks):
        c.key_rank[g] = int(r)
    c.value_rank = int(value_rank)
    c.fmt = L.FMT[fmt]
    c.page_tokens = page_tokens
    c.rope_theta = float(rope_theta)
    return c


def hybrid_layout_init(cfg: L.HybridConfig) -> L.Layout:
    lay = L.Layout()
    L.check(L.load().starkv_hybrid_layout_init(ctypes.byref(cfg), ctypes.byref(lay)),
            "starkv_hybrid_layout_init")
    return lay


def hybrid_decode(lay, q, cache, block_table, seq_lens, Bk_t, Bv, rope_table, out, workspace,
                  status, stream=None) -> None:
    """Decode with the hybrid assignment.  Bk_t: fp16, the blocks [d][r_k,g] of the KV heads in
    order (flat); Bv: fp32 [r_v][H_kv d]."""
    c = lay.cfg
    batch = seq_lens.shape[0]
    _need(seq_lens, "seq_lens", torch.int32, ndim=1)
    _need(block_table, "block_table", torch.int32, ndim=2)
    if block_table.shape[0] < batch:
        raise ValueError(f"block_table: {block_table.shape[0]} rows for {batch} sequences")
    rk = sum(lay.seg[g].rank for g in range(c.n_kv_heads))
    _need(q, "q", torch.bfloat16, batch * c.n_q_heads * c.head_dim)
    _need(Bk_t, "Bk_t", torch.float16, c.head_dim * rk)
    _need(Bv, "Bv", torch.float32, lay.value_rank_total * c.n_kv_heads * c.head_dim)
    _need(out, "out", torch.float32, batch * c.n_q_heads * c.head_dim)
    _need(status, "status", torch.int32, 1)
    L.check(L.load().starkv_hybrid_decode(
        ctypes.byref(lay), _ptr(q), _ptr(cache), cache.numel() * cache.element_size() // lay.page_bytes,
        _ptr(block_table), block_table.shape[1], _ptr(seq_lens), batch, _ptr(Bk_t), _ptr(Bv),
        _ptr(rope_table), rope_table.numel() * rope_table.element_size(), _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)), "starkv_hybrid_decode")


def alloc(lay: L.Layout, num_pages: int, batch: int, max_pages: int,
          max_append_tokens: int) -> L.Sizes:
    s = L.Sizes()
    L.check(L.load().starkv_alloc(ctypes.byref(lay), num_pages, batch, max_pages,
                                  max_append_tokens, ctypes.byref(s)), "starkv_alloc")
    return s


def rope_init(lay: L.Layout, max_pages: int, table: torch.Tensor, stream=None) -> None:
    L.check(L.load().starkv_rope_init(ctypes.byref(lay), max_pages, _ptr(table),
                                      table.numel() * table.element_size(), _stream(stream)),
            "starkv_rope_init")


def quant_pack(lay, latents, tok_seq, tok_pos, block_table, cache, status, stream=None) -> None:
    n_tok = latents.shape[0]
    _need(latents, "latents", torch.float32, n_tok * lay.proj_cols)
    _check_tokens(n_tok, tok_seq, tok_pos, block_table, status)
    L.check(L.load().starkv_quant_pack(
        ctypes.byref(lay), _ptr(latents), n_tok, _ptr(tok_seq), _ptr(tok_pos), _ptr(block_table),
        block_table.shape[1], block_table.shape[0], _ptr(cache),
        cache.numel() * cache.element_size() // lay.page_bytes, _ptr(status), _stream(stream)),
        "starkv_quant_pack")


def append(lay, x, A_t, tok_seq, tok_pos, block_table, cache, workspace, status,
           latents_out=None, stream=None) -> None:
    n_tok = x.shape[0]
    _need(x, "x", _operand_dtype(lay), n_tok * lay.cfg.d_model)
    _need(A_t, "A_t", _operand_dtype(lay), lay.proj_cols * lay.cfg.d_model)
    _need(latents_out, "latents_out", torch.float32, n_tok * lay.proj_cols)
    _check_tokens(n_tok, tok_seq, tok_pos, block_table, status)
    L.check(L.load().starkv_append(
        ctypes.byref(lay), _ptr(x), x.shape[0], _ptr(A_t), _ptr(tok_seq), _ptr(tok_pos),
        _ptr(block_table), block_table.shape[1], block_table.shape[0], _ptr(cache),
        cache.numel() * cache.element_size() // lay.page_bytes, _ptr(latents_out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(status),
        _stream(stream)), "starkv_append")


def dequant(lay, cache, tok_seq, tok_pos, block_table, latents_out, status, stream=None) -> None:
    n_tok = tok_seq.shape[0]
    _need(latents_out, "latents_out", torch.float32, n_tok * lay.proj_cols)
    _check_tokens(n_tok, tok_seq, tok_pos, block_table, status)
    L.check(L.load().starkv_dequant(
        ctypes.byref(lay), _ptr(cache), cache.numel() * cache.element_size() // lay.page_bytes,
        _ptr(tok_seq), _ptr(tok_pos), tok_seq.shape[0], _ptr(block_table), block_table.shape[1],
        block_table.shape[0], _ptr(latents_out), _ptr(status), _stream(stream)), "starkv_dequant")


def decode_attention(lay, q, cache, block_table, seq_lens, Bk_t, Bv, rope_table, out, workspace,
                     status, max_ctas: int = 0, n_ranges: int = 0, timeout_ms: int = 0,
                     cta_group: int = 0, stream=None) -> None:
    _check_decode(lay, q, block_table, seq_lens, Bk_t, Bv, out, status)
    opts = L.DecodeOpts(max_ctas, n_ranges, timeout_ms, cta_group)
    L.check(L.load().starkv_decode_attention(
        ctypes.byref(lay), _ptr(q), _ptr(cache),
        cache.numel() * cache.element_size() // lay.page_bytes, _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], _ptr(Bk_t), _ptr(Bv),
        _ptr(rope_table), rope_table.numel() * rope_table.element_size(), _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), ctypes.byref(opts),
        _ptr(status), _stream(stream)), "starkv_decode_attention")


def decode_attention_noalloc(lay, q, cache, block_table, seq_lens, Bk_t, Bv, rope_table, out,
                             status, max_ctas: int = 0, n_ranges: int = 0, timeout_ms: int = 0,
                             stream=None) -> None:
    """decode_attention with the library's built-in 16 MiB scratch instead of a workspace
    (for callers that cannot allocate device memory; see include/starkv.h)."""
    _check_decode(lay, q, block_table, seq_lens, Bk_t, Bv, out, status)
    opts = L.DecodeOpts(max_ctas, n_ranges, timeout_ms, 0)
    L.check(L.load().starkv_decode_attention_noalloc(
        ctypes.byref(lay), _ptr(q), _ptr(cache),
        cache.numel() * cache.element_size() // lay.page_bytes, _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], _ptr(Bk_t), _ptr(Bv),
        _ptr(rope_table), rope_table.numel() * rope_table.element_size(), _ptr(out),
        ctypes.byref(opts), _ptr(status), _stream(stream)), "starkv_decode_attention_noalloc")


def decode_plan(lay, batch: int, max_pages: int, max_ctas: int = 0, n_ranges: int = 0,
                cta_group: int = 0, num_sms: int = 148, smem_per_block: int = 232448) -> L.DecodePlan:
    """The launch shape the decode calls choose (host only; defaults are a B200's figures)."""
    opts = L.DecodeOpts(max_ctas, n_ranges, 0, cta_group)
    out = L.DecodePlan()
    L.check(L.load().starkv_decode_plan_query(ctypes.byref(lay), batch, max_pages,
                                              ctypes.byref(opts), num_sms, smem_per_block,
                                              ctypes.byref(out)), "starkv_decode_plan_query")
    return out


def decode_partials(lay, q, cache, block_table, seq_lens, Bk_t, rope_table, workspace, status,
                    max_ctas: int = 0, n_ranges: int = 0, timeout_ms: int = 0,
                    cta_group: int = 0, stream=None) -> None:
    _check_decode(lay, q, block_table, seq_lens, Bk_t, None, None, status)
    opts = L.DecodeOpts(max_ctas, n_ranges, timeout_ms, cta_group)
    L.check(L.load().starkv_decode_partials(
        ctypes.byref(lay), _ptr(q), _ptr(cache),
        cache.numel() * cache.element_size() // lay.page_bytes, _ptr(block_table),
        block_table.shape[1], _ptr(seq_lens), seq_lens.shape[0], _ptr(Bk_t), _ptr(rope_table),
        rope_table.numel() * rope_table.element_size(), _ptr(workspace),
        workspace.numel() * workspace.element_size(), ctypes.byref(opts), _ptr(status),
        _stream(stream)), "starkv_decode_partials")


def decode_combine(lay, seq_lens, max_pages: int, Bv, workspace, out, stream=None) -> None:
    c = lay.cfg
    _need(seq_lens, "seq_lens", torch.int32, ndim=1)
    _need(Bv, "Bv", torch.float32, lay.value_rank_total * c.head_dim)
    _need(out, "out", torch.float32, seq_lens.shape[0] * c.n_q_heads * c.head_dim)
    L.check(L.load().starkv_decode_combine(
        ctypes.byref(lay), _ptr(seq_lens), seq_lens.shape[0], max_pages, _ptr(Bv),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out),
        _stream(stream)), "starkv_decode_combine")


def absorbed_sizes(lay, batch: int, d_out: int) -> tuple[int, int]:
    """(rows of the absorbed matrix M, scratch bytes of decode_combine_absorbed)."""
    rows, nbytes = ctypes.c_int64(0), ctypes.c_size_t(0)
    L.check(L.load().starkv_absorbed_sizes(ctypes.byref(lay), batch, d_out, ctypes.byref(rows),
                                           ctypes.byref(nbytes)), "starkv_absorbed_sizes")
    return int(rows.value), int(nbytes.value)


def absorb_output_weights(lay, Bv, Wo, M, stream=None) -> None:
    """M[rows of head h] = B_v,g(h) Wo[h d:(h+1) d] (fp32, on the device)."""
    c = lay.cfg
    _need(Bv, "Bv", torch.float32, lay.value_rank_total * c.head_dim)
    _need(Wo, "Wo", torch.float32, c.n_q_heads * c.head_dim, ndim=2)
    if Wo.shape[0] != c.n_q_heads * c.head_dim:
        raise ValueError(f"Wo: {Wo.shape[0]} rows, expected n_q_heads * head_dim")
    rows, _ = absorbed_sizes(lay, 1, Wo.shape[1])
    _need(M, "M", torch.float32, rows * Wo.shape[1])
    L.check(L.load().starkv_absorb_output_weights(ctypes.byref(lay), _ptr(Bv), _ptr(Wo),
                                                  Wo.shape[1], _ptr(M), _stream(stream)),
            "starkv_absorb_output_weights")


def decode_combine_absorbed(lay, seq_lens, max_pages: int, M, workspace, scratch, out,
                            stream=None) -> None:
    """Merge the partial records and write out[b] = sum_h a_b,h M_h (out: [batch][d_out])."""
    _need(seq_lens, "seq_lens", torch.int32, ndim=1)
    _need(out, "out", torch.float32, ndim=2)
    if out.shape[0] < seq_lens.shape[0]:
        raise ValueError(f"out: {out.shape[0]} rows for {seq_lens.shape[0]} sequences")
    rows, _ = absorbed_sizes(lay, seq_lens.shape[0], out.shape[1])
    _need(M, "M", torch.float32, rows * out.shape[1])
    L.check(L.load().starkv_decode_combine_absorbed(
        ctypes.byref(lay), _ptr(seq_lens), seq_lens.shape[0], max_pages, _ptr(M), out.shape[1],
        _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(scratch),
        scratch.numel() * scratch.element_size(), _ptr(out), _stream(stream)),
        "starkv_decode_combine_absorbed")


def diag_bounded_wait(timeout_ms: int, status, stream=None) -> None:
    L.check(L.load().starkv_diag_bounded_wait(timeout_ms, _ptr(status), _stream(stream)),
            "starkv_diag_bounded_wait")


def _bytes(n: int, device) -> torch.Tensor:
    # 256-byte aligned raw buffer (the caching allocator aligns blocks to 512 bytes)
    return torch.empty(max(int(n), 16), dtype=torch.uint8, device=device)


@dataclass
class LatentCache:
    """Caller-side buffers of one layer's compressed cache: the page pool, the RoPE table and
    the workspaces, sized by ``starkv_alloc``.  Plain device memory owned by PyTorch."""

    layout: L.Layout
    num_pages: int
    batch: int
    max_pages: int
    max_append_tokens: int
    cache: torch.Tensor
    rope: torch.Tensor
    decode_ws: torch.Tensor
    append_ws: torch.Tensor
    status: torch.Tensor

    @classmethod
    def create(cls, lay: L.Layout, num_pages: int, batch: int, max_pages: int,
               max_append_tokens: int, device="cuda") -> "LatentCache":
        s = alloc(lay, num_pages, batch, max_pages, max_append_tokens)
        c = cls(lay, num_pages, batch, max_pages, max_append_tokens,
                _bytes(s.cache_bytes, device), _bytes(s.rope_table_bytes, device),
                _bytes(s.decode_workspace_bytes, device), _bytes(s.append_workspace_bytes, device),
                torch.zeros(1, dtype=torch.int32, device=device))
        rope_init(lay, max_pages, c.rope)
        return c
