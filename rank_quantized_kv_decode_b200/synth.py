"""Seeded synthetic inputs shared by the CUDA path's tests/bench and by the fp64 oracle.

This module holds only random material and the stated workload shapes: Haar-random
orthonormal frames, Gaussian hidden rows, queries and latent draws, page permutations and
sequence lengths.  It contains none of the method's arithmetic (no SVD, no thresholding,
no quantisation, no RoPE, no attention).  Both sides call it with the same seed and
receive the same numbers; each side then runs its own setup and its own computation.

Every generator is a NumPy ``PCG64`` stream keyed by ``(workload index, stream name)`` so
that the draws for one tensor never depend on the order in which other tensors are drawn.
"""
from __future__ import annotations

import hashlib

import numpy as np

# --------------------------------------------------------------------------------------
# The five stated workloads.  Shapes only; ranks that the method derives (value ranks) are
# described by the rule that derives them (threshold tau, or clip range + target mean).
# --------------------------------------------------------------------------------------
WORKLOADS = {
    1: dict(
        name="tiny-f32-4h-d64-ctx256",
        batch=1, n_q_heads=4, n_kv_heads=4, head_dim=64, d_model=256, context=256,
        spectrum_scale=16.0, key_rank=64, value_tau=0.05, value_clip=None, value_mean=None,
        fmt="f32", rope_theta=10000.0, page_tokens=64, shuffle_pages=False,
        latents_from_x=True, prefill_tokens=0,
    ),
    2: dict(
        name="llama2-7b-mha-bf16-b8-ctx4096",
        batch=8, n_q_heads=32, n_kv_heads=32, head_dim=128, d_model=4096, context=4096,
        spectrum_scale=256.0, key_rank=1024, value_tau=None, value_clip=(16, 64), value_mean=32,
        fmt="bf16", rope_theta=10000.0, page_tokens=64, shuffle_pages=False,
        latents_from_x=False, prefill_tokens=0,
    ),
    3: dict(
        name="llama2-7b-mha-int8int4-b16-ctx16384",
        batch=16, n_q_heads=32, n_kv_heads=32, head_dim=128, d_model=4096, context=16384,
        spectrum_scale=256.0, key_rank=1024, value_tau=None, value_clip=(16, 64), value_mean=32,
        fmt="mixed", rope_theta=10000.0, page_tokens=64, shuffle_pages=False,
        latents_from_x=False, prefill_tokens=0,
    ),
    4: dict(
        name="llama3-8b-gqa-int8int4-b32-ctx32768-paged",
        batch=32, n_q_heads=32, n_kv_heads=8, head_dim=128, d_model=4096, context=32768,
        spectrum_scale=256.0, key_rank=256, value_tau=None, value_clip=(8, 48), value_mean=32,
        fmt="mixed", rope_theta=500000.0, page_tokens=64, shuffle_pages=True,
        latents_from_x=False, prefill_tokens=0,
    ),
    5: dict(
        name="llama3-8b-gqa-int8int4-b1-ctx131072-splitk+prefill8192",
        batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, d_model=4096, context=131072,
        spectrum_scale=256.0, key_rank=256, value_tau=None, value_clip=(8, 48), value_mean=32,
        fmt="mixed", rope_theta=500000.0, page_tokens=64, shuffle_pages=True,
        latents_from_x=False, prefill_tokens=8192,
    ),
}


# The hybrid assignment (keys head-wise, values joint) at the shape of workload 4: GQA 32/8,
# d 128, int8/int4, 32 sequences x 32768 tokens, paged.  Per-head key ranks are multiples of 16
# (the hybrid kernel's k-step) averaging 32, the same total of 256 as workload 4's joint key;
# one joint value latent of rank 256, the same total as workload 4's head-wise values.
HYBRID_INDEX = 6
HYBRID = dict(
    name="llama3-8b-gqa-hybrid-int8int4-b32-ctx32768-paged",
    batch=32, n_q_heads=32, n_kv_heads=8, head_dim=128, d_model=4096, context=32768,
    spectrum_scale=256.0, key_ranks=(32, 16, 48, 32, 32, 16, 48, 32), value_rank=256,
    fmt="mixed", rope_theta=500000.0, page_tokens=64, shuffle_pages=True,
)


def hybrid_workload(**overrides) -> dict:
    """A copy of the hybrid workload with optional shape overrides."""
    w = dict(HYBRID)
    w.update(overrides)
    w["index"] = HYBRID_INDEX
    return w


def hybrid_factors(w: dict):
    """Factors of a hybrid layer: per KV head g, B_k,g (r_k,g x d) with orthonormal rows; the
    joint B_v (r_v x H_kv d) with orthonormal rows.  Returned as fp64."""
    d, Hkv = w["head_dim"], w["n_kv_heads"]
    Bk = [haar_frame(rng(w["index"], f"Bk{g}"), d, int(r)).T for g, r in enumerate(w["key_ranks"])]
    Bv = haar_frame(rng(w["index"], "Bv"), Hkv * d, int(w["value_rank"])).T
    return Bk, Bv


def hybrid_latents(w: dict, b: int, t0: int, t1: int) -> np.ndarray:
    """fp32 latents [C_k,0 | ... | C_k,H_kv-1 | C_v] of sequence b, positions t0..t1-1, each
    latent drawn with the spectrum's leading values as per-channel deviations."""
    L = w["context"]
    parts = [latent_draw(rng(w["index"], f"hk{g}:{b}"), L, spectrum(int(r), w["spectrum_scale"]))
             for g, r in enumerate(w["key_ranks"])]
    parts.append(latent_draw(rng(w["index"], f"hv:{b}"), L,
                             spectrum(int(w["value_rank"]), w["spectrum_scale"])))
    return np.concatenate(parts, axis=1)[t0:t1]


def workload(index: int, **overrides) -> dict:
    """Return a copy of workload ``index`` with optional shape overrides (for reduced-size
    parity cases that keep the structure of the stated workload)."""
    w = dict(WORKLOADS[index])
    w.update(overrides)
    w["index"] = index
    return w


def rng(index: int, stream: str) -> np.random.Generator:
    """Independent PCG64 stream for (workload index, tensor name)."""
    h = hashlib.sha256(f"{index}:{stream}".encode()).digest()
    return np.random.Generator(np.random.PCG64(int.from_bytes(h[:8], "little")))


def spectrum(n: int, scale: float) -> np.ndarray:
    """The stated singular-value profile sigma_i = exp(-i/scale), i = 0..n-1 (0-based)."""
    return np.exp(-np.arange(n, dtype=np.float64) / scale)


def haar_frame(g: np.random.Generator, n: int, k: int) -> np.ndarray:
    """n x k matrix with Haar-distributed orthonormal columns: QR of a Gaussian matrix with
    the signs of diag(R) moved into Q (so the distribution is exactly Haar)."""
    z = g.standard_normal((n, k))
    q, r = np.linalg.qr(z)
    d = np.sign(np.diag(r))
    d[d == 0] = 1.0
    return q * d[None, :]


def gaussian(g: np.random.Generator, shape, dtype=np.float64) -> np.ndarray:
    return g.standard_normal(shape, dtype=dtype)


def latent_draw(g: np.random.Generator, n_tokens: int, stds: np.ndarray) -> np.ndarray:
    """fp32 latents with per-channel standard deviation ``stds`` (channel order as given):
    c[t, i] = fp32(stds[i]) * z[t, i], z ~ N(0, 1) drawn in fp32."""
    z = g.standard_normal((n_tokens, len(stds)), dtype=np.float32)
    return z * np.asarray(stds, dtype=np.float32)[None, :]


def page_permutation(g: np.random.Generator, num_pages: int) -> np.ndarray:
    return g.permutation(num_pages).astype(np.int32)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even to bfloat16, returned as float32 (the storage dtype of inputs
    such as hidden rows and queries).  Input conversion, not part of the method."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    out = (u.astype(np.uint32) << 16).view(np.float32)
    nan = np.isnan(a)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out
