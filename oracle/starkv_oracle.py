"""fp64 reference ("oracle") of STAR-KV-style low-rank, quantised KV-cache decode.

TEST INFRASTRUCTURE.  Imported only by the test-suite, the smoke check and the
benchmark's CPU-baseline leg.  The CUDA library never calls into it and the two share no
code: the only thing both sides use is the seeded generator module, which holds no
arithmetic of the method.

It is deliberately plain: NumPy in float64 (float32 / float16 exactly where a storage or
quantisation step fixes that precision), one library primitive per step (an SVD, a matmul),
no blocking, no fusion, no split-K.

Sources, cited by page title and section:
  [S1] "STAR-KV: Low-Rank KV Cache Compression via Soft Thresholding for Adaptive Rank
       Control", technical summary (gist.science), Methodology §1 "Adaptive Rank Selection
       via Soft Thresholding" -- thresholds on singular values, converted to hard
       thresholds offline, projection matrices truncated before inference.
  [S2] same page, Methodology §2 "Hybrid Decomposition Strategy" -- Joint Decomposition
       (JD: factor the concatenated heads) and Head-wise Decomposition (HD: factor each head).
  [S3] same page, Methodology §3 "Low-Rank-Aware Mixed-Precision Quantization" -- outlier
       channels are the leading channels in singular-value order; those get more bits.
  [S4] same page, "Key Results" -- 75 % low-rank compression, 20x with 3.2-bit quantisation.
  [AB] the paper's abstract (arXiv 2606.08382 listing) -- latent projection of the KV cache.
  [WL] the stated workload, not the pages: latent storage as fp32, bf16, or int8 (leading
       quarter of the channels) + int4 (rest) with one fp16 scale per 32 channels per token,
       64-token pages, RoPE applied to the reconstructed keys.

Readings where the pages are silent (each is listed again in the design notes):
  * Keys use JD (one latent per token over all KV heads), values use HD (one latent per KV
    head), as the stated workload fixes it; the pages' own assignment is the reverse [S2].
  * The threshold is applied as a hard cut at tau: rank r = #{sigma_i > tau}, the support
    of the soft-threshold prox sigma -> max(sigma - tau, 0); kept singular values are not
    shrunk [S1].  Sigma goes entirely into the down-projection A = U_r Sigma_r, B = V_r^T.
  * Quantiser: symmetric absmax, qmax = 2^(b-1) - 1, fp16 scale = RNE(fp32(amax)/qmax)
    saturated to 65504, code = clamp(rint_half_even(fp32(c) / fp32(scale))), scale 0 gives
    code 0.  Groups of 32 restart where the int4 part starts.  int4 pairs: low nibble is
    the even channel.  int8 channels: the first ceil(r/4).
  * RoPE: half-split (rotate-half) form, theta_j = base^(-2j/d), 0-based positions, the
    decode query at position L-1.  Output fp32-comparable fp64.
  * The pages' own assignment [S2] (keys head-wise, values joint) is decode_attention_hybrid;
    the pages' weight absorption [S2] with per-head values gives each query head its own
    M_h = B_v,g(h) W_o,h (absorb_output_weights, decode_attention_absorbed).
  * The pages' own quantiser [S3] (block-wise Hadamard, 4-bit outliers, 3-bit inliers):
    outlier block = the leading ceil(r/5) channels; each block is rotated by normalised
    Sylvester Hadamard matrices, one per set bit of its size (largest first), the transform
    folded into the factors (A T, T^T B); then the quantiser above with 4 and 3 bits, groups
    of 32 restarting at the block boundary; 3-bit codes packed eight to three bytes, code i
    in bits [3i, 3i+3) of the little-endian 24-bit word, two's complement.
"""
from __future__ import annotations

import math

import numpy as np

F32, BF16, MIXED = "f32", "bf16", "mixed"
HAD43 = "had43"  # the pages' own format: block-wise Hadamard, 4-bit outliers, 3-bit inliers
GROUP = 32


# ======================================================================================
# [S1] rank selection by thresholding singular values
# ======================================================================================
def svt(W: np.ndarray, tau: float) -> np.ndarray:
    """Soft threshold of the singular values, the prox of tau*||X||_*:
    U diag(max(sigma - tau, 0)) V^T  [S1]."""
    U, s, Vt = np.linalg.svd(np.asarray(W, dtype=np.float64), full_matrices=False)
    return (U * np.maximum(s - tau, 0.0)[None, :]) @ Vt


def kept_rank(sigma: np.ndarray, tau: float) -> int:
    """Number of singular values the threshold keeps, #{sigma_i > tau}; this is the rank of
    svt(W, tau) and the rank the offline hard threshold truncates to [S1]."""
    return int(np.count_nonzero(np.asarray(sigma, dtype=np.float64) > tau))


def truncated_factors(W: np.ndarray, r: int):
    """Hard truncation to rank r [S1]: A = U_r Sigma_r (m x r), B = V_r^T (r x n), so that
    A @ B is the best rank-r approximation of W.  Returns (A, B, all singular values)."""
    U, s, Vt = np.linalg.svd(np.asarray(W, dtype=np.float64), full_matrices=False)
    return U[:, :r] * s[None, :r], Vt[:r, :].copy(), s


def factors_from_svd(U: np.ndarray, s: np.ndarray, V: np.ndarray, r: int):
    """The same truncation when the SVD W = U diag(s) V^T is known by construction."""
    return U[:, :r] * s[None, :r], V[:, :r].T.copy()


def canonical_signs(A, B):
    """Fix the sign freedom of each singular pair: row i of B (a right singular vector) is
    negated, together with column i of A, when its entry of largest magnitude is negative.
    A @ B is unchanged; the convention gives a drawn latent channel one meaning."""
    B = np.array(B, dtype=np.float64, copy=True)
    idx = np.argmax(np.abs(B), axis=1)
    flip = np.where(B[np.arange(B.shape[0]), idx] < 0, -1.0, 1.0)
    B *= flip[:, None]
    if A is not None:
        A = np.array(A, dtype=np.float64, copy=True) * flip[None, :]
    return A, B


# ======================================================================================
# [S2] joint and head-wise decompositions
# ======================================================================================
def joint_factors(W: np.ndarray, r: int):
    """JD: factor the concatenated heads W (d_model x H_kv*d) as a whole [S2]."""
    return truncated_factors(W, r)


def head_slice(W: np.ndarray, g: int, head_dim: int) -> np.ndarray:
    return W[:, g * head_dim:(g + 1) * head_dim]


def headwise_spectra(W: np.ndarray, n_heads: int, head_dim: int):
    """Singular values of each head's column slice (HD) [S2]."""
    return [np.linalg.svd(head_slice(W, g, head_dim), compute_uv=False) for g in range(n_heads)]


def headwise_factors(W: np.ndarray, n_heads: int, head_dim: int, ranks):
    """HD: factor each head's slice independently, head g at rank ranks[g] [S2].
    Returns a list of (A_g, B_g, sigma_g)."""
    return [truncated_factors(head_slice(W, g, head_dim), int(ranks[g])) for g in range(n_heads)]


def tau_for_mean_rank(spectra, target_mean: float, lo: int, hi: int):
    """Threshold tau whose clipped kept ranks clip(#{s_g > tau}, lo, hi) have a mean closest
    to ``target_mean``; on a tie the larger tau wins.  The mean is a step function of tau
    that only changes at singular values, so every breakpoint (each distinct singular value,
    and 0) is tried, from the largest down.  Returns (tau, ranks)."""
    sorted_s = [np.sort(np.asarray(s, dtype=np.float64)) for s in spectra]
    cands = np.unique(np.concatenate(sorted_s))[::-1]
    cands = np.append(cands, 0.0)
    best = None
    best_err = math.inf
    for tau in cands:
        ranks = np.array([len(s) - np.searchsorted(s, tau, side="right") for s in sorted_s])
        clipped = np.clip(ranks, lo, hi)
        err = abs(float(clipped.mean()) - target_mean)
        if err < best_err:
            best_err = err
            best = (float(tau), clipped.astype(np.int64))
    return best


# ======================================================================================
# [WL] page layout of the latent cache
# ======================================================================================
def mixed_split(r: int) -> dict:
    """int8 channels [0, n8) and int4 channels [n8, r) of a rank-r latent, in singular-value
    order (leading channels carry the outliers [S3]); one fp16 scale per group of 32."""
    n8 = -(-r // 4)
    n4 = r - n8
    return dict(n8=n8, n4=n4, g8=-(-n8 // GROUP), g4=-(-n4 // GROUP), nb4=-(-n4 // 2))


def _align16(x: int) -> int:
    return (x + 15) // 16 * 16


def page_layout(fmt: str, key_rank: int, value_ranks, page_tokens: int = 64) -> dict:
    """Byte layout of one page of ``page_tokens`` tokens.  Latents in order K, V_0 .. V_{H-1};
    for each latent its blocks are stored token-major ([token][channel]):
      f32:   values  (4 B/channel)
      bf16:  values  (2 B/channel)
      mixed: int8 codes (n8 B) | packed int4 codes (nb4 B) | fp16 scales (2*(g8+g4) B)
      had43: packed 4-bit codes (nb_hi B) | packed 3-bit codes (nb_lo B) | fp16 scales
             (2*(g_hi+g_lo) B), for latents of factors rotated by rotate_factors [S3]
    Every block starts on a 16-byte boundary."""
    ranks = [int(key_rank)] + [int(r) for r in value_ranks]
    off = 0
    segs = []
    token_bytes = 0

    def place(nbytes):
        nonlocal off
        o = off
        off = _align16(off + nbytes)
        return o

    for r in ranks:
        s = dict(rank=r)
        if fmt == F32:
            s["plain"] = place(page_tokens * r * 4)
            s["pitch"] = r * 4
            token_bytes += r * 4
        elif fmt == BF16:
            s["plain"] = place(page_tokens * r * 2)
            s["pitch"] = r * 2
            token_bytes += r * 2
        elif fmt == MIXED:
            sp = mixed_split(r)
            s.update(sp)
            s["i8"] = place(page_tokens * sp["n8"])
            s["i4"] = place(page_tokens * sp["nb4"])
            s["sc"] = place(page_tokens * 2 * (sp["g8"] + sp["g4"]))
            token_bytes += sp["n8"] + sp["nb4"] + 2 * (sp["g8"] + sp["g4"])
        elif fmt == HAD43:
            sp = hadamard_split(r)
            s.update(sp)
            s["nb_hi"] = -(-sp["n_hi"] // 2)
            s["nb_lo"] = 3 * -(-sp["n_lo"] // 8)
            s["hi"] = place(page_tokens * s["nb_hi"])
            s["lo"] = place(page_tokens * s["nb_lo"])
            s["sc"] = place(page_tokens * 2 * (sp["g_hi"] + sp["g_lo"]))
            token_bytes += s["nb_hi"] + s["nb_lo"] + 2 * (sp["g_hi"] + sp["g_lo"])
        else:
            raise ValueError(fmt)
        segs.append(s)
    return dict(fmt=fmt, page_tokens=page_tokens, segs=segs, page_bytes=off,
                token_bytes=token_bytes, key_rank=int(key_rank),
                value_ranks=[int(r) for r in value_ranks])


def hybrid_page_layout(fmt: str, key_ranks, value_rank: int, page_tokens: int = 64) -> dict:
    """Byte layout of a page with the hybrid assignment (STAR-KV technical summary,
    Methodology §2: keys head-wise, values joint): the key latents of KV heads 0..H_kv-1, then
    the joint value latent, each placed exactly as page_layout places a latent of its rank."""
    ranks = [int(r) for r in key_ranks] + [int(value_rank)]
    return page_layout(fmt, ranks[0], ranks[1:], page_tokens)


def mixed_bits_per_channel(r: int) -> float:
    """Average stored bits per latent channel of the int8/int4 + fp16-scale format."""
    sp = mixed_split(r)
    return 8.0 * (sp["n8"] + sp["nb4"] + 2 * (sp["g8"] + sp["g4"])) / r


def two_level_bits(outlier_fraction: float, hi_bits: int, lo_bits: int) -> float:
    """Average bits of a two-level mixed precision split, scales not counted [S3]."""
    return outlier_fraction * hi_bits + (1.0 - outlier_fraction) * lo_bits


def total_reduction(kept_fraction: float, avg_bits: float, base_bits: int = 16) -> float:
    """Overall KV-cache size reduction of low-rank projection followed by quantisation [S4]."""
    return (1.0 / kept_fraction) * (base_bits / avg_bits)


# ======================================================================================
# [S3]/[WL] quantisation and packing
# ======================================================================================
def fp16_scale(amax, qmax) -> np.float16:
    """fp16 scale of a group: round-to-nearest-even of the fp32 quotient amax/qmax,
    saturated to the largest finite fp16."""
    s32 = np.float32(amax) / np.float32(qmax)
    with np.errstate(over="ignore"):
        s16 = np.float16(s32)
    if not np.isfinite(s16):
        s16 = np.float16(65504.0)
    return s16


def quantize_group(c, bits: int):
    """Symmetric absmax quantisation of one group of fp32 values.
    Returns (fp16 scale, int8 array of codes in [-qmax, qmax])."""
    c = np.asarray(c, dtype=np.float32)
    qmax = (1 << (bits - 1)) - 1
    amax = np.max(np.abs(c)) if c.size else np.float32(0.0)
    s16 = fp16_scale(amax, qmax)
    s = np.float32(s16)
    if s == 0:
        return s16, np.zeros(c.shape, dtype=np.int8)
    r = c / s  # float32 / float32: IEEE round-to-nearest
    q = np.clip(np.rint(r), -qmax, qmax)  # rint: half to even
    return s16, q.astype(np.int8)


def quantize_latent(c, r: int):
    """One token's rank-r latent (fp32, singular-value order) -> (int8 codes [n8],
    int4 codes [n4] as int8 values in [-7, 7], fp16 scales [g8 + g4])."""
    c = np.asarray(c, dtype=np.float32)
    assert c.shape == (r,)
    sp = mixed_split(r)
    n8, n4 = sp["n8"], sp["n4"]
    scales, q8, q4 = [], [], []
    for gi in range(sp["g8"]):
        s, q = quantize_group(c[gi * GROUP:min((gi + 1) * GROUP, n8)], 8)
        scales.append(s)
        q8.append(q)
    for gi in range(sp["g4"]):
        s, q = quantize_group(c[n8 + gi * GROUP:n8 + min((gi + 1) * GROUP, n4)], 4)
        scales.append(s)
        q4.append(q)
    q8 = np.concatenate(q8) if q8 else np.zeros(0, np.int8)
    q4 = np.concatenate(q4) if q4 else np.zeros(0, np.int8)
    return q8, q4, np.array(scales, dtype=np.float16)


# ======================================================================================
# [S3] the pages' own format: block-wise Hadamard rotation, 4-bit / 3-bit
# ======================================================================================
def sylvester_hadamard(n: int) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix of order n (a power of two): entries +-1/sqrt(n),
    H H^T = I."""
    assert n >= 1 and n & (n - 1) == 0
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H / math.sqrt(n)


def block_hadamard(n: int) -> np.ndarray:
    """Orthogonal n x n transform for a block of n channels: normalised Sylvester blocks down
    the diagonal, one per set bit of n, largest first."""
    T = np.zeros((n, n))
    at = 0
    for k in reversed(range(max(n.bit_length(), 1))):
        size = 1 << k
        if n & size:
            T[at:at + size, at:at + size] = sylvester_hadamard(size)
            at += size
    return T


def hadamard_split(r: int) -> dict:
    """Outlier block [0, n_hi) -- the leading fifth of the channels in singular-value order,
    rounded up -- and inlier block [n_hi, r) [S3]."""
    n_hi = -(-r // 5)
    n_lo = r - n_hi
    return dict(n_hi=n_hi, n_lo=n_lo, g_hi=-(-n_hi // GROUP), g_lo=-(-n_lo // GROUP))


def hadamard_transform(r: int) -> np.ndarray:
    """The block-wise transform of a rank-r latent: independent rotations of the outlier and
    the inlier block [S3]."""
    sp = hadamard_split(r)
    T = np.zeros((r, r))
    T[:sp["n_hi"], :sp["n_hi"]] = block_hadamard(sp["n_hi"])
    T[sp["n_hi"]:, sp["n_hi"]:] = block_hadamard(sp["n_lo"])
    return T


def rotate_factors(A, B):
    """Fold the transform into the factors ("zero overhead" [S3]): A' = A T, B' = T^T B, so
    A' B' = A B and the latents x A' are the rotated latents."""
    A = np.asarray(A, np.float64)
    T = hadamard_transform(A.shape[1])
    return A @ T, T.T @ np.asarray(B, np.float64)


def quantize_hadamard_latent(c, r: int):
    """One token's rotated rank-r latent (fp32) -> (4-bit codes of the outlier block, 3-bit
    codes of the inlier block, fp16 scales [g_hi + g_lo]) [S3]."""
    c = np.asarray(c, dtype=np.float32)
    assert c.shape == (r,)
    sp = hadamard_split(r)
    n_hi, n_lo = sp["n_hi"], sp["n_lo"]
    scales, qh, ql = [], [], []
    for gi in range(sp["g_hi"]):
        s, q = quantize_group(c[gi * GROUP:min((gi + 1) * GROUP, n_hi)], 4)
        scales.append(s)
        qh.append(q)
    for gi in range(sp["g_lo"]):
        s, q = quantize_group(c[n_hi + gi * GROUP:n_hi + min((gi + 1) * GROUP, n_lo)], 3)
        scales.append(s)
        ql.append(q)
    qh = np.concatenate(qh) if qh else np.zeros(0, np.int8)
    ql = np.concatenate(ql) if ql else np.zeros(0, np.int8)
    return qh, ql, np.array(scales, dtype=np.float16)


def dequantize_hadamard_latent(qh, ql, scales, r: int) -> np.ndarray:
    """Codes times their group's fp16 scale (exact in fp32), in channel order."""
    sp = hadamard_split(r)
    out = np.zeros(r, np.float64)
    for i in range(sp["n_hi"]):
        out[i] = np.float64(scales[i // GROUP]) * int(qh[i])
    for j in range(sp["n_lo"]):
        out[sp["n_hi"] + j] = np.float64(scales[sp["g_hi"] + j // GROUP]) * int(ql[j])
    return out


def pack_int3(codes) -> np.ndarray:
    """3-bit two's-complement codes in [-4, 3], eight per three bytes: code i of a group of
    eight in bits [3i, 3i+3) of a little-endian 24-bit word; a short tail is padded with 0."""
    codes = np.asarray(codes, dtype=np.int64)
    assert codes.size == 0 or (codes.min() >= -4 and codes.max() <= 3)
    n = codes.size
    padded = np.zeros(-(-n // 8) * 8, np.int64)
    padded[:n] = codes
    out = []
    for k in range(0, padded.size, 8):
        word = 0
        for i in range(8):
            word |= (int(padded[k + i]) & 7) << (3 * i)
        out += [word & 0xFF, (word >> 8) & 0xFF, (word >> 16) & 0xFF]
    return np.array(out, dtype=np.uint8)


def unpack_int3(packed, n: int) -> np.ndarray:
    """Inverse of pack_int3: the first n codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = []
    for k in range(0, packed.size, 3):
        word = int(packed[k]) | (int(packed[k + 1]) << 8) | (int(packed[k + 2]) << 16)
        for i in range(8):
            v = (word >> (3 * i)) & 7
            out.append(v - 8 if v >= 4 else v)
    return np.array(out[:n], dtype=np.int8)


def pack_int4(codes) -> np.ndarray:
    """Two 4-bit two's-complement codes per byte; channel 2i in the low nibble, 2i+1 in the
    high nibble; an odd count leaves the last high nibble 0."""
    codes = np.asarray(codes, dtype=np.int64)
    out = np.zeros(-(-len(codes) // 2), dtype=np.uint8)
    for i, v in enumerate(codes):
        nib = int(v) & 0xF
        if i % 2 == 0:
            out[i // 2] |= nib
        else:
            out[i // 2] |= nib << 4
    return out


def unpack_int4(packed, n: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.zeros(n, dtype=np.int8)
    for i in range(n):
        b = int(packed[i // 2])
        nib = (b >> 4) & 0xF if i % 2 else b & 0xF
        out[i] = nib - 16 if nib >= 8 else nib
    return out


def dequantize_latent(q8, q4, scales, r: int) -> np.ndarray:
    """c_hat = scale * code per channel; exact in fp32 and fp64 (11-bit x 8-bit products)."""
    sp = mixed_split(r)
    n8 = sp["n8"]
    out = np.zeros(r, dtype=np.float64)
    for i in range(n8):
        out[i] = float(scales[i // GROUP]) * int(q8[i])
    for i in range(sp["n4"]):
        out[n8 + i] = float(scales[sp["g8"] + i // GROUP]) * int(q4[i])
    return out


def bf16_rne(a) -> np.ndarray:
    """Round fp32 values to bfloat16 (nearest, ties to even); returned as fp32."""
    a = np.atleast_1d(np.asarray(a, dtype=np.float32))
    bits = a.view(np.uint32).astype(np.uint64)
    keep = bits >> 16
    rem = bits & 0xFFFF
    up = (rem > 0x8000) | ((rem == 0x8000) & ((keep & 1) == 1))
    keep = keep + up.astype(np.uint64)
    return (keep.astype(np.uint32) << 16).view(np.float32)


# ---- one token in a page ----------------------------------------------------------------
def encode_token(page: np.ndarray, layout: dict, li: int, slot: int, c) -> None:
    """Store latent ``li`` (0 = K, 1+g = V_g) of one token at ``slot`` of ``page`` (uint8)."""
    seg = layout["segs"][li]
    r = seg["rank"]
    c = np.asarray(c, dtype=np.float32)
    fmt = layout["fmt"]
    if fmt == F32:
        o = seg["plain"] + slot * seg["pitch"]
        page[o:o + 4 * r] = c.view(np.uint8)
    elif fmt == BF16:
        o = seg["plain"] + slot * seg["pitch"]
        hi = (bf16_rne(c).view(np.uint32) >> 16).astype(np.uint16)
        page[o:o + 2 * r] = hi.view(np.uint8)
    elif fmt == HAD43:
        qh, ql, sc = quantize_hadamard_latent(c, r)
        o = seg["hi"] + slot * seg["nb_hi"]
        page[o:o + seg["nb_hi"]] = pack_int4(qh)
        o = seg["lo"] + slot * seg["nb_lo"]
        page[o:o + seg["nb_lo"]] = pack_int3(ql)
        ns = seg["g_hi"] + seg["g_lo"]
        o = seg["sc"] + slot * 2 * ns
        page[o:o + 2 * ns] = sc.view(np.uint8)
    else:
        q8, q4, sc = quantize_latent(c, r)
        o = seg["i8"] + slot * seg["n8"]
        page[o:o + seg["n8"]] = q8.view(np.uint8)
        o = seg["i4"] + slot * seg["nb4"]
        page[o:o + seg["nb4"]] = pack_int4(q4)
        ns = seg["g8"] + seg["g4"]
        o = seg["sc"] + slot * 2 * ns
        page[o:o + 2 * ns] = sc.view(np.uint8)


def decode_token(page: np.ndarray, layout: dict, li: int, slot: int) -> np.ndarray:
    """The stored value of latent ``li`` at ``slot`` as fp64 (dequantised for mixed)."""
    seg = layout["segs"][li]
    r = seg["rank"]
    fmt = layout["fmt"]
    if fmt == F32:
        o = seg["plain"] + slot * seg["pitch"]
        return page[o:o + 4 * r].copy().view(np.float32).astype(np.float64)
    if fmt == BF16:
        o = seg["plain"] + slot * seg["pitch"]
        hi = page[o:o + 2 * r].copy().view(np.uint16).astype(np.uint32) << 16
        return hi.view(np.float32).astype(np.float64)
    if fmt == HAD43:
        o = seg["hi"] + slot * seg["nb_hi"]
        qh = unpack_int4(page[o:o + seg["nb_hi"]], seg["n_hi"])
        o = seg["lo"] + slot * seg["nb_lo"]
        ql = unpack_int3(page[o:o + seg["nb_lo"]], seg["n_lo"])
        ns = seg["g_hi"] + seg["g_lo"]
        o = seg["sc"] + slot * 2 * ns
        sc = page[o:o + 2 * ns].copy().view(np.float16)
        return dequantize_hadamard_latent(qh, ql, sc, r)
    o = seg["i8"] + slot * seg["n8"]
    q8 = page[o:o + seg["n8"]].copy().view(np.int8)
    o = seg["i4"] + slot * seg["nb4"]
    q4 = unpack_int4(page[o:o + seg["nb4"]], seg["n4"])
    ns = seg["g8"] + seg["g4"]
    o = seg["sc"] + slot * 2 * ns
    sc = page[o:o + 2 * ns].copy().view(np.float16)
    return dequantize_latent(q8, q4, sc, r)


def encode_tokens(cache: np.ndarray, layout: dict, block_table: np.ndarray, tok_seq, tok_pos,
                  latents: np.ndarray) -> None:
    """Write rows of concatenated latents [K | V_0 | ...] (fp32) into a cache viewed as
    (num_pages, page_bytes) uint8; token (b, p) lives at page block_table[b, p // P],
    slot p % P."""
    P = layout["page_tokens"]
    ranks = [s["rank"] for s in layout["segs"]]
    cols = np.concatenate([[0], np.cumsum(ranks)])
    for n in range(latents.shape[0]):
        b, p = int(tok_seq[n]), int(tok_pos[n])
        page = cache[int(block_table[b, p // P])]
        for li in range(len(ranks)):
            encode_token(page, layout, li, p % P, latents[n, cols[li]:cols[li + 1]])


def read_sequence(cache: np.ndarray, layout: dict, table_row, L: int):
    """Stored latents of positions 0..L-1 of one sequence, as fp64:
    (C_k [L x r_k], [C_v,g [L x r_g] for each KV head g])."""
    P = layout["page_tokens"]
    n_lat = len(layout["segs"])
    out = [np.zeros((L, s["rank"])) for s in layout["segs"]]
    for t in range(L):
        page = cache[int(table_row[t // P])]
        for li in range(n_lat):
            out[li][t] = decode_token(page, layout, li, t % P)
    return out[0], out[1:]


def store_latents(latents, fmt: str) -> np.ndarray:
    """Element-wise storage rounding of fp32 latents for the unquantised formats (fp64 out)."""
    latents = np.asarray(latents, dtype=np.float32)
    if fmt == F32:
        return latents.astype(np.float64)
    if fmt == BF16:
        return bf16_rne(latents).reshape(latents.shape).astype(np.float64)
    raise ValueError(fmt)


# ======================================================================================
# [WL] rotary position embedding, applied after reconstruction
# ======================================================================================
def rope_inv_freq(theta: float, d: int) -> np.ndarray:
    j = np.arange(d // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * j / d)


def apply_rope(v: np.ndarray, pos, theta: float) -> np.ndarray:
    """Half-split rotation: for j < d/2 the pair (v_j, v_{j+d/2}) is rotated by the angle
    pos * theta^(-2j/d)."""
    v = np.asarray(v, dtype=np.float64)
    d = v.shape[-1]
    h = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(theta, d)
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(v)
    out[..., :h] = v[..., :h] * c - v[..., h:] * s
    out[..., h:] = v[..., h:] * c + v[..., :h] * s
    return out


# ======================================================================================
# decode attention read from the latents [AB][S2]
# ======================================================================================
def reconstruct_keys(C_k: np.ndarray, B_k: np.ndarray) -> np.ndarray:
    """K = C_k B_k (JD keys: one latent per token, B_k spans all KV heads)."""
    return np.asarray(C_k, np.float64) @ np.asarray(B_k, np.float64)


def latent_attention(q, C_k, C_v, B_k, theta: float, n_kv_heads: int, heads=None):
    """Single-token decode attention of one sequence in the latent space of the values.

    q   : (H, d) query of the token at position L-1, before RoPE.
    C_k : (L, r_k) key latents;  C_v: list over KV heads g of (L, r_g) value latents.
    B_k : (r_k, H_kv*d).
    Steps: K = C_k B_k; per head g(h) = h // (H/H_kv): RoPE on K_g at positions 0..L-1 and
    on q_h at L-1; scores q'.k'/sqrt(d); softmax (max subtracted, fp64); a_h = p C_v,g.
    Returns the list of a_h (each (r_g(h),)) for ``heads`` (default: all, in order)."""
    q = np.asarray(q, dtype=np.float64)
    H, d = q.shape
    G = H // n_kv_heads
    L = C_k.shape[0]
    heads = range(H) if heads is None else heads
    pos = np.arange(L)
    out = []
    cache_k = {}
    for h in heads:
        g = h // G
        if g not in cache_k:
            Bg = np.asarray(B_k, np.float64)[:, g * d:(g + 1) * d]
            cache_k[g] = apply_rope(np.asarray(C_k, np.float64) @ Bg, pos, theta)
        Kg = cache_k[g]
        qh = apply_rope(q[h], L - 1, theta)
        s = Kg @ qh / math.sqrt(d)
        s = s - s.max()
        p = np.exp(s)
        p = p / p.sum()
        out.append(p @ np.asarray(C_v[g], np.float64))
    return out


def tile_partials(q, C_k, C_v, B_k, theta: float, n_kv_heads: int, tile: int = 128, heads=None):
    """The split-K view of latent_attention: per query head h and per block of ``tile``
    consecutive positions [t0, t0 + tile), the block's largest score in log2 units
    m = max_t s_t log2(e), its weight sum l = sum_t 2^(s_t log2(e) - m) and its unnormalised
    latent sum a = sum_t 2^(s_t log2(e) - m) c_v,g(h),t, with s_t = q'.k'_t/sqrt(d) as in
    latent_attention.  The exact merge of the blocks (log-sum-exp) is latent_attention's a_h:
    a_h = sum_b 2^(m_b - M) a_b / sum_b 2^(m_b - M) l_b, M = max_b m_b.
    Returns, for each head of ``heads`` (default all), a list over blocks of (m, l, a)."""
    q = np.asarray(q, dtype=np.float64)
    H, d = q.shape
    G = H // n_kv_heads
    L = C_k.shape[0]
    heads = range(H) if heads is None else heads
    pos = np.arange(L)
    log2e = 1.0 / math.log(2.0)
    out = []
    cache_k = {}
    for h in heads:
        g = h // G
        if g not in cache_k:
            Bg = np.asarray(B_k, np.float64)[:, g * d:(g + 1) * d]
            cache_k[g] = apply_rope(np.asarray(C_k, np.float64) @ Bg, pos, theta)
        s = cache_k[g] @ apply_rope(q[h], L - 1, theta) / math.sqrt(d) * log2e
        Cv = np.asarray(C_v[g], np.float64)
        blocks = []
        for t0 in range(0, L, tile):
            sb = s[t0:t0 + tile]
            m = sb.max()
            w = np.power(2.0, sb - m)
            blocks.append((m, w.sum(), w @ Cv[t0:t0 + tile]))
        out.append(blocks)
    return out


def decode_attention(q, C_k, C_v, B_k, B_v, theta: float, n_kv_heads: int, heads=None):
    """Single-token decode attention of one sequence from its stored latents: the latent
    outputs a_h of latent_attention, up-projected o_h = a_h B_v,g(h) (B_v: list over g of
    (r_g, d)).  Returns (H, d), or only ``heads`` rows (in that order) when given."""
    H = np.asarray(q).shape[0]
    G = H // n_kv_heads
    heads = list(range(H)) if heads is None else list(heads)
    a = latent_attention(q, C_k, C_v, B_k, theta, n_kv_heads, heads)
    return np.array([a_h @ np.asarray(B_v[h // G], np.float64) for a_h, h in zip(a, heads)])


def absorb_output_weights(B_v, W_o, n_q_heads: int) -> list:
    """Weight absorption (STAR-KV technical summary, Methodology §2: the value up-projection
    is folded into the attention output projection, so values are never reconstructed): for
    each query head h, M_h = B_v,g(h) W_o,h with W_o,h the rows [h d, (h+1) d) of W_o
    (H d x d_out).  Returns the list of M_h, each (r_g(h), d_out)."""
    W_o = np.asarray(W_o, np.float64)
    n_kv = len(B_v)
    G = n_q_heads // n_kv
    d = np.asarray(B_v[0]).shape[1]
    return [np.asarray(B_v[h // G], np.float64) @ W_o[h * d:(h + 1) * d] for h in range(n_q_heads)]


def decode_attention_absorbed(q, C_k, C_v, B_k, M, theta: float, n_kv_heads: int) -> np.ndarray:
    """The attention block's output for the decoded token with absorbed weights:
    y = sum_h a_h M_h (a_h from latent_attention, M_h from absorb_output_weights), i.e.
    (concat_h o_h) W_o without forming o.  Returns (d_out,)."""
    a = latent_attention(q, C_k, C_v, B_k, theta, n_kv_heads)
    return np.sum([a_h @ M_h for a_h, M_h in zip(a, M)], axis=0)


def decode_attention_hybrid(q, C_k, C_v, B_k, B_v, theta: float, n_kv_heads: int, heads=None):
    """Decode attention with the pages' own assignment (STAR-KV technical summary,
    Methodology §2 "Hybrid Decomposition Strategy": keys head-wise, values joint).

    q   : (H, d) query of the token at position L-1, before RoPE.
    C_k : list over KV heads g of (L, r_k,g) key latents;  B_k: list over g of (r_k,g, d).
    C_v : (L, r_v) joint value latents;  B_v: (r_v, H_kv*d).
    Steps: K_g = C_k,g B_k,g; RoPE on K_g at positions 0..L-1 and on q_h at L-1; scores
    q'.k'/sqrt(d); softmax (max subtracted, fp64); a_h = p C_v in the joint latent space
    (r_v values, the same space for every head); o_h = a_h B_v[:, g(h) d:(g(h)+1) d].
    Returns (H, d), or only ``heads`` rows (in that order) when given."""
    q = np.asarray(q, dtype=np.float64)
    H, d = q.shape
    G = H // n_kv_heads
    L = np.asarray(C_v).shape[0]
    heads = range(H) if heads is None else heads
    pos = np.arange(L)
    Cv = np.asarray(C_v, np.float64)
    Bv = np.asarray(B_v, np.float64)
    out = []
    cache_k = {}
    for h in heads:
        g = h // G
        if g not in cache_k:
            cache_k[g] = apply_rope(np.asarray(C_k[g], np.float64) @ np.asarray(B_k[g], np.float64),
                                    pos, theta)
        s = cache_k[g] @ apply_rope(q[h], L - 1, theta) / math.sqrt(d)
        s = s - s.max()
        p = np.exp(s)
        p = p / p.sum()
        out.append((p @ Cv) @ Bv[:, g * d:(g + 1) * d])
    return np.array(out)


def project(x, A) -> np.ndarray:
    """Latent write of new tokens: c = x A, with A = [A_k | A_v,0 | A_v,1 | ...] [AB]."""
    return np.asarray(x, np.float64) @ np.asarray(A, np.float64)


# ======================================================================================
# the same quantiser over many tokens at once (NumPy vector form of quantize_latent /
# dequantize_latent; pinned against the per-token definitions by the tests)
# ======================================================================================
def _quantize_block(C: np.ndarray, bits: int):
    """C: (n, k) fp32 group members (k <= 32).  Returns fp16 scales (n,), codes (n, k)."""
    qmax = np.float32((1 << (bits - 1)) - 1)
    amax = np.max(np.abs(C), axis=1) if C.shape[1] else np.zeros(C.shape[0], np.float32)
    with np.errstate(over="ignore"):
        s16 = (amax.astype(np.float32) / qmax).astype(np.float16)
    s16 = np.where(np.isfinite(s16), s16, np.float16(65504.0)).astype(np.float16)
    s = s16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = C / s[:, None]
    q = np.clip(np.rint(r), -qmax, qmax)
    q = np.where(s[:, None] == 0, 0, q)
    return s16, q.astype(np.int8)


def quantize_rows(C, r: int):
    """quantize_latent for every row of C (n, r) fp32: (q8 (n, n8), q4 (n, n4), scales (n, ng))."""
    C = np.asarray(C, dtype=np.float32)
    sp = mixed_split(r)
    n8, n4 = sp["n8"], sp["n4"]
    scales, q8, q4 = [], [], []
    for gi in range(sp["g8"]):
        s, q = _quantize_block(C[:, gi * GROUP:min((gi + 1) * GROUP, n8)], 8)
        scales.append(s)
        q8.append(q)
    for gi in range(sp["g4"]):
        s, q = _quantize_block(C[:, n8 + gi * GROUP:n8 + min((gi + 1) * GROUP, n4)], 4)
        scales.append(s)
        q4.append(q)
    n = C.shape[0]
    q8 = np.concatenate(q8, axis=1) if q8 else np.zeros((n, 0), np.int8)
    q4 = np.concatenate(q4, axis=1) if q4 else np.zeros((n, 0), np.int8)
    return q8, q4, np.stack(scales, axis=1)


def dequantize_rows(q8, q4, scales, r: int) -> np.ndarray:
    sp = mixed_split(r)
    s8 = np.repeat(scales[:, :sp["g8"]].astype(np.float64), GROUP, axis=1)[:, :sp["n8"]]
    s4 = np.repeat(scales[:, sp["g8"]:].astype(np.float64), GROUP, axis=1)[:, :sp["n4"]]
    return np.concatenate([s8 * q8, s4 * q4], axis=1)


def quantize_hadamard_rows(C, r: int):
    """quantize_hadamard_latent for every row of C (n, r) fp32 (rotated latents):
    (4-bit codes (n, n_hi), 3-bit codes (n, n_lo), scales (n, g_hi + g_lo))."""
    C = np.asarray(C, dtype=np.float32)
    sp = hadamard_split(r)
    n_hi, n_lo = sp["n_hi"], sp["n_lo"]
    scales, qh, ql = [], [], []
    for gi in range(sp["g_hi"]):
        s, q = _quantize_block(C[:, gi * GROUP:min((gi + 1) * GROUP, n_hi)], 4)
        scales.append(s)
        qh.append(q)
    for gi in range(sp["g_lo"]):
        s, q = _quantize_block(C[:, n_hi + gi * GROUP:n_hi + min((gi + 1) * GROUP, n_lo)], 3)
        scales.append(s)
        ql.append(q)
    n = C.shape[0]
    qh = np.concatenate(qh, axis=1) if qh else np.zeros((n, 0), np.int8)
    ql = np.concatenate(ql, axis=1) if ql else np.zeros((n, 0), np.int8)
    return qh, ql, np.stack(scales, axis=1)


def dequantize_hadamard_rows(qh, ql, scales, r: int) -> np.ndarray:
    sp = hadamard_split(r)
    sh = np.repeat(scales[:, :sp["g_hi"]].astype(np.float64), GROUP, axis=1)[:, :sp["n_hi"]]
    sl = np.repeat(scales[:, sp["g_hi"]:].astype(np.float64), GROUP, axis=1)[:, :sp["n_lo"]]
    return np.concatenate([sh * qh, sl * ql], axis=1)


def stored_rows(C, r: int, fmt: str) -> np.ndarray:
    """Stored value (fp64) of every row of C (n, r) fp32 in format ``fmt``."""
    if fmt == MIXED:
        return dequantize_rows(*quantize_rows(C, r), r)
    if fmt == HAD43:
        return dequantize_hadamard_rows(*quantize_hadamard_rows(C, r), r)
    return store_latents(C, fmt)
