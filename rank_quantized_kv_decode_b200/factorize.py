"""Offline factorisation of the key/value projections into latent factors (host, fp64).

This is the step that runs once per model before inference (STAR-KV technical summary,
Methodology §1: thresholds on the singular values are converted to hard thresholds offline
and the projection matrices are truncated before inference).  It is not on the decode hot
path; its outputs (A, B and the ranks) are the inputs of the CUDA library.

  keys   (joint decomposition, JD): W_k = U S V^T, A_k = U_r S_r, B_k = V_r^T
  values (head-wise decomposition, HD): the same for each KV head's column slice
  rank at threshold tau: r = #{sigma_i > tau}
"""
from __future__ import annotations

import numpy as np


def rank_at(sigma: np.ndarray, tau: float) -> int:
    return int((np.asarray(sigma) > tau).sum())


def split_factors(U: np.ndarray, s: np.ndarray, Vt: np.ndarray, r: int):
    """A = U_r diag(s_r) (singular values kept unshrunk, all in A), B = V_r^T."""
    return U[:, :r] * s[:r], np.ascontiguousarray(Vt[:r])


def fix_signs(A, B):
    """Make the largest-magnitude entry of every row of B positive, negating the matching
    column of A (A @ B unchanged).  Fixes the SVD's sign freedom, so that a latent channel
    drawn on its own has the same meaning for every caller."""
    rows = np.arange(B.shape[0])
    s = np.sign(B[rows, np.abs(B).argmax(axis=1)])
    s[s == 0] = 1.0
    return (None if A is None else A * s), B * s[:, None]


def truncate(W: np.ndarray, r: int):
    U, s, Vt = np.linalg.svd(W, full_matrices=False)
    A, B = split_factors(U, s, Vt, r)
    return A, B, s


def head_svds(W: np.ndarray, n_kv_heads: int, head_dim: int):
    """(U_g, s_g, Vt_g) of every KV head's column slice of W."""
    return [np.linalg.svd(W[:, g * head_dim:(g + 1) * head_dim], full_matrices=False)
            for g in range(n_kv_heads)]


def ranks_for_target_mean(spectra, lo: int, hi: int, target: float):
    """Per-head ranks clip(#{s_g > tau}, lo, hi) for the threshold tau whose mean clipped
    rank is closest to ``target`` (larger tau on ties).  Sweeps tau downward through the
    pooled singular values, updating the per-head counts incrementally."""
    pooled = sorted(((float(v), g) for g, s in enumerate(spectra) for v in s), reverse=True)
    counts = np.zeros(len(spectra), dtype=np.int64)
    best_err = abs(np.clip(counts, lo, hi).mean() - target)  # tau above every value
    best = np.clip(counts, lo, hi).copy()
    i = 0
    while i < len(pooled):
        v = pooled[i][0]
        # tau = v counts the values strictly above v: evaluate before admitting the values == v
        err = abs(np.clip(counts, lo, hi).mean() - target)
        if err < best_err:
            best_err, best = err, np.clip(counts, lo, hi).copy()
        while i < len(pooled) and pooled[i][0] == v:
            counts[pooled[i][1]] += 1
            i += 1
    err = abs(np.clip(counts, lo, hi).mean() - target)  # tau = 0: everything above zero
    if err < best_err:
        best = np.clip(counts, lo, hi).copy()
    return [int(r) for r in best]
