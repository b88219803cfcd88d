"""Oracle side of the synthetic workloads: factors, stored latents and expected decode
outputs, computed with the oracle's own functions from the raw material of the seeded
generator module alone (never from values produced by the CUDA path).

TEST INFRASTRUCTURE, like the rest of this package.
"""
from __future__ import annotations

import functools

import numpy as np

from . import starkv_oracle as O
from rank_quantized_kv_decode_b200 import synth


def tolerance_check(got, want, rel_l2=2e-3, max_abs=1e-2):
    """The parity bar of the decode output against the fp64 oracle."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = got - want
    rl2 = np.linalg.norm(err) / max(np.linalg.norm(want), 1e-30)
    ma = float(np.max(np.abs(err))) if err.size else 0.0
    assert np.all(np.isfinite(got)), "non-finite output"
    assert rl2 <= rel_l2 and ma <= max_abs, f"rel L2 {rl2:.3e} (bar {rel_l2}), max abs {ma:.3e} (bar {max_abs})"
    return rl2, ma


def stored_factor(a, fmt):
    """The factor values the tensor cores see: fp64 -> fp32 -> storage dtype, each nearest."""
    a32 = np.asarray(a, dtype=np.float32)
    if fmt == O.F32:
        return a32.astype(np.float64)
    if fmt == O.BF16:
        return O.bf16_rne(a32).reshape(a32.shape).astype(np.float64)
    return a32.astype(np.float16).astype(np.float64)


class Ref:
    """Oracle setup of one workload (``w`` from synth.workload, possibly with a smaller batch
    or context: the factors depend only on the layer shape)."""

    def __init__(self, w: dict, need_down: bool):
        self.w = w
        idx = w["index"]
        self.need_down = need_down
        Hkv, d, dm = w["n_kv_heads"], w["head_dim"], w["d_model"]
        n = Hkv * d
        m = min(dm, n)
        self.sigma = synth.spectrum(m, w["spectrum_scale"])
        r_k = w["key_rank"]
        # JD keys: W_k = U_k S V_k^T is its own SVD; truncate to r_k
        Vk = synth.haar_frame(synth.rng(idx, "Vk"), n, r_k)
        Uk = synth.haar_frame(synth.rng(idx, "Uk"), dm, r_k) if need_down else np.zeros((dm, r_k))
        Ak, Bk = O.factors_from_svd(Uk, self.sigma[:r_k], Vk, r_k)
        self.Ak, self.Bk = O.canonical_signs(Ak, Bk)
        # HD values: SVD of each KV head's column slice of W_v = U_v S V_v^T
        Vv = synth.haar_frame(synth.rng(idx, "Vv"), n, m)
        Uv = synth.haar_frame(synth.rng(idx, "Uv"), dm, m)
        Wv = (Uv * self.sigma) @ Vv.T
        spectra = O.headwise_spectra(Wv, Hkv, d)
        if w["value_tau"] is not None:
            ranks = [max(1, O.kept_rank(s, w["value_tau"])) for s in spectra]
        else:
            lo, hi = w["value_clip"]
            _, ranks = O.tau_for_mean_rank(spectra, w["value_mean"], lo, hi)
        self.ranks = [int(r) for r in ranks]
        self.Av, self.Bv, self.stds = [], [], []
        for A_g, B_g, s_g in O.headwise_factors(Wv, Hkv, d, self.ranks):
            A_g, B_g = O.canonical_signs(A_g, B_g)
            self.Av.append(A_g)
            self.Bv.append(B_g)
            self.stds.append(s_g[:B_g.shape[0]])
        fmt = w["fmt"]
        self.Bk_s = stored_factor(self.Bk, fmt)
        self.Bv_s = [np.asarray(b, np.float32).astype(np.float64) for b in self.Bv]
        xdt = O.F32 if fmt == O.F32 else O.BF16
        A = np.concatenate([self.Ak] + self.Av, axis=1)
        self.A_s = stored_factor(A, xdt)  # the down-projection in the dtype of x

    # ---- inputs (same synth streams as the workload builder) ----
    def queries(self):
        w = self.w
        q = synth.gaussian(synth.rng(w["index"], "q"), (w["batch"], w["n_q_heads"], w["head_dim"]),
                           np.float32)
        return q if w["fmt"] == O.F32 else synth.bf16_round(q)

    def hidden(self, name, n):
        w = self.w
        x = synth.gaussian(synth.rng(w["index"], name), (n, w["d_model"]), np.float32)
        return x if w["fmt"] == O.F32 else synth.bf16_round(x)

    def drawn_latents(self, b):
        """fp32 latents [K | V_0 | ...] of sequence b, positions 0..context-1."""
        w = self.w
        parts = [synth.latent_draw(synth.rng(w["index"], f"ck:{b}"), w["context"],
                                   self.sigma[:w["key_rank"]])]
        for g, s in enumerate(self.stds):
            parts.append(synth.latent_draw(synth.rng(w["index"], f"cv{g}:{b}"), w["context"], s))
        return np.concatenate(parts, axis=1)

    def projected_latents(self, x):
        """c = x A (fp64, then fp32 as the storage step's input)."""
        return O.project(x, self.A_s).astype(np.float32)

    def sequence_latents(self, b):
        """fp32 latents of sequence b over the whole context, as the workload writes them."""
        w = self.w
        L = w["context"]
        if w["latents_from_x"]:
            lat = self.projected_latents(self.hidden(f"x:{b}", L))
        else:
            lat = self.drawn_latents(b)
        P = w["prefill_tokens"]
        if P and b == 0:
            lat = lat.copy()
            lat[L - P:] = self.projected_latents(self.hidden("prefill", P))
        return lat

    def stored(self, lat):
        """Stored values (fp64) of fp32 latents: (C_k, [C_v,g])."""
        fmt = self.w["fmt"]
        cols = np.concatenate([[0], np.cumsum([self.w["key_rank"]] + self.ranks)])
        out = [O.stored_rows(lat[:, cols[i]:cols[i + 1]], int(cols[i + 1] - cols[i]), fmt)
               for i in range(len(cols) - 1)]
        return out[0], out[1:]

    def expected(self, b, seq_len, heads=None, q=None):
        lat = self.sequence_latents(b)[:seq_len]
        Ck, Cv = self.stored(lat)
        qq = (self.queries() if q is None else q)[b]
        return O.decode_attention(qq, Ck, Cv, self.Bk_s, self.Bv_s, self.w["rope_theta"],
                                  self.w["n_kv_heads"], heads)


    def reshaped(self, **overrides) -> "Ref":
        """The same layer (factors) with other batch / context sizes."""
        r = object.__new__(Ref)
        r.__dict__.update(self.__dict__)
        r.w = dict(self.w, **overrides)
        return r


@functools.lru_cache(maxsize=8)
def _base(index: int, need_down: bool) -> Ref:
    return Ref(synth.workload(index), need_down)


def ref_for(index: int, need_down: bool = False, **overrides) -> Ref:
    return _base(index, need_down).reshaped(**overrides)


class HybridRef:
    """Oracle side of the hybrid workload (keys head-wise, values joint; STAR-KV technical
    summary, Methodology §2): the same seeded factors and latents as the device builder, the
    oracle's own storage step, and decode_attention_hybrid."""

    def __init__(self, **overrides):
        self.w = synth.hybrid_workload(**overrides)
        Bk, Bv = synth.hybrid_factors(self.w)
        # the factor values the tensor cores see: B_k,g as fp16; B_v as fp32
        self.Bk_s = [stored_factor(b, O.MIXED) for b in Bk]
        self.Bv_s = np.asarray(Bv, np.float32).astype(np.float64)

    def queries(self):
        w = self.w
        q = synth.gaussian(synth.rng(w["index"], "q"), (w["batch"], w["n_q_heads"], w["head_dim"]),
                           np.float32)
        return synth.bf16_round(q)

    def stored(self, lat):
        """Stored values (fp64) of fp32 latents [C_k,0 | ... | C_v]: ([C_k,g], C_v)."""
        ranks = list(self.w["key_ranks"]) + [self.w["value_rank"]]
        cols = np.concatenate([[0], np.cumsum(ranks)])
        out = [O.stored_rows(lat[:, cols[i]:cols[i + 1]], int(ranks[i]), self.w["fmt"])
               for i in range(len(ranks))]
        return out[:-1], out[-1]

    def expected(self, b, seq_len, heads=None, q=None):
        if seq_len == 0:
            n = self.w["n_q_heads"] if heads is None else len(heads)
            return np.zeros((n, self.w["head_dim"]))
        lat = synth.hybrid_latents(self.w, b, 0, seq_len)
        Ck, Cv = self.stored(lat)
        qq = (self.queries() if q is None else q)[b]
        return O.decode_attention_hybrid(qq, Ck, Cv, self.Bk_s, self.Bv_s, self.w["rope_theta"],
                                         self.w["n_kv_heads"], heads)
