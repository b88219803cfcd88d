"""ctypes mirror of include/starkv.h and the loader of ``libstarkv.so``.

Loading fails loudly: there is no fallback path.  Build the library with
``python -m rank_quantized_kv_decode_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

MAX_KV_HEADS = 64
GROUP = 32
TILE_TOKENS = 128

FMT = {"f32": 0, "bf16": 1, "mixed": 2, "had43": 3}
ASSIGN_JOINT_KEYS, ASSIGN_HYBRID = 0, 1

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_WORKSPACE = 0, 1, 2, 3, 4
DEV_BOUNDS, DEV_TIMEOUT = 1, 2

i32, i64, f64, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
vp = ctypes.c_void_p


class Config(ctypes.Structure):
    _fields_ = [("n_q_heads", i32), ("n_kv_heads", i32), ("head_dim", i32), ("d_model", i32),
                ("key_rank", i32), ("value_rank", i32 * MAX_KV_HEADS), ("fmt", i32),
                ("page_tokens", i32), ("rope_theta", f64)]


class HybridConfig(ctypes.Structure):
    _fields_ = [("n_q_heads", i32), ("n_kv_heads", i32), ("head_dim", i32), ("d_model", i32),
                ("key_rank", i32 * MAX_KV_HEADS), ("value_rank", i32), ("fmt", i32),
                ("page_tokens", i32), ("rope_theta", f64)]


class Segment(ctypes.Structure):
    _fields_ = [("rank", i32), ("col", i32), ("n8", i32), ("n4", i32), ("g8", i32), ("g4", i32),
                ("nb4", i32), ("pitch", i32), ("off_plain", i64), ("off_i8", i64),
                ("off_i4", i64), ("off_sc", i64)]


class Layout(ctypes.Structure):
    _fields_ = [("cfg", Config), ("n_latents", i32), ("proj_cols", i32),
                ("value_rank_total", i32), ("value_rank_max", i32), ("page_bytes", i64),
                ("token_bytes", i64), ("seg", Segment * (1 + MAX_KV_HEADS)),
                ("assignment", i32), ("reserved", i32), ("hybrid", HybridConfig)]


class Sizes(ctypes.Structure):
    _fields_ = [("cache_bytes", sz), ("rope_table_bytes", sz), ("decode_workspace_bytes", sz),
                ("append_workspace_bytes", sz)]


class DecodeOpts(ctypes.Structure):
    _fields_ = [("max_ctas", i32), ("n_ranges", i32), ("timeout_ms", i32), ("cta_group", i32)]


class DecodePlan(ctypes.Structure):
    _fields_ = [("cta_group", i32), ("key_mode", i32), ("chunk_cols", i32), ("n_chunks", i32),
                ("n_ranges", i32), ("stages", i32), ("value_buffers", i32), ("smem_bytes", i32),
                ("grid", i32), ("work_units", i32)]


EXPORTS = {
    "starkv_layout_init": (i32, [ctypes.POINTER(Config), ctypes.POINTER(Layout)]),
    "starkv_hybrid_layout_init": (i32, [ctypes.POINTER(HybridConfig), ctypes.POINTER(Layout)]),
    "starkv_hybrid_decode": (i32, [ctypes.POINTER(Layout), vp, vp, i64, vp, i32, vp, i32, vp, vp,
                                   vp, sz, vp, vp, sz, vp, vp]),
    "starkv_alloc": (i32, [ctypes.POINTER(Layout), i64, i32, i32, i32, ctypes.POINTER(Sizes)]),
    "starkv_rope_init": (i32, [ctypes.POINTER(Layout), i32, vp, sz, vp]),
    "starkv_quant_pack": (i32, [ctypes.POINTER(Layout), vp, i32, vp, vp, vp, i32, i32, vp, i64,
                                vp, vp]),
    "starkv_append": (i32, [ctypes.POINTER(Layout), vp, i32, vp, vp, vp, vp, i32, i32, vp, i64,
                            vp, vp, sz, vp, vp]),
    "starkv_dequant": (i32, [ctypes.POINTER(Layout), vp, i64, vp, vp, i32, vp, i32, i32, vp, vp,
                             vp]),
    "starkv_decode_attention": (i32, [ctypes.POINTER(Layout), vp, vp, i64, vp, i32, vp, i32, vp,
                                      vp, vp, sz, vp, vp, sz, ctypes.POINTER(DecodeOpts), vp,
                                      vp]),
    "starkv_decode_partials": (i32, [ctypes.POINTER(Layout), vp, vp, i64, vp, i32, vp, i32, vp, vp,
                                     sz, vp, sz, ctypes.POINTER(DecodeOpts), vp, vp]),
    "starkv_decode_plan_query": (i32, [ctypes.POINTER(Layout), i32, i32, ctypes.POINTER(DecodeOpts),
                                       i32, i64, ctypes.POINTER(DecodePlan)]),
    "starkv_decode_combine": (i32, [ctypes.POINTER(Layout), vp, i32, i32, vp, vp, sz, vp, vp]),
    "starkv_decode_attention_noalloc": (i32, [ctypes.POINTER(Layout), vp, vp, i64, vp, i32, vp, i32,
                                              vp, vp, vp, sz, vp, ctypes.POINTER(DecodeOpts), vp,
                                              vp]),
    "starkv_absorbed_sizes": (i32, [ctypes.POINTER(Layout), i32, i32, ctypes.POINTER(i64),
                                    ctypes.POINTER(sz)]),
    "starkv_absorb_output_weights": (i32, [ctypes.POINTER(Layout), vp, vp, i32, vp, vp]),
    "starkv_decode_combine_absorbed": (i32, [ctypes.POINTER(Layout), vp, i32, i32, vp, i32, vp, sz,
                                             vp, sz, vp, vp]),
    "starkv_diag_bounded_wait": (i32, [i32, vp, vp]),
    "starkv_last_error": (ctypes.c_char_p, []),
    "starkv_version": (i32, []),
}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libstarkv.so")
_lib = None


def load() -> ctypes.CDLL:
    """Load the in-tree CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m rank_quantized_kv_decode_b200.build`"
                " (there is no CPU fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class StarkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = load().starkv_last_error().decode(errors="replace")
        super().__init__(f"{where} failed with status {status}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != OK:
        raise StarkvError(status, where)
