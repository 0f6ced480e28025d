"""Python binding of libkvq (argument marshalling only).

Every function here has the name of the C entry point it forwards to
(include/kvq.h) and does nothing but convert arguments: all computation runs
in the CUDA kernels of ``libkvq.so``. There is no fallback: importing the
package without the built library raises.

Tensors are passed as raw device addresses (``tensor.data_ptr()``) and the
stream as a ``cudaStream_t`` value (``torch.cuda.current_stream().cuda_stream``);
PyTorch is used by callers for device memory and streams only.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkvq.so")

KVQ_OK, KVQ_ERR_INVALID, KVQ_ERR_UNSUPPORTED, KVQ_ERR_ALIGN, KVQ_ERR_CUDA, KVQ_ERR_TIMEOUT = range(6)
KVQ_ROT_NONE, KVQ_ROT_FWHT_HEAD, KVQ_ROT_FWHT_GROUP, KVQ_ROT_ISO_SO4, KVQ_ROT_ISO_SO3 = range(5)
KVQ_Q_MINMAX, KVQ_Q_CODEBOOK, KVQ_Q_CODEBOOK_DYN = 0, 1, 2
KVQ_FIELD_CODES, KVQ_FIELD_SCALE_ZERO, KVQ_FIELD_SINK, KVQ_FIELD_NORM, KVQ_FIELD_EXT = range(5)

EXPORTED = ("kvq_encode", "kvq_decode", "kvq_score", "kvq_score_literal", "kvq_attend", "kvq_attend_noalloc", "kvq_attend_workspace_bytes",
            "kvq_calibrate_perm", "kvq_calibrate_workspace_bytes", "kvq_pair_energy",
            "kvq_detect_sinks", "kvq_detect_sinks_workspace_bytes",
            "kvq_calibrate_codebook", "kvq_calibrate_codebook_workspace_bytes",
            "kvq_packed_bytes", "kvq_rope_table", "kvq_rope_table_ex", "kvq_lloyd_max_codebook", "kvq_check", "kvq_debug_expire_wait",
            "kvq_status_str", "kvq_version")


class kvq_desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "heads", "head_dim", "tokens", "t0", "t_cap", "bits", "group", "group_heads", "rope",
        "n_sink", "rot", "quant")]


class kvq_packed(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scale_zero", ctypes.c_void_p), ("sink", ctypes.c_void_p),
                ("norm", ctypes.c_void_p), ("ext", ctypes.c_void_p)]


class kvq_tables(ctypes.Structure):
    _fields_ = [("perm", ctypes.c_void_p), ("rope_cs", ctypes.c_void_p), ("rope_rows", ctypes.c_int32),
                ("qL", ctypes.c_void_p), ("qR", ctypes.c_void_p), ("codebook", ctypes.c_void_p),
                ("sink_pos", ctypes.c_void_p), ("codebook_wide", ctypes.c_void_p), ("ch_scale", ctypes.c_void_p),
                ("ch_wide", ctypes.c_void_p)]


class KvqError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {kvq_status_str(status)} ({status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python kv_cache_rotation_b200/build.py` "
                          "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    vp, i32, st = ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p
    L.kvq_encode.argtypes = [P(kvq_desc), vp, P(kvq_tables), P(kvq_packed), st]
    L.kvq_decode.argtypes = [P(kvq_desc), P(kvq_packed), P(kvq_tables), vp, i32, st]
    L.kvq_score.argtypes = [P(kvq_desc), vp, i32, P(kvq_packed), P(kvq_tables), i32, ctypes.c_float, vp, st]
    L.kvq_score_literal.argtypes = L.kvq_score.argtypes
    L.kvq_attend.argtypes = [P(kvq_desc), P(kvq_desc), vp, i32, P(kvq_packed), P(kvq_tables), P(kvq_packed),
                             P(kvq_tables), i32, ctypes.c_float, vp, vp, ctypes.c_size_t, st]
    L.kvq_attend_noalloc.argtypes = [P(kvq_desc), P(kvq_desc), vp, i32, P(kvq_packed), P(kvq_tables),
                                     P(kvq_packed), P(kvq_tables), i32, ctypes.c_float, vp, st]
    L.kvq_calibrate_perm.argtypes = [P(kvq_desc), vp, P(kvq_tables), vp, vp, ctypes.c_size_t, st]
    L.kvq_pair_energy.argtypes = [P(kvq_desc), vp, vp, vp, st]
    L.kvq_detect_sinks.argtypes = [P(kvq_desc), vp, ctypes.c_double, i32, vp, vp, vp, ctypes.c_size_t, st]
    L.kvq_detect_sinks_workspace_bytes.argtypes = [P(kvq_desc)]
    L.kvq_detect_sinks_workspace_bytes.restype = ctypes.c_size_t
    L.kvq_calibrate_codebook.argtypes = [P(kvq_desc), vp, P(kvq_tables), vp, vp, vp, ctypes.c_size_t, st]
    L.kvq_calibrate_codebook_workspace_bytes.argtypes = [P(kvq_desc)]
    L.kvq_calibrate_codebook_workspace_bytes.restype = ctypes.c_size_t
    L.kvq_calibrate_workspace_bytes.argtypes = [P(kvq_desc)]
    L.kvq_calibrate_workspace_bytes.restype = ctypes.c_size_t
    L.kvq_attend_workspace_bytes.argtypes = [P(kvq_desc), P(kvq_desc), i32, i32]
    L.kvq_attend_workspace_bytes.restype = ctypes.c_size_t
    L.kvq_packed_bytes.argtypes = [P(kvq_desc), i32]
    L.kvq_packed_bytes.restype = ctypes.c_size_t
    L.kvq_rope_table.argtypes = [vp, i32, i32, ctypes.c_double]
    L.kvq_rope_table_ex.argtypes = [vp, i32, i32, ctypes.c_double, i32]
    L.kvq_lloyd_max_codebook.argtypes = [vp, i32, i32]
    L.kvq_check.argtypes = [st]
    L.kvq_debug_expire_wait.argtypes = [ctypes.c_uint32, st]
    L.kvq_status_str.argtypes = [i32]
    L.kvq_status_str.restype = ctypes.c_char_p
    L.kvq_version.restype = i32
    for n in ("kvq_encode", "kvq_decode", "kvq_score", "kvq_score_literal", "kvq_attend", "kvq_attend_noalloc", "kvq_calibrate_perm",
              "kvq_pair_energy", "kvq_detect_sinks", "kvq_calibrate_codebook",
              "kvq_rope_table", "kvq_rope_table_ex",
              "kvq_lloyd_max_codebook",
              "kvq_check", "kvq_debug_expire_wait"):
        getattr(L, n).restype = i32
    return L


lib = _load()


# ---------------------------------------------------------------- entry points
def kvq_encode(desc: kvq_desc, x: int, tables: kvq_tables, out: kvq_packed, stream: int = 0) -> int:
    return lib.kvq_encode(ctypes.byref(desc), x, ctypes.byref(tables), ctypes.byref(out), stream)


def kvq_decode(desc: kvq_desc, packed: kvq_packed, tables: kvq_tables, x_out: int, out_fp32: int,
               stream: int = 0) -> int:
    return lib.kvq_decode(ctypes.byref(desc), ctypes.byref(packed), ctypes.byref(tables), x_out, int(out_fp32),
                          stream)


def kvq_score(desc: kvq_desc, q: int, q_heads: int, cache: kvq_packed, tables: kvq_tables, n_tokens: int,
              scale: float, scores: int, stream: int = 0) -> int:
    return lib.kvq_score(ctypes.byref(desc), q, q_heads, ctypes.byref(cache), ctypes.byref(tables), n_tokens,
                         scale, scores, stream)


def kvq_score_literal(desc: kvq_desc, q: int, q_heads: int, cache: kvq_packed, tables: kvq_tables, n_tokens: int,
                      scale: float, scores: int, stream: int = 0) -> int:
    return lib.kvq_score_literal(ctypes.byref(desc), q, q_heads, ctypes.byref(cache), ctypes.byref(tables),
                                 n_tokens, scale, scores, stream)


def kvq_attend(dk: kvq_desc, dv: kvq_desc, q: int, q_heads: int, k_cache: kvq_packed, tk: kvq_tables,
               v_cache: kvq_packed, tv: kvq_tables, n_tokens: int, scale: float, out: int, workspace: int,
               workspace_bytes: int, stream: int = 0) -> int:
    return lib.kvq_attend(ctypes.byref(dk), ctypes.byref(dv), q, q_heads, ctypes.byref(k_cache), ctypes.byref(tk),
                          ctypes.byref(v_cache), ctypes.byref(tv), n_tokens, scale, out, workspace, workspace_bytes,
                          stream)


def kvq_attend_noalloc(dk: kvq_desc, dv: kvq_desc, q: int, q_heads: int, k_cache: kvq_packed, tk: kvq_tables,
                       v_cache: kvq_packed, tv: kvq_tables, n_tokens: int, scale: float, out: int,
                       stream: int = 0) -> int:
    return lib.kvq_attend_noalloc(ctypes.byref(dk), ctypes.byref(dv), q, q_heads, ctypes.byref(k_cache),
                                  ctypes.byref(tk), ctypes.byref(v_cache), ctypes.byref(tv), n_tokens, scale, out,
                                  stream)


def kvq_calibrate_perm(d: kvq_desc, x: int, tb: kvq_tables, perm_out: int, workspace: int, workspace_bytes: int,
                       stream: int = 0) -> int:
    return lib.kvq_calibrate_perm(ctypes.byref(d), x, ctypes.byref(tb), perm_out, workspace, workspace_bytes, stream)


def kvq_pair_energy(d: kvq_desc, x: int, energy_out: int, rank_out: int, stream: int = 0) -> int:
    return lib.kvq_pair_energy(ctypes.byref(d), x, energy_out, rank_out, stream)


def kvq_detect_sinks(d: kvq_desc, x: int, tau: float, max_sinks: int, sink_pos: int, count: int, workspace: int,
                     workspace_bytes: int, stream: int = 0) -> int:
    return lib.kvq_detect_sinks(ctypes.byref(d), x, tau, max_sinks, sink_pos, count, workspace, workspace_bytes,
                                stream)


def kvq_calibrate_codebook(d: kvq_desc, x: int, tb: kvq_tables, ch_scale_out: int, ch_wide_out: int,
                           workspace: int, workspace_bytes: int, stream: int = 0) -> int:
    return lib.kvq_calibrate_codebook(ctypes.byref(d), x, ctypes.byref(tb), ch_scale_out, ch_wide_out, workspace,
                                      workspace_bytes, stream)


def kvq_calibrate_codebook_workspace_bytes(d: kvq_desc) -> int:
    return lib.kvq_calibrate_codebook_workspace_bytes(ctypes.byref(d))


def kvq_detect_sinks_workspace_bytes(d: kvq_desc) -> int:
    return lib.kvq_detect_sinks_workspace_bytes(ctypes.byref(d))


def kvq_calibrate_workspace_bytes(d: kvq_desc) -> int:
    return lib.kvq_calibrate_workspace_bytes(ctypes.byref(d))


def kvq_attend_workspace_bytes(dk: kvq_desc, dv: kvq_desc, q_heads: int, n_tokens: int) -> int:
    return lib.kvq_attend_workspace_bytes(ctypes.byref(dk), ctypes.byref(dv), q_heads, n_tokens)


def kvq_packed_bytes(desc: kvq_desc, field: int) -> int:
    return lib.kvq_packed_bytes(ctypes.byref(desc), field)


def kvq_rope_table(cs_host: int, t_max: int, head_dim: int, base: float = 10000.0) -> int:
    return lib.kvq_rope_table(cs_host, t_max, head_dim, base)


KVQ_ROPE_STANDARD, KVQ_ROPE_FREQ_AWARE = 0, 1


def kvq_rope_table_ex(cs_host: int, t_max: int, head_dim: int, base: float = 10000.0,
                      freq: int = KVQ_ROPE_STANDARD) -> int:
    return lib.kvq_rope_table_ex(cs_host, t_max, head_dim, base, freq)


def kvq_lloyd_max_codebook(levels_host: int, bits: int, head_dim: int) -> int:
    return lib.kvq_lloyd_max_codebook(levels_host, bits, head_dim)


def kvq_check(stream: int = 0) -> int:
    return lib.kvq_check(stream)


def kvq_debug_expire_wait(limit_us: int, stream: int = 0) -> int:
    return lib.kvq_debug_expire_wait(limit_us, stream)


def kvq_status_str(status: int) -> str:
    return lib.kvq_status_str(status).decode()


def kvq_version() -> int:
    return lib.kvq_version()


def check(status: int, what: str = "kvq") -> None:
    """Raise KvqError unless status is KVQ_OK."""
    if status != KVQ_OK:
        raise KvqError(status, what)


from . import torch_api  # noqa: E402,F401  (marshalling helpers for torch tensors)
