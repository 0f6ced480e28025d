"""CPU oracle for KV-cache rotation + low-bit quantization.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs may import this package. The
product path (``kv_cache_rotation_b200``) never imports it, and this package
imports nothing from the product.

The arithmetic lives in ``kvq_oracle.c`` (plain C, fp32 encode with a fixed
operation order, fp64 decode and score); this module only compiles it and
marshals numpy arrays through ctypes. Every function is pinned by
``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkvq_oracle.so")
_lock = threading.Lock()
_lib = None

ROT_NONE, ROT_FWHT_HEAD, ROT_FWHT_GROUP, ROT_ISO, ROT_ISO3 = 0, 1, 2, 3, 4
Q_MINMAX, Q_CODEBOOK = 0, 1

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library next to its source (gcc)."""
    with _lock:
        stale = not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _LIB_PATH + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _p(a, ct):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ct))


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        f32p, f64p = ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double)
        u8p, u16p = ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_uint16)
        i16p, i64p = ctypes.POINTER(ctypes.c_int16), ctypes.POINTER(ctypes.c_int64)
        ci, cd = ctypes.c_int, ctypes.c_double
        L.orc_half_to_float.restype = ctypes.c_float
        L.orc_half_to_float.argtypes = [ctypes.c_uint16]
        for n in ("orc_float_to_half_rn", "orc_float_to_half_rd", "orc_float_to_half_ru"):
            getattr(L, n).restype = ctypes.c_uint16
            getattr(L, n).argtypes = [ctypes.c_float]
        L.orc_rope_theta.restype = cd
        L.orc_rope_theta.argtypes = [ci, ci, cd, ci]
        L.orc_rope_cs.argtypes = [ctypes.c_int64, ci, cd, ci, f32p, f32p]
        L.orc_rope_apply_f32.argtypes = [f32p, f32p, f32p, f32p, ci]
        L.orc_rope_apply_f32_mode.argtypes = [f32p, f32p, f32p, f32p, ci, ci]
        L.orc_rope_apply_f64.argtypes = [f64p, f64p, ctypes.c_int64, ci, cd, ci, ci]
        L.orc_fwht_f32.argtypes = [f32p, ci]
        L.orc_fwht_f64.argtypes = [f64p, ci]
        L.orc_fwht_scale_f32.restype = ctypes.c_float
        L.orc_fwht_scale_f32.argtypes = [ci]
        L.orc_minmax_group.argtypes = [f32p, ci, ci, u8p, u16p, u16p]
        L.orc_pack.argtypes = [u8p, ci, ci, u8p]
        L.orc_unpack.argtypes = [u8p, ci, ci, u8p]
        L.orc_quat_mul_f32.argtypes = [f32p, f32p, f32p]
        L.orc_quat_mul_f64.argtypes = [f64p, f64p, f64p]
        L.orc_lloyd_max_normal.restype = ci
        L.orc_lloyd_max_normal.argtypes = [ci, f64p, f64p]
        L.orc_codebook.argtypes = [ci, ci, f32p]
        L.orc_encode.restype = ci
        i32p = ctypes.POINTER(ctypes.c_int32)
        L.orc_encode.argtypes = [ci, ci, ci, ci, i64p, ci, ci, ci, ci, ci, ci, ci, cd,
                                 u16p, i16p, f32p, f32p, f32p, u8p, u16p, u16p, f32p, f32p, i32p]
        L.orc_decode.restype = ci
        L.orc_decode.argtypes = [ci, ci, ci, ci, i64p, ci, ci, ci, ci, ci, ci, ci, cd,
                                 u8p, u16p, u16p, f32p, i16p, f32p, f32p, f32p, f64p, i32p]
        L.orc_score.restype = ci
        L.orc_score.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, cd,
                                u16p, u8p, u16p, u16p, f32p, i16p, f32p, f32p, f32p, i64p, ci, cd, f64p, i32p]
        L.orc_attend.restype = ci
        L.orc_attend.argtypes = [ci, ci, ci, ci, ci, ci, ci, ci, ci, ci, cd, u16p,
                                 u8p, u16p, u16p, i16p, ci, u8p, u16p, u16p, i16p, ci, cd, f64p, i32p]
        L.orc_calibrate_perm.restype = ci
        L.orc_calibrate_perm.argtypes = [ci, ci, ci, ci, i64p, ci, ci, cd, u16p, i16p, i32p]
        L.orc_detect_sinks.restype = ci
        L.orc_detect_sinks.argtypes = [ci, ci, ci, ci, i64p, u16p, cd, ci, i32p, i32p]
        L.orc_pair_energy.restype = ci
        L.orc_pair_energy.argtypes = [ci, ci, ci, ci, u16p, ctypes.POINTER(ctypes.c_uint64), i16p]
        u32p = ctypes.POINTER(ctypes.c_uint32)
        L.orc_dyn_calibrate.restype = ci
        L.orc_dyn_calibrate.argtypes = [ci, ci, ci, ci, i64p, ci, ci, u16p, f32p, f32p, i32p, f64p, f32p, u32p]
        L.orc_dyn_encode.restype = ci
        L.orc_dyn_encode.argtypes = [ci, ci, ci, ci, i64p, ci, ci, ci, u16p, f32p, f32p, f32p, f32p, f32p, u32p,
                                     u8p, u16p, u16p, f32p, f32p, i32p]
        L.orc_dyn_decode.restype = ci
        L.orc_dyn_decode.argtypes = [ci, ci, ci, ci, i64p, ci, ci, ci, u8p, u16p, u16p, f32p, f32p, f32p, f32p,
                                     f32p, f32p, u32p, f64p, i32p]
        _lib = L
    return _lib


# ---------------------------------------------------------------- scalar helpers
def half_to_float(h: int) -> float:
    return lib().orc_half_to_float(int(h))


def float_to_half(f: float, mode: str = "rn") -> int:
    return getattr(lib(), f"orc_float_to_half_{mode}")(float(f))


# RoPE frequency tables, passed where a rope flag goes: ROPE_STD (1) the
# standard theta_i = base^(-2i/d), ROPE_FREQ_AWARE (2) the frequency-aware table.
ROPE_STD, ROPE_FREQ_AWARE = 1, 2
# added to either: the half-split pairing (i, i + d/2) instead of the interleaved (2i, 2i + 1)
ROPE_HALF = 4


def rope_theta(i: int, d: int, base: float = 10000.0, mode: int = ROPE_STD) -> float:
    return lib().orc_rope_theta(i, d, base, mode)


def rope_cs(m: int, d: int, base: float = 10000.0, mode: int = ROPE_STD):
    c = np.zeros(d // 2, np.float32)
    s = np.zeros(d // 2, np.float32)
    lib().orc_rope_cs(int(m), d, base, mode, _p(c, ctypes.c_float), _p(s, ctypes.c_float))
    return c, s


def rope_f32(x, c, s, mode: int = ROPE_STD):
    """fp32 RoPE of one vector with the given (cos, sin); mode's ROPE_HALF bit
    chooses the half-split pairs."""
    x = np.ascontiguousarray(x, np.float32)
    y = np.empty_like(x)
    lib().orc_rope_apply_f32_mode(_p(y, ctypes.c_float), _p(x, ctypes.c_float),
                                  _p(np.ascontiguousarray(c, np.float32), ctypes.c_float),
                                  _p(np.ascontiguousarray(s, np.float32), ctypes.c_float), x.size, int(mode))
    return y


def rope_f64(x, m: int, base: float = 10000.0, inverse: bool = False, mode: int = ROPE_STD):
    x = np.ascontiguousarray(x, np.float64)
    y = np.empty_like(x)
    lib().orc_rope_apply_f64(_p(y, ctypes.c_double), _p(x, ctypes.c_double), int(m), x.size, base, mode,
                             int(inverse))
    return y


def fwht_f32(x):
    p = np.array(x, np.float32, copy=True)
    lib().orc_fwht_f32(_p(p, ctypes.c_float), p.size)
    return p


def fwht_f64(x):
    p = np.array(x, np.float64, copy=True)
    lib().orc_fwht_f64(_p(p, ctypes.c_double), p.size)
    return p


def fwht_scale_f32(n: int) -> float:
    return lib().orc_fwht_scale_f32(n)


def minmax_group(p, bits: int):
    p = np.ascontiguousarray(p, np.float32)
    codes = np.zeros(p.size, np.uint8)
    s16 = ctypes.c_uint16()
    z16 = ctypes.c_uint16()
    lib().orc_minmax_group(_p(p, ctypes.c_float), p.size, bits, _p(codes, ctypes.c_uint8),
                           ctypes.byref(s16), ctypes.byref(z16))
    return codes, s16.value, z16.value


def pack(codes, bits: int):
    codes = np.ascontiguousarray(codes, np.uint8)
    out = np.zeros((codes.size * bits + 7) // 8, np.uint8)
    lib().orc_pack(_p(codes, ctypes.c_uint8), codes.size, bits, _p(out, ctypes.c_uint8))
    return out


def unpack(data, n: int, bits: int):
    data = np.ascontiguousarray(data, np.uint8)
    out = np.zeros(n, np.uint8)
    lib().orc_unpack(_p(data, ctypes.c_uint8), n, bits, _p(out, ctypes.c_uint8))
    return out


def quat_mul_f32(a, b):
    a = np.ascontiguousarray(a, np.float32)
    b = np.ascontiguousarray(b, np.float32)
    o = np.zeros(4, np.float32)
    lib().orc_quat_mul_f32(_p(a, ctypes.c_float), _p(b, ctypes.c_float), _p(o, ctypes.c_float))
    return o


def quat_mul_f64(a, b):
    a = np.ascontiguousarray(a, np.float64)
    b = np.ascontiguousarray(b, np.float64)
    o = np.zeros(4, np.float64)
    lib().orc_quat_mul_f64(_p(a, ctypes.c_double), _p(b, ctypes.c_double), _p(o, ctypes.c_double))
    return o


def lloyd_max_normal(bits: int):
    lv = np.zeros(1 << bits, np.float64)
    mse = ctypes.c_double()
    it = lib().orc_lloyd_max_normal(bits, _p(lv, ctypes.c_double), ctypes.byref(mse))
    return lv, mse.value, it


def codebook(bits: int, d: int):
    out = np.zeros(1 << bits, np.float32)
    lib().orc_codebook(bits, d, _p(out, ctypes.c_float))
    return out


# ---------------------------------------------------------------- tensor ops
def _packed_shapes(B, H, T, D, bits, group, n_sink):
    rb = D * bits // 8
    ng = D // group if group else 1
    return (B, H, T, rb), (B, H, T, ng, 2), (B, H, max(n_sink, 0), D), (B, H, T)


def encode(x, pos, *, rot, quant=Q_MINMAX, bits, group=0, group_heads=1, rope=0, n_sink=0,
           base=10000.0, perm=None, qL=None, qR=None, cb=None, want_pre=False, sink_pos=None):
    """x: uint16 (fp16 bits) [B][H][T][D]; pos: int64 [T]. Returns a dict of
    codes [B][H][T][D*bits/8], sz uint16 [B][H][T][D/G][2], sink uint16
    [B][H][n_sink][D], norm f32 [B][H][T], and with want_pre the rotated
    pre-quantization values pre f32 [B][H][T][D]. sink_pos: int32 [B][n_sink]
    sink positions (-1 unused), or None for positions 0 .. n_sink-1."""
    x = np.ascontiguousarray(x, np.uint16)
    B, H, T, D = x.shape
    pos = np.ascontiguousarray(pos, np.int64)
    cs, zs, ss, ns = _packed_shapes(B, H, T, D, bits, group if rot not in (ROT_ISO, ROT_ISO3) else 0, n_sink)
    codes = np.zeros(cs, np.uint8)
    sz = np.zeros(zs, np.uint16)
    sink = np.zeros(ss if n_sink > 0 else (1,), np.uint16)
    norm = np.zeros(ns, np.float32)
    pre = np.zeros((B, H, T, D), np.float32) if want_pre else None
    perm_a = None if perm is None else np.ascontiguousarray(perm, np.int16)
    qL_a = None if qL is None else np.ascontiguousarray(qL, np.float32)
    qR_a = None if qR is None else np.ascontiguousarray(qR, np.float32)
    cb_a = None if cb is None else np.ascontiguousarray(cb, np.float32)
    sp_a = None if sink_pos is None else np.ascontiguousarray(sink_pos, np.int32)
    rc = lib().orc_encode(B, H, T, D, _p(pos, ctypes.c_int64), rot, quant, bits, group, group_heads,
                          rope, n_sink, base, _p(x, ctypes.c_uint16), _p(perm_a, ctypes.c_int16),
                          _p(qL_a, ctypes.c_float), _p(qR_a, ctypes.c_float), _p(cb_a, ctypes.c_float),
                          _p(codes, ctypes.c_uint8), _p(sz, ctypes.c_uint16), _p(sink, ctypes.c_uint16),
                          _p(norm, ctypes.c_float), _p(pre, ctypes.c_float), _p(sp_a, ctypes.c_int32))
    if rc:
        raise ValueError("oracle encode: unsupported parameters")
    return {"codes": codes, "sz": sz, "sink": sink if n_sink > 0 else None, "norm": norm, "pre": pre}


def decode(packed, pos, shape, *, rot, quant=Q_MINMAX, bits, group=0, group_heads=1, rope=0,
           n_sink=0, base=10000.0, perm=None, qL=None, qR=None, cb=None, sink_pos=None):
    """Inverse of encode, in fp64. shape = (B, H, T, D); packed arrays are
    dense over the same T tokens. Returns float64 [B][H][T][D]."""
    B, H, T, D = shape
    pos = np.ascontiguousarray(pos, np.int64)
    out = np.zeros((B, H, T, D), np.float64)
    codes = np.ascontiguousarray(packed["codes"], np.uint8)
    sz = np.ascontiguousarray(packed["sz"], np.uint16) if packed.get("sz") is not None else None
    sink = np.ascontiguousarray(packed["sink"], np.uint16) if packed.get("sink") is not None else None
    norm = np.ascontiguousarray(packed["norm"], np.float32) if packed.get("norm") is not None else None
    perm_a = None if perm is None else np.ascontiguousarray(perm, np.int16)
    qL_a = None if qL is None else np.ascontiguousarray(qL, np.float32)
    qR_a = None if qR is None else np.ascontiguousarray(qR, np.float32)
    cb_a = None if cb is None else np.ascontiguousarray(cb, np.float32)
    sp_a = None if sink_pos is None else np.ascontiguousarray(sink_pos, np.int32)
    rc = lib().orc_decode(B, H, T, D, _p(pos, ctypes.c_int64), rot, quant, bits, group, group_heads,
                          rope, n_sink, base, _p(codes, ctypes.c_uint8), _p(sz, ctypes.c_uint16),
                          _p(sink, ctypes.c_uint16), _p(norm, ctypes.c_float), _p(perm_a, ctypes.c_int16),
                          _p(qL_a, ctypes.c_float), _p(qR_a, ctypes.c_float), _p(cb_a, ctypes.c_float),
                          _p(out, ctypes.c_double), _p(sp_a, ctypes.c_int32))
    if rc:
        raise ValueError("oracle decode: unsupported parameters")
    return out


def score(q, cache, tokens, *, H, t_cap, rot, quant=Q_MINMAX, bits, group=0, group_heads=1, rope=0,
          n_sink=0, base=10000.0, scale, perm=None, qL=None, qR=None, cb=None, sink_pos=None):
    """q: uint16 [B][Hq][D] (attention space); cache arrays laid out over
    t_cap slots; tokens: int64 positions to score. Returns float64
    [B][Hq][len(tokens)]."""
    q = np.ascontiguousarray(q, np.uint16)
    B, Hq, D = q.shape
    tok = np.ascontiguousarray(tokens, np.int64)
    out = np.zeros((B, Hq, tok.size), np.float64)
    codes = np.ascontiguousarray(cache["codes"], np.uint8)
    sz = np.ascontiguousarray(cache["sz"], np.uint16) if cache.get("sz") is not None else None
    sink = np.ascontiguousarray(cache["sink"], np.uint16) if cache.get("sink") is not None else None
    norm = np.ascontiguousarray(cache["norm"], np.float32) if cache.get("norm") is not None else None
    perm_a = None if perm is None else np.ascontiguousarray(perm, np.int16)
    qL_a = None if qL is None else np.ascontiguousarray(qL, np.float32)
    qR_a = None if qR is None else np.ascontiguousarray(qR, np.float32)
    cb_a = None if cb is None else np.ascontiguousarray(cb, np.float32)
    sp_a = None if sink_pos is None else np.ascontiguousarray(sink_pos, np.int32)
    rc = lib().orc_score(B, H, Hq, D, t_cap, rot, quant, bits, group, group_heads, rope, n_sink, base,
                         _p(q, ctypes.c_uint16), _p(codes, ctypes.c_uint8), _p(sz, ctypes.c_uint16),
                         _p(sink, ctypes.c_uint16), _p(norm, ctypes.c_float), _p(perm_a, ctypes.c_int16),
                         _p(qL_a, ctypes.c_float), _p(qR_a, ctypes.c_float), _p(cb_a, ctypes.c_float),
                         _p(tok, ctypes.c_int64), tok.size, float(scale), _p(out, ctypes.c_double),
                         _p(sp_a, ctypes.c_int32))
    if rc:
        raise ValueError("oracle score: unsupported parameters")
    return out


def attend(q, kcache, vcache, n_tok, *, H, t_cap, rot, bits, group, n_sink=0, base=10000.0, scale,
           kperm=None, vperm=None, krope=1, vrope=0, sink_pos=None):
    """Decode-step attention (orc_attend). q: uint16 [B][Hq][D] in attention
    space; kcache / vcache: dicts of codes, sz and sink laid out over t_cap
    slots; sink_pos: int32 [B][n_sink] sink list of both caches, or None for
    the positions < n_sink. Returns float64 [B][Hq][D]."""
    q = np.ascontiguousarray(q, np.uint16)
    B, Hq, D = q.shape
    out = np.zeros((B, Hq, D), np.float64)

    def arrs(c, perm):
        codes = np.ascontiguousarray(c["codes"], np.uint8)
        sz = np.ascontiguousarray(c["sz"], np.uint16)
        sink = np.ascontiguousarray(c["sink"], np.uint16) if c.get("sink") is not None else None
        pm = None if perm is None else np.ascontiguousarray(perm, np.int16)
        return codes, sz, sink, pm

    kc, kz, ks, kp = arrs(kcache, kperm)
    vc, vz, vs, vp = arrs(vcache, vperm)
    sp = None if sink_pos is None else np.ascontiguousarray(sink_pos, np.int32)
    rc = lib().orc_attend(B, H, Hq, D, t_cap, int(n_tok), rot, bits, group, n_sink, base, _p(q, ctypes.c_uint16),
                          _p(kc, ctypes.c_uint8), _p(kz, ctypes.c_uint16), _p(ks, ctypes.c_uint16),
                          _p(kp, ctypes.c_int16), int(krope), _p(vc, ctypes.c_uint8), _p(vz, ctypes.c_uint16),
                          _p(vs, ctypes.c_uint16), _p(vp, ctypes.c_int16), int(vrope), float(scale),
                          _p(out, ctypes.c_double), _p(sp, ctypes.c_int32))
    if rc:
        raise ValueError("oracle attend: unsupported parameters")
    return out


def calibrate_perm(x, pos, *, rope=0, n_sink=0, base=10000.0, sink_pos=None):
    x = np.ascontiguousarray(x, np.uint16)
    B, H, T, D = x.shape
    pos = np.ascontiguousarray(pos, np.int64)
    perm = np.zeros((H, D), np.int16)
    sp_a = None if sink_pos is None else np.ascontiguousarray(sink_pos, np.int32)
    lib().orc_calibrate_perm(B, H, T, D, _p(pos, ctypes.c_int64), rope, n_sink, base,
                             _p(x, ctypes.c_uint16), _p(perm, ctypes.c_int16), _p(sp_a, ctypes.c_int32))
    return perm


def detect_sinks(x, pos, *, tau, max_sinks):
    """Sinks by massive activations (orc_detect_sinks): x uint16 [B][H][T][D];
    returns (int32 [B][max_sinks] ascending positions padded with -1, int32 [B] counts)."""
    x = np.ascontiguousarray(x, np.uint16)
    B, H, T, D = x.shape
    pos = np.ascontiguousarray(pos, np.int64)
    sp = np.zeros((B, max_sinks), np.int32)
    cnt = np.zeros(B, np.int32)
    rc = lib().orc_detect_sinks(B, H, T, D, _p(pos, ctypes.c_int64), _p(x, ctypes.c_uint16), float(tau),
                                int(max_sinks), _p(sp, ctypes.c_int32), _p(cnt, ctypes.c_int32))
    if rc:
        raise ValueError("oracle detect_sinks: unsupported parameters")
    return sp, cnt


def pair_energy(x):
    """orc_pair_energy: per head, the exact energy of each RoPE pair summed over
    batches and tokens, as Python ints in units of 2^-48, and the pairs ranked
    by descending energy (ties in ascending pair order). x: uint16 [B][H][T][D]."""
    x = np.ascontiguousarray(x, np.uint16)
    B, H, T, D = x.shape
    e = np.zeros((H, D // 2, 2), np.uint64)
    rank = np.zeros((H, D // 2), np.int16)
    if lib().orc_pair_energy(B, H, T, D, _p(x, ctypes.c_uint16), _p(e, ctypes.c_uint64), _p(rank, ctypes.c_int16)):
        raise MemoryError("oracle pair energy")
    return e, rank


def energy_ints(e):
    """(lo, hi) uint64 pairs -> Python ints."""
    return [[int(p[0]) | (int(p[1]) << 64) for p in row] for row in e]


# ---------------------------------------------------------------- dynamic codebooks
def _opt(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype)


def dyn_calibrate(x, pos, *, rot, qL, qR=None, n_sink=0, sink_pos=None):
    """Per-channel statistics of the rotated unit vectors (orc_dyn_calibrate):
    returns (m2 float64 [H][D], sigma float32 [H][D], wide uint32 [H][D/32])."""
    x = np.ascontiguousarray(x, np.uint16)
    B, H, T, D = x.shape
    pos = np.ascontiguousarray(pos, np.int64)
    qL = np.ascontiguousarray(qL, np.float32)
    qR = _opt(qR, np.float32)
    sp = _opt(sink_pos, np.int32)
    m2 = np.zeros((H, D), np.float64)
    sigma = np.zeros((H, D), np.float32)
    wide = np.zeros((H, D // 32), np.uint32)
    rc = lib().orc_dyn_calibrate(B, H, T, D, _p(pos, ctypes.c_int64), rot, n_sink, _p(x, ctypes.c_uint16),
                                 _p(qL, ctypes.c_float), _p(qR, ctypes.c_float) if qR is not None else None,
                                 _p(sp, ctypes.c_int32) if sp is not None else None, _p(m2, ctypes.c_double),
                                 _p(sigma, ctypes.c_float), _p(wide, ctypes.c_uint32))
    if rc:
        raise ValueError("orc_dyn_calibrate: unsupported arguments")
    return m2, sigma, wide


def dyn_encode(x, pos, *, rot, bits, qL, qR=None, cb, cbw, sigma, wide, n_sink=0, sink_pos=None, want_pre=False):
    """IsoQuant with per-channel codebooks (orc_dyn_encode): codes [B][H][T][D*bits/8],
    ext uint16 [B][H][T], sink uint16 [B][H][n_sink][D], norm f32 [B][H][T], pre (optional)."""
    x = np.ascontiguousarray(x, np.uint16)
    B, H, T, D = x.shape
    pos = np.ascontiguousarray(pos, np.int64)
    out = {"codes": np.zeros((B, H, T, D * bits // 8), np.uint8), "ext": np.zeros((B, H, T), np.uint16),
           "sink": np.zeros((B, H, max(n_sink, 1), D), np.uint16), "norm": np.zeros((B, H, T), np.float32)}
    pre = np.zeros((B, H, T, D), np.float32) if want_pre else None
    qL = np.ascontiguousarray(qL, np.float32)
    qR = _opt(qR, np.float32)
    cb, cbw = np.ascontiguousarray(cb, np.float32), np.ascontiguousarray(cbw, np.float32)
    sigma, wide = np.ascontiguousarray(sigma, np.float32), np.ascontiguousarray(wide, np.uint32)
    sp = _opt(sink_pos, np.int32)
    rc = lib().orc_dyn_encode(B, H, T, D, _p(pos, ctypes.c_int64), rot, bits, n_sink, _p(x, ctypes.c_uint16),
                              _p(qL, ctypes.c_float), _p(qR, ctypes.c_float) if qR is not None else None,
                              _p(cb, ctypes.c_float), _p(cbw, ctypes.c_float), _p(sigma, ctypes.c_float),
                              _p(wide, ctypes.c_uint32), _p(out["codes"], ctypes.c_uint8),
                              _p(out["ext"], ctypes.c_uint16), _p(out["sink"], ctypes.c_uint16),
                              _p(out["norm"], ctypes.c_float), _p(pre, ctypes.c_float) if pre is not None else None,
                              _p(sp, ctypes.c_int32) if sp is not None else None)
    if rc:
        raise ValueError("orc_dyn_encode: unsupported arguments")
    if not n_sink:
        out["sink"] = None
    if want_pre:
        out["pre"] = pre
    return out


def dyn_decode(packed, pos, shape, *, rot, bits, qL, qR=None, cb, cbw, sigma, wide, n_sink=0, sink_pos=None):
    """Inverse of dyn_encode in fp64: float64 [B][H][T][D]."""
    B, H, T, D = shape
    pos = np.ascontiguousarray(pos, np.int64)
    out = np.zeros((B, H, T, D), np.float64)
    codes = np.ascontiguousarray(packed["codes"], np.uint8)
    ext = np.ascontiguousarray(packed["ext"], np.uint16)
    norm = np.ascontiguousarray(packed["norm"], np.float32)
    sink = packed.get("sink")
    sink = np.ascontiguousarray(sink, np.uint16) if sink is not None else np.zeros(1, np.uint16)
    qL = np.ascontiguousarray(qL, np.float32)
    qR = _opt(qR, np.float32)
    cb, cbw = np.ascontiguousarray(cb, np.float32), np.ascontiguousarray(cbw, np.float32)
    sigma, wide = np.ascontiguousarray(sigma, np.float32), np.ascontiguousarray(wide, np.uint32)
    sp = _opt(sink_pos, np.int32)
    rc = lib().orc_dyn_decode(B, H, T, D, _p(pos, ctypes.c_int64), rot, bits, n_sink, _p(codes, ctypes.c_uint8),
                              _p(ext, ctypes.c_uint16), _p(sink, ctypes.c_uint16), _p(norm, ctypes.c_float),
                              _p(qL, ctypes.c_float), _p(qR, ctypes.c_float) if qR is not None else None,
                              _p(cb, ctypes.c_float), _p(cbw, ctypes.c_float), _p(sigma, ctypes.c_float),
                              _p(wide, ctypes.c_uint32), _p(out, ctypes.c_double),
                              _p(sp, ctypes.c_int32) if sp is not None else None)
    if rc:
        raise ValueError("orc_dyn_decode: unsupported arguments")
    return out
