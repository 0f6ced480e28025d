"""Marshalling helpers between torch tensors and the libkvq C ABI.

Nothing here computes: tensors are allocated with torch (device memory is
PyTorch's job), their addresses are put into the ABI structs, and the C entry
points run the CUDA kernels. Host-side tables (RoPE cos/sin, Lloyd-Max
levels) are filled by the library's own host helpers and uploaded.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import (KVQ_FIELD_CODES, KVQ_FIELD_EXT, KVQ_FIELD_NORM, KVQ_FIELD_SCALE_ZERO, KVQ_FIELD_SINK,
               KVQ_Q_CODEBOOK, KVQ_Q_CODEBOOK_DYN, KVQ_Q_MINMAX, KVQ_ROT_FWHT_GROUP, KVQ_ROT_FWHT_HEAD, KVQ_ROT_ISO_SO3, KVQ_ROT_ISO_SO4, KVQ_ROT_NONE,
               check,
               kvq_decode, kvq_desc, kvq_encode, kvq_lloyd_max_codebook, kvq_packed, kvq_packed_bytes,
               kvq_rope_table, kvq_score, kvq_score_literal, kvq_tables)

ROT = {"none": KVQ_ROT_NONE, "fwht_head": KVQ_ROT_FWHT_HEAD, "fwht_group": KVQ_ROT_FWHT_GROUP,
       "iso": KVQ_ROT_ISO_SO4, "iso3": KVQ_ROT_ISO_SO3}
QUANT = {"minmax": KVQ_Q_MINMAX, "codebook": KVQ_Q_CODEBOOK, "codebook_dyn": KVQ_Q_CODEBOOK_DYN}


def make_desc(*, batch, heads, head_dim=128, tokens, t0=0, t_cap=None, bits, group=128, group_heads=1, rope=0,
              n_sink=0, rot="fwht_head", quant="minmax") -> kvq_desc:
    d = kvq_desc()
    d.batch, d.heads, d.head_dim, d.tokens, d.t0 = batch, heads, head_dim, tokens, t0
    d.t_cap = t0 + tokens if t_cap is None else t_cap
    d.bits, d.group, d.group_heads, d.rope, d.n_sink = bits, group, group_heads, int(rope), n_sink
    d.rot = ROT[rot] if isinstance(rot, str) else rot
    d.quant = QUANT[quant] if isinstance(quant, str) else quant
    return d


@dataclass
class Packed:
    codes: torch.Tensor
    scale_zero: Optional[torch.Tensor]
    sink: Optional[torch.Tensor]
    norm: Optional[torch.Tensor]
    ext: Optional[torch.Tensor] = None

    def struct(self) -> kvq_packed:
        p = kvq_packed()
        p.codes = self.codes.data_ptr()
        p.scale_zero = self.scale_zero.data_ptr() if self.scale_zero is not None else None
        p.sink = self.sink.data_ptr() if self.sink is not None else None
        p.norm = self.norm.data_ptr() if self.norm is not None else None
        p.ext = self.ext.data_ptr() if self.ext is not None else None
        return p

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size()
                   for t in (self.codes, self.scale_zero, self.sink, self.norm, self.ext) if t is not None)


def alloc_packed(d: kvq_desc, device="cuda", zero=True) -> Packed:
    """Allocate the cache buffers of a descriptor (sizes from kvq_packed_bytes)."""
    alloc = torch.zeros if zero else torch.empty

    def buf(field, dtype, shape):
        n = kvq_packed_bytes(d, field)
        if n == 0:
            return None
        t = alloc(n, dtype=torch.uint8, device=device)
        return t.view(dtype).view(shape)

    B, H, C, D = d.batch, d.heads, d.t_cap, d.head_dim
    codes = buf(KVQ_FIELD_CODES, torch.uint8, (B, H, C, D * d.bits // 8))
    ng = D // d.group if d.quant == KVQ_Q_MINMAX else 0
    sz = buf(KVQ_FIELD_SCALE_ZERO, torch.int16, (B, H, C, ng, 2)) if ng else None
    sink = buf(KVQ_FIELD_SINK, torch.float16, (B, H, d.n_sink, D)) if d.n_sink else None
    norm = buf(KVQ_FIELD_NORM, torch.float32, (B, H, C))
    ext = buf(KVQ_FIELD_EXT, torch.int16, (B, H, C))
    return Packed(codes, sz, sink, norm, ext)


def rope_table(t_max: int, head_dim: int, device="cuda", base: float = 10000.0, freq: int = 0) -> torch.Tensor:
    """(cos, sin) table [t_max][head_dim/2][2] filled by kvq_rope_table_ex (freq: KVQ_ROPE_*)."""
    from . import kvq_rope_table_ex
    host = torch.empty((t_max, head_dim // 2, 2), dtype=torch.float32)
    check(kvq_rope_table_ex(host.data_ptr(), t_max, head_dim, base, freq), "kvq_rope_table_ex")
    return host.to(device)


def lloyd_max_codebook(bits: int, head_dim: int, device="cuda") -> torch.Tensor:
    host = torch.empty(1 << bits, dtype=torch.float32)
    check(kvq_lloyd_max_codebook(host.data_ptr(), bits, head_dim), "kvq_lloyd_max_codebook")
    return host.to(device)


@dataclass
class Tables:
    """Device tables of one call; holds the tensors so their memory stays
    alive for as long as the struct built from them is in use."""
    perm: Optional[torch.Tensor] = None
    rope_cs: Optional[torch.Tensor] = None
    qL: Optional[torch.Tensor] = None
    qR: Optional[torch.Tensor] = None
    codebook: Optional[torch.Tensor] = None
    sink_pos: Optional[torch.Tensor] = None  # int32 [B][n_sink]: the list form of the sink set
    codebook_wide: Optional[torch.Tensor] = None  # dynamic codebooks: the (bits+1)-bit N(0,1) levels
    ch_scale: Optional[torch.Tensor] = None  # dynamic codebooks: f32 [H][D]
    ch_wide: Optional[torch.Tensor] = None  # dynamic codebooks: int32 [H][D/32] outlier-channel masks

    def struct(self) -> kvq_tables:
        tb = kvq_tables()
        tb.perm = self.perm.data_ptr() if self.perm is not None else None
        tb.rope_cs = self.rope_cs.data_ptr() if self.rope_cs is not None else None
        tb.rope_rows = self.rope_cs.shape[0] if self.rope_cs is not None else 0
        tb.qL = self.qL.data_ptr() if self.qL is not None else None
        tb.qR = self.qR.data_ptr() if self.qR is not None else None
        tb.codebook = self.codebook.data_ptr() if self.codebook is not None else None
        if self.sink_pos is not None:
            _req(self.sink_pos, "sink_pos", (torch.int32,))
            tb.sink_pos = self.sink_pos.data_ptr()
        tb.codebook_wide = self.codebook_wide.data_ptr() if self.codebook_wide is not None else None
        tb.ch_scale = self.ch_scale.data_ptr() if self.ch_scale is not None else None
        tb.ch_wide = self.ch_wide.data_ptr() if self.ch_wide is not None else None
        return tb


def make_tables(perm=None, rope_cs=None, qL=None, qR=None, codebook=None, sink_pos=None, codebook_wide=None,
                ch_scale=None, ch_wide=None) -> Tables:
    return Tables(perm, rope_cs, qL, qR, codebook, sink_pos, codebook_wide, ch_scale, ch_wide)


def _req(t: torch.Tensor, name: str, dtypes, shape=None) -> None:
    """Reject a tensor the C ABI would misread: it must be a contiguous CUDA
    tensor of one of `dtypes`, shaped `shape` when given."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def _kv_shape(d: kvq_desc):
    return (d.batch, d.heads, d.tokens, d.head_dim)


def _q_heads(d: kvq_desc, q: torch.Tensor) -> int:
    _req(q, "q", (torch.float16,))
    if q.dim() != 3 or q.shape[0] != d.batch or q.shape[2] != d.head_dim:
        raise ValueError(f"q: shape {tuple(q.shape)}, expected ({d.batch}, q_heads, {d.head_dim})")
    return int(q.shape[1])


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def encode(d: kvq_desc, x: torch.Tensor, tables: Tables, packed: Packed, stream=None) -> None:
    _req(x, "x", (torch.float16,), _kv_shape(d))
    check(kvq_encode(d, x.data_ptr(), tables.struct(), packed.struct(), _stream(stream)), "kvq_encode")


def decode(d: kvq_desc, packed: Packed, tables: Tables, out: torch.Tensor, stream=None) -> None:
    _req(out, "out", (torch.float16, torch.float32), _kv_shape(d))
    fp32 = 1 if out.dtype == torch.float32 else 0
    check(kvq_decode(d, packed.struct(), tables.struct(), out.data_ptr(), fp32, _stream(stream)), "kvq_decode")


def score(d: kvq_desc, q: torch.Tensor, packed: Packed, tables: Tables, n_tokens: int, scale: float,
          out: torch.Tensor, stream=None) -> None:
    hq = _q_heads(d, q)
    _req(out, "scores", (torch.float32,), (d.batch, hq, n_tokens))
    check(kvq_score(d, q.data_ptr(), hq, packed.struct(), tables.struct(), n_tokens, scale,
                    out.data_ptr(), _stream(stream)), "kvq_score")


def score_literal(d: kvq_desc, q: torch.Tensor, packed: Packed, tables: Tables, n_tokens: int, scale: float,
                  out: torch.Tensor, stream=None) -> None:
    """The scores of score(), every key decoded on the fly (the literal per-token form)."""
    hq = _q_heads(d, q)
    _req(out, "scores", (torch.float32,), (d.batch, hq, n_tokens))
    check(kvq_score_literal(d, q.data_ptr(), hq, packed.struct(), tables.struct(), n_tokens, scale,
                            out.data_ptr(), _stream(stream)), "kvq_score_literal")


def attend_workspace(dk: kvq_desc, dv: kvq_desc, q_heads: int, n_tokens: int, device="cuda") -> torch.Tensor:
    """A workspace tensor for kvq_attend (256-byte aligned, as torch allocates)."""
    from . import kvq_attend_workspace_bytes
    nb = kvq_attend_workspace_bytes(dk, dv, q_heads, n_tokens)
    if nb == 0:
        raise ValueError("kvq_attend: invalid or unsupported shapes")
    return torch.empty(nb, dtype=torch.uint8, device=device)


def attend(dk: kvq_desc, dv: kvq_desc, q: torch.Tensor, k_packed: Packed, tk: Tables, v_packed: Packed, tv: Tables,
           n_tokens: int, scale: float, out: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    from . import kvq_attend
    hq = _q_heads(dk, q)
    _req(out, "out", (torch.float32,), (dk.batch, hq, dk.head_dim))
    _req(workspace, "workspace", (torch.uint8,))
    check(kvq_attend(dk, dv, q.data_ptr(), hq, k_packed.struct(), tk.struct(), v_packed.struct(),
                     tv.struct(), n_tokens, scale, out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                     _stream(stream)), "kvq_attend")


def attend_noalloc(dk: kvq_desc, dv: kvq_desc, q: torch.Tensor, k_packed: Packed, tk: Tables, v_packed: Packed,
                   tv: Tables, n_tokens: int, scale: float, out: torch.Tensor, stream=None) -> None:
    """kvq_attend through the library's fixed scratch (no workspace tensor)."""
    from . import kvq_attend_noalloc
    hq = _q_heads(dk, q)
    _req(out, "out", (torch.float32,), (dk.batch, hq, dk.head_dim))
    check(kvq_attend_noalloc(dk, dv, q.data_ptr(), hq, k_packed.struct(), tk.struct(), v_packed.struct(),
                             tv.struct(), n_tokens, scale, out.data_ptr(), _stream(stream)), "kvq_attend_noalloc")


def calibrate_workspace(d: kvq_desc, device="cuda") -> torch.Tensor:
    """A workspace tensor for kvq_calibrate_perm."""
    from . import kvq_calibrate_workspace_bytes
    nb = kvq_calibrate_workspace_bytes(d)
    if nb == 0:
        raise ValueError("kvq_calibrate_perm: invalid or unsupported descriptor")
    return torch.empty(nb, dtype=torch.uint8, device=device)


def calibrate_perm(d: kvq_desc, x: torch.Tensor, tb: Tables, perm_out: torch.Tensor = None,
                   workspace: torch.Tensor = None, stream=None) -> torch.Tensor:
    """Channel permutation by abs-max (int16 [H][head_dim]) for kvq_tables.perm."""
    from . import kvq_calibrate_perm
    _req(x, "x", (torch.float16,), _kv_shape(d))
    if perm_out is None:
        perm_out = torch.empty((d.heads, d.head_dim), dtype=torch.int16, device=x.device)
    if workspace is None:
        workspace = calibrate_workspace(d, x.device)
    _req(perm_out, "perm_out", (torch.int16,), (d.heads, d.head_dim))
    check(kvq_calibrate_perm(d, x.data_ptr(), tb.struct(), perm_out.data_ptr(), workspace.data_ptr(),
                             workspace.numel(), _stream(stream)), "kvq_calibrate_perm")
    return perm_out


def calibrate_codebook(d: kvq_desc, x: torch.Tensor, tb: Tables, ch_scale: torch.Tensor = None,
                       ch_wide: torch.Tensor = None, workspace: torch.Tensor = None, stream=None):
    """Dynamic codebook tables (ch_scale f32 [H][D], ch_wide int32 [H][D/32] bit masks) for
    Tables.ch_scale / Tables.ch_wide."""
    from . import kvq_calibrate_codebook, kvq_calibrate_codebook_workspace_bytes
    _req(x, "x", (torch.float16,), _kv_shape(d))
    if ch_scale is None:
        ch_scale = torch.empty((d.heads, d.head_dim), dtype=torch.float32, device=x.device)
    if ch_wide is None:
        ch_wide = torch.empty((d.heads, d.head_dim // 32), dtype=torch.int32, device=x.device)
    if workspace is None:
        nb = kvq_calibrate_codebook_workspace_bytes(d)
        if nb == 0:
            raise ValueError("kvq_calibrate_codebook: invalid or unsupported descriptor")
        workspace = torch.empty(nb, dtype=torch.uint8, device=x.device)
    _req(ch_scale, "ch_scale", (torch.float32,), (d.heads, d.head_dim))
    _req(ch_wide, "ch_wide", (torch.int32,), (d.heads, d.head_dim // 32))
    check(kvq_calibrate_codebook(d, x.data_ptr(), tb.struct(), ch_scale.data_ptr(), ch_wide.data_ptr(),
                                 workspace.data_ptr(), workspace.numel(), _stream(stream)), "kvq_calibrate_codebook")
    return ch_scale, ch_wide


def detect_sinks_workspace(d: kvq_desc, device="cuda") -> torch.Tensor:
    """A workspace tensor for kvq_detect_sinks."""
    from . import kvq_detect_sinks_workspace_bytes
    nb = kvq_detect_sinks_workspace_bytes(d)
    if nb == 0:
        raise ValueError("kvq_detect_sinks: invalid descriptor")
    return torch.empty(nb, dtype=torch.uint8, device=device)


def detect_sinks(d: kvq_desc, x: torch.Tensor, *, tau: float, max_sinks: int, sink_pos: torch.Tensor = None,
                 count: torch.Tensor = None, workspace: torch.Tensor = None, stream=None):
    """Attention sinks by massive activations: (sink_pos int32 [B][max_sinks], ascending
    positions padded with -1, for Tables.sink_pos with n_sink = max_sinks; count int32 [B])."""
    from . import kvq_detect_sinks
    _req(x, "x", (torch.float16,), _kv_shape(d))
    if sink_pos is None:
        sink_pos = torch.empty((d.batch, max_sinks), dtype=torch.int32, device=x.device)
    if count is None:
        count = torch.empty((d.batch,), dtype=torch.int32, device=x.device)
    if workspace is None:
        workspace = detect_sinks_workspace(d, x.device)
    _req(sink_pos, "sink_pos", (torch.int32,), (d.batch, max_sinks))
    _req(count, "count", (torch.int32,), (d.batch,))
    check(kvq_detect_sinks(d, x.data_ptr(), float(tau), int(max_sinks), sink_pos.data_ptr(), count.data_ptr(),
                           workspace.data_ptr(), workspace.numel(), _stream(stream)), "kvq_detect_sinks")
    return sink_pos, count


def bind_detect_sinks(d: kvq_desc, x: torch.Tensor, tau: float, sink_pos: torch.Tensor, count: torch.Tensor,
                      workspace: torch.Tensor, stream=None):
    from . import lib
    _req(x, "x", (torch.float16,), _kv_shape(d))
    _req(sink_pos, "sink_pos", (torch.int32,))
    _req(count, "count", (torch.int32,), (d.batch,))
    if sink_pos.dim() != 2 or sink_pos.shape[0] != d.batch:
        raise ValueError(f"sink_pos: shape {tuple(sink_pos.shape)}, expected ({d.batch}, max_sinks)")
    st = _stream(stream)
    args = (ctypes.byref(d), x.data_ptr(), float(tau), int(sink_pos.shape[1]), sink_pos.data_ptr(),
            count.data_ptr(), workspace.data_ptr(), workspace.numel(), st)
    keep = (d, x, sink_pos, count, workspace)

    def call():
        check(lib.kvq_detect_sinks(*args), "kvq_detect_sinks")
    call.keep = keep
    return call


def pair_energy(d: kvq_desc, x: torch.Tensor, stream=None):
    """Exact RoPE-pair energies (uint64 [H][head_dim/2][2]: low, high words of the count of
    2^-48) and the pairs ranked by descending energy (int16 [H][head_dim/2])."""
    from . import kvq_pair_energy
    _req(x, "x", (torch.float16,), _kv_shape(d))
    energy = torch.empty((d.heads, d.head_dim // 2, 2), dtype=torch.uint64, device=x.device)
    rank = torch.empty((d.heads, d.head_dim // 2), dtype=torch.int16, device=x.device)
    check(kvq_pair_energy(d, x.data_ptr(), energy.data_ptr(), rank.data_ptr(), _stream(stream)), "kvq_pair_energy")
    return energy, rank


def bind_pair_energy(d: kvq_desc, x: torch.Tensor, energy: torch.Tensor, rank: torch.Tensor, stream=None):
    from . import lib
    _req(x, "x", (torch.float16,), _kv_shape(d))
    _req(energy, "energy", (torch.uint64,), (d.heads, d.head_dim // 2, 2))
    _req(rank, "rank", (torch.int16,), (d.heads, d.head_dim // 2))
    st = _stream(stream)
    args = (ctypes.byref(d), x.data_ptr(), energy.data_ptr(), rank.data_ptr(), st)
    keep = (d, x, energy, rank)

    def call():
        check(lib.kvq_pair_energy(*args), "kvq_pair_energy")
    call.keep = keep
    return call


def bind_calibrate(d: kvq_desc, x: torch.Tensor, tb: Tables, perm_out: torch.Tensor, workspace: torch.Tensor,
                   stream=None):
    from . import lib
    _req(x, "x", (torch.float16,), _kv_shape(d))
    _req(perm_out, "perm_out", (torch.int16,), (d.heads, d.head_dim))
    tbs, st = tb.struct(), _stream(stream)
    args = (ctypes.byref(d), x.data_ptr(), ctypes.byref(tbs), perm_out.data_ptr(), workspace.data_ptr(),
            workspace.numel(), st)
    keep = (d, x, tb, tbs, perm_out, workspace)

    def call():
        check(lib.kvq_calibrate_perm(*args), "kvq_calibrate_perm")
    call.keep = keep
    return call


def bind_attend(dk: kvq_desc, dv: kvq_desc, q: torch.Tensor, k_packed: Packed, tk: Tables, v_packed: Packed,
                tv: Tables, n_tokens: int, scale: float, out: torch.Tensor, workspace: torch.Tensor, stream=None):
    from . import lib
    hq = _q_heads(dk, q)
    _req(out, "out", (torch.float32,), (dk.batch, hq, dk.head_dim))
    _req(workspace, "workspace", (torch.uint8,))
    tks, kps, tvs, vps, st = tk.struct(), k_packed.struct(), tv.struct(), v_packed.struct(), _stream(stream)
    args = (ctypes.byref(dk), ctypes.byref(dv), q.data_ptr(), hq, ctypes.byref(kps), ctypes.byref(tks),
            ctypes.byref(vps), ctypes.byref(tvs), n_tokens, ctypes.c_float(scale), out.data_ptr(),
            workspace.data_ptr(), workspace.numel(), st)
    keep = (dk, dv, q, k_packed, tk, v_packed, tv, out, workspace, tks, kps, tvs, vps)

    def call():
        check(lib.kvq_attend(*args), "kvq_attend")
    call.keep = keep
    return call


# ---------------------------------------------------------------- pre-bound calls
# The same marshalling, done once: the returned zero-argument callables hold
# the ctypes structs and raw addresses and launch with no per-call Python
# struct building (for tight loops such as a benchmark or a decode loop).
def bind_encode(d: kvq_desc, x: torch.Tensor, tables: Tables, packed: Packed, stream=None):
    from . import lib
    _req(x, "x", (torch.float16,), _kv_shape(d))
    tb, pk, st = tables.struct(), packed.struct(), _stream(stream)
    args = (ctypes.byref(d), x.data_ptr(), ctypes.byref(tb), ctypes.byref(pk), st)
    keep = (d, x, tables, packed, tb, pk)

    def call():
        check(lib.kvq_encode(*args), "kvq_encode")
    call.keep = keep
    return call


def bind_decode(d: kvq_desc, packed: Packed, tables: Tables, out: torch.Tensor, stream=None):
    from . import lib
    _req(out, "out", (torch.float16, torch.float32), _kv_shape(d))
    tb, pk, st = tables.struct(), packed.struct(), _stream(stream)
    fp32 = 1 if out.dtype == torch.float32 else 0
    args = (ctypes.byref(d), ctypes.byref(pk), ctypes.byref(tb), out.data_ptr(), fp32, st)
    keep = (d, packed, tables, out, tb, pk)

    def call():
        check(lib.kvq_decode(*args), "kvq_decode")
    call.keep = keep
    return call


def bind_score(d: kvq_desc, q: torch.Tensor, packed: Packed, tables: Tables, n_tokens: int, scale: float,
               out: torch.Tensor, stream=None, literal: bool = False):
    """A prepared kvq_score call (kvq_score_literal with literal=True)."""
    from . import lib
    hq = _q_heads(d, q)
    _req(out, "scores", (torch.float32,), (d.batch, hq, n_tokens))
    tb, pk, st = tables.struct(), packed.struct(), _stream(stream)
    args = (ctypes.byref(d), q.data_ptr(), hq, ctypes.byref(pk), ctypes.byref(tb), n_tokens,
            ctypes.c_float(scale), out.data_ptr(), st)
    keep = (d, q, packed, tables, out, tb, pk)

    fn, name = (lib.kvq_score_literal, "kvq_score_literal") if literal else (lib.kvq_score, "kvq_score")

    def call():
        check(fn(*args), name)
    call.keep = keep
    return call
