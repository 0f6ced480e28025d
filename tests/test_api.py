"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates arguments before launching anything, sizes the
packed buffers, and its host helpers agree with the oracle's own tables."""
import ctypes
import os
import re

import numpy as np
import pytest

import kv_cache_rotation_b200 as K
from kv_cache_rotation_b200 import torch_api as TA

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert set(names) == set(K.EXPORTED)
    lib = ctypes.CDLL(K.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings():
    assert K.kvq_version() >= 100
    for s in range(6):
        assert K.kvq_status_str(s)


def _desc(**kw):
    base = dict(batch=2, heads=8, tokens=16, bits=2, group=64, rope=0)
    base.update(kw)
    return TA.make_desc(**base)


def _packed(d, codes=256, sz=256, sink=0, norm=0):
    p = K.kvq_packed()
    p.codes, p.scale_zero, p.sink, p.norm = codes, sz, sink or None, norm or None
    return p


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), K.KVQ_ERR_INVALID),
    (dict(heads=-1), K.KVQ_ERR_INVALID),
    (dict(tokens=-1), K.KVQ_ERR_INVALID),
    (dict(t0=10, t_cap=20, tokens=16), K.KVQ_ERR_INVALID),
    (dict(bits=5), K.KVQ_ERR_UNSUPPORTED),
    (dict(bits=1), K.KVQ_ERR_UNSUPPORTED),
    (dict(head_dim=96), K.KVQ_ERR_UNSUPPORTED),
    (dict(group=48), K.KVQ_ERR_UNSUPPORTED),
    (dict(head_dim=64, group=128), K.KVQ_ERR_INVALID),
    (dict(rot="fwht_group", group_heads=3), K.KVQ_ERR_UNSUPPORTED),
    (dict(rot="fwht_group", group_heads=8, heads=12), K.KVQ_ERR_INVALID),
    (dict(rot="fwht_group", group_heads=8, head_dim=64), K.KVQ_ERR_UNSUPPORTED),
    (dict(rot="iso", quant="minmax"), K.KVQ_ERR_UNSUPPORTED),
    (dict(rot="fwht_head", quant="codebook"), K.KVQ_ERR_UNSUPPORTED),
    (dict(rope=2), K.KVQ_ERR_INVALID),
    (dict(rot=9), K.KVQ_ERR_INVALID),
])
def test_encode_rejects_bad_desc(kw, status):
    d = _desc(**kw)
    tb = K.kvq_tables()
    assert K.kvq_encode(d, 256, tb, _packed(d), 0) == status
    assert K.kvq_decode(d, _packed(d), tb, 256, 0, 0) == status


def test_null_and_alignment_checks():
    d = _desc()
    tb = K.kvq_tables()
    assert K.kvq_encode(d, None, tb, _packed(d), 0) == K.KVQ_ERR_INVALID
    assert K.kvq_encode(d, 258, tb, _packed(d), 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_encode(d, 256, tb, _packed(d, codes=0), 0) == K.KVQ_ERR_INVALID
    assert K.kvq_encode(d, 256, tb, _packed(d, codes=264), 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_encode(d, 256, tb, _packed(d, sz=0), 0) == K.KVQ_ERR_INVALID
    assert K.lib.kvq_encode(None, 256, ctypes.byref(tb), ctypes.byref(_packed(d)), None) == K.KVQ_ERR_INVALID
    ds = _desc(n_sink=4)
    assert K.kvq_encode(ds, 256, tb, _packed(ds), 0) == K.KVQ_ERR_INVALID  # sinks need a buffer
    dr = _desc(rope=1)
    assert K.kvq_encode(dr, 256, tb, _packed(dr), 0) == K.KVQ_ERR_INVALID  # rope needs the table
    tb.rope_cs, tb.rope_rows = 256, 8  # too few rows for t0 + T = 16
    assert K.kvq_encode(dr, 256, tb, _packed(dr), 0) == K.KVQ_ERR_INVALID
    tb.rope_cs, tb.rope_rows = 260, 64
    assert K.kvq_encode(dr, 256, tb, _packed(dr), 0) == K.KVQ_ERR_ALIGN
    di = _desc(rot="iso", quant="codebook", bits=3)
    assert K.kvq_encode(di, 256, K.kvq_tables(), _packed(di, norm=256), 0) == K.KVQ_ERR_INVALID
    assert K.kvq_decode(d, _packed(d), K.kvq_tables(), 256, 2, 0) == K.KVQ_ERR_INVALID


def test_score_argument_checks():
    d = _desc(t_cap=32, tokens=0)
    tb = K.kvq_tables()
    p = _packed(d)
    assert K.kvq_score(d, 256, 12, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_INVALID  # 12 % 8
    assert K.kvq_score(d, 256, 8, p, tb, 33, 1.0, 256, 0) == K.KVQ_ERR_INVALID  # > t_cap
    assert K.kvq_score(d, 258, 8, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_ALIGN
    dg = _desc(t_cap=32, rot="fwht_group", group_heads=8, group=128)
    assert K.kvq_score(dg, 256, 8, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_UNSUPPORTED
    assert K.kvq_score(d, 256, 8, p, tb, 0, 1.0, 256, 0) == K.KVQ_OK  # empty: nothing to do


def test_score_literal_argument_checks():
    d = _desc(t_cap=32, tokens=0, head_dim=128)
    tb = K.kvq_tables()
    p = _packed(d)
    f = K.kvq_score_literal
    assert K.lib.kvq_score_literal(None, 256, 8, ctypes.byref(p), ctypes.byref(tb), 16, ctypes.c_float(1.0), 256,
                                   None) == K.KVQ_ERR_INVALID
    assert f(d, 256, 12, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_INVALID  # 12 % 8
    assert f(d, 256, 24, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_UNSUPPORTED  # 3 query heads per KV head
    assert f(d, 256, 8, p, tb, 33, 1.0, 256, 0) == K.KVQ_ERR_INVALID  # > t_cap
    assert f(d, 258, 8, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_ALIGN
    assert f(d, 256, 8, p, tb, 16, 1.0, 260, 0) == K.KVQ_ERR_ALIGN
    assert f(_desc(t_cap=32, tokens=0, head_dim=64, group=32), 256, 8, p, tb, 16, 1.0, 256, 0) == \
        K.KVQ_ERR_UNSUPPORTED
    dg = _desc(t_cap=32, rot="fwht_group", group_heads=8, group=128)
    assert f(dg, 256, 8, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_UNSUPPORTED
    di = _desc(t_cap=32, tokens=0, rot="iso", quant="codebook", bits=3)
    assert f(di, 256, 8, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_UNSUPPORTED
    assert f(d, 256, 8, p, tb, 0, 1.0, 256, 0) == K.KVQ_OK  # empty: nothing to do


def test_attend_argument_checks():
    dk = _desc(t_cap=32, tokens=0, rope=1)
    dv = _desc(t_cap=32, tokens=0, rope=0)
    tb = K.kvq_tables()
    p = _packed(dk)
    ws = K.kvq_attend_workspace_bytes(dk, dv, 16, 20)
    assert ws > 0
    assert K.kvq_attend_workspace_bytes(dk, dv, 12, 20) == 0  # 12 % 8
    assert K.kvq_attend_workspace_bytes(dk, dv, 8 * 16, 20) == 0  # 16 query heads per KV head
    assert K.kvq_attend(dk, dv, 256, 16, p, tb, p, tb, 33, 1.0, 256, 256, ws, 0) == K.KVQ_ERR_INVALID  # > t_cap
    assert K.kvq_attend(dk, dv, 256, 16, p, tb, p, tb, 0, 1.0, 256, 256, ws, 0) == K.KVQ_ERR_INVALID  # no token
    assert K.kvq_attend(dk, dv, 256, 16, p, tb, p, tb, 20, 1.0, 256, 256, ws - 1, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_attend(dk, dv, 256, 16, p, tb, p, tb, 20, 1.0, 256, 512 + 16, ws, 0) == K.KVQ_ERR_ALIGN
    dvr = _desc(t_cap=32, tokens=0, rope=1)
    assert K.kvq_attend(dk, dvr, 256, 16, p, tb, p, tb, 20, 1.0, 256, 256, ws, 0) == K.KVQ_ERR_UNSUPPORTED
    dv4 = _desc(t_cap=32, tokens=0, rope=0, bits=4)
    assert K.kvq_attend(dk, dv4, 256, 16, p, tb, p, tb, 20, 1.0, 256, 256, ws, 0) == K.KVQ_ERR_INVALID


def test_attend_workspace_covers_both_sink_forms():
    """Up to 32 sinks both forms take the same path; above that a list runs the
    three-kernel form, so the workspace covers the larger of the two layouts."""
    def ws(n_sink, group=128, n=4097):
        dk = _desc(batch=4, heads=8, t_cap=n, tokens=0, rope=1, group=group, n_sink=n_sink)
        dv = _desc(batch=4, heads=8, t_cap=n, tokens=0, rope=0, group=group, n_sink=n_sink)
        return K.kvq_attend_workspace_bytes(dk, dv, 32, n)

    def a256(x):
        return (x + 255) // 256 * 256
    bq, n, d = 4 * 32, 4097, 128
    chunks_f = min((n + 15) // 16, 256)  # fused: 16-token tiles, at most 256 chunks per query head
    fused = a256(bq * chunks_f * d * 4) + a256(bq * chunks_f * 2 * 4)
    chunks_u = (n + 511) // 512  # three kernels: scores, then 512-token chunks
    three = a256(bq * n * 4) + a256(bq * chunks_u * d * 4) + a256(bq * chunks_u * 2 * 4)
    assert ws(4) == fused and ws(32) == fused
    assert ws(40) == max(fused, three)
    assert ws(4, group=64) == three and ws(40, group=64) == three


def test_attend_sink_list_in_both_tables():
    dk = _desc(t_cap=32, tokens=0, rope=1, n_sink=2)
    dv = _desc(t_cap=32, tokens=0, rope=0, n_sink=2)
    p = _packed(dk, sink=4096)
    ws = K.kvq_attend_workspace_bytes(dk, dv, 16, 20)
    tk, tv = K.kvq_tables(), K.kvq_tables()
    tk.rope_cs, tk.rope_rows = 256, 32
    tk.sink_pos = 1024  # keys listed, values not
    assert K.kvq_attend(dk, dv, 256, 16, p, tk, p, tv, 20, 1.0, 256, 256, ws, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_attend_noalloc(dk, dv, 256, 16, p, tk, p, tv, 20, 1.0, 256, 0) == K.KVQ_ERR_INVALID
    tv.sink_pos = 1024
    tk.rope_rows = 8  # a list needs RoPE rows up to n_tokens
    assert K.kvq_attend(dk, dv, 256, 16, p, tk, p, tv, 20, 1.0, 256, 256, ws, 0) == K.KVQ_ERR_INVALID
    tk.sink_pos = 1026  # 4-byte alignment
    tk.rope_rows = 32
    assert K.kvq_attend(dk, dv, 256, 16, p, tk, p, tv, 20, 1.0, 256, 256, ws, 0) == K.KVQ_ERR_ALIGN


def test_attend_noalloc_rejects_oversize():
    # 8 sequences x 64 query heads x 32768 tokens: 67 MB of scores alone, more than the 40 MiB scratch
    dk = _desc(batch=8, heads=8, t_cap=32768, tokens=0, rope=0)
    dv = _desc(batch=8, heads=8, t_cap=32768, tokens=0, rope=0)
    assert K.kvq_attend_workspace_bytes(dk, dv, 64, 32768) > (40 << 20)
    p, tb = _packed(dk), K.kvq_tables()
    assert K.kvq_attend_noalloc(dk, dv, 256, 64, p, tb, p, tb, 32768, 1.0, 256, 0) == K.KVQ_ERR_UNSUPPORTED
    assert K.kvq_attend_noalloc(dk, dv, 258, 64, p, tb, p, tb, 16, 1.0, 256, 0) == K.KVQ_ERR_ALIGN


def test_empty_call_is_a_noop():
    d = _desc(tokens=0, t_cap=4)
    assert K.kvq_encode(d, 256, K.kvq_tables(), _packed(d), 0) == K.KVQ_OK
    assert K.kvq_decode(d, _packed(d), K.kvq_tables(), 256, 1, 0) == K.KVQ_OK


def test_packed_bytes_and_compression_ratios():
    """Bytes per 128-channel fp16 vector (256 B) of each format, and the
    resulting compression ratios: 4-bit G128 68 B (3.76x), 2-bit G64 40 B
    (6.4x), 2-bit G128 36 B (7.11x), 3-bit codebook + fp32 norm 52 B (4.92x)."""
    for kw, per_vec in ((dict(bits=4, group=128), 68), (dict(bits=2, group=64), 40),
                        (dict(bits=2, group=128), 36), (dict(bits=3, rot="iso", quant="codebook"), 52)):
        d = _desc(batch=3, heads=5, tokens=7, t_cap=11, head_dim=128, **kw)
        tot = sum(K.kvq_packed_bytes(d, f) for f in (0, 1, 3))
        assert tot == 3 * 5 * 11 * per_vec
    d = _desc(n_sink=4, t_cap=16)
    assert K.kvq_packed_bytes(d, K.KVQ_FIELD_SINK) == 2 * 8 * 4 * 128 * 2
    assert K.kvq_packed_bytes(d, 7) == 0
    assert K.kvq_packed_bytes(_desc(bits=9), 0) == 0


def test_rope_table_matches_oracle(orc):
    import torch
    cs = TA.rope_table(40000, 128, device="cpu").numpy()
    for m in (0, 1, 777, 32768, 39999):
        c, s = orc.rope_cs(m, 128)
        assert np.array_equal(cs[m, :, 0], c) and np.array_equal(cs[m, :, 1], s)
    assert K.kvq_rope_table(None, 4, 128, 10000.0) == K.KVQ_ERR_INVALID
    assert K.kvq_rope_table(torch.empty(8).data_ptr(), 4, 127, 10000.0) == K.KVQ_ERR_INVALID


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_codebook_matches_oracle(orc, bits):
    cb = TA.lloyd_max_codebook(bits, 128, device="cpu").numpy()
    assert np.array_equal(cb, orc.codebook(bits, 128))


def test_calibrate_argument_checks():
    d = _desc(tokens=40, rope=1)
    nb = K.kvq_calibrate_workspace_bytes(d)
    assert nb == 8 * 128 * 4  # the fp32 maxima of 8 heads x 128 channels
    tb = K.kvq_tables()
    tb.rope_cs, tb.rope_rows = 256, 40
    ok = (256, tb, 512, 1024, nb, 0)
    assert K.kvq_calibrate_perm(_desc(batch=0), *ok) == K.KVQ_ERR_INVALID
    assert K.kvq_calibrate_perm(d, 0, tb, 512, 1024, nb, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_calibrate_perm(d, 258, tb, 512, 1024, nb, 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_calibrate_perm(d, 256, tb, 514, 1024, nb, 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_calibrate_perm(d, 256, tb, 512, 1040, nb, 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_calibrate_perm(d, 256, tb, 512, 1024, nb - 4, 0) == K.KVQ_ERR_INVALID
    short = K.kvq_tables()
    short.rope_cs, short.rope_rows = 256, 39  # positions 0..39 need 40 rows
    assert K.kvq_calibrate_perm(d, 256, short, 512, 1024, nb, 0) == K.KVQ_ERR_INVALID
    iso = _desc(rot="iso", quant="codebook", bits=3, group=128)
    assert K.kvq_calibrate_workspace_bytes(iso) == 0
    assert K.kvq_calibrate_perm(iso, 256, tb, 512, 1024, nb, 0) == K.KVQ_ERR_UNSUPPORTED
    # grouped keys permute the raw input: no RoPE table needed
    g = _desc(tokens=40, rope=1, rot="fwht_group", group_heads=8, group=128)
    assert K.kvq_calibrate_workspace_bytes(g) == nb


def test_pair_energy_argument_checks():
    d = _desc(tokens=40)
    assert K.kvq_pair_energy(_desc(batch=0), 256, 512, 1024, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_pair_energy(d, 0, 512, 1024, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_pair_energy(d, 264, 512, 1024, 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_pair_energy(d, 256, 520, 1024, 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_pair_energy(d, 256, 512, 1032, 0) == K.KVQ_ERR_ALIGN


@pytest.mark.parametrize("d", [16, 64, 128])
def test_freq_aware_rope_table_matches_oracle(orc, d):
    import torch
    cs = TA.rope_table(40000, d, device="cpu", freq=K.KVQ_ROPE_FREQ_AWARE).numpy()
    for m in (0, 1, 777, 32768, 39999):
        c, s = orc.rope_cs(m, d, mode=orc.ROPE_FREQ_AWARE)
        assert np.array_equal(cs[m, :, 0], c) and np.array_equal(cs[m, :, 1], s)
    buf = torch.empty(4 * 12).data_ptr()
    assert K.kvq_rope_table_ex(buf, 4, 12, 10000.0, K.KVQ_ROPE_FREQ_AWARE) == K.KVQ_ERR_INVALID  # not a multiple of 8
    assert K.kvq_rope_table_ex(buf, 4, 8, 10000.0, 7) == K.KVQ_ERR_INVALID


def test_sink_and_codebook_entry_point_checks():
    """Argument checks of the detection, sink-list and dynamic-codebook entry
    points (all host-side: nothing is launched)."""
    d = _desc(head_dim=64, group=64)
    ws_need = K.kvq_detect_sinks_workspace_bytes(d)
    assert ws_need == (2 * 16 * 2 + 15) // 16 * 16
    assert K.kvq_detect_sinks(d, None, 2.0, 4, 256, 0, 256, ws_need, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks(d, 256, float("nan"), 4, 256, 0, 256, ws_need, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks(d, 256, 2.0, 0, 256, 0, 256, ws_need, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks(d, 256, 2.0, 70000, 256, 0, 256, ws_need, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks(d, 256, 2.0, 4, 256, 0, 256, ws_need - 16, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks(d, 264, 2.0, 4, 256, 0, 256, ws_need, 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_detect_sinks(d, 256, 2.0, 4, 258, 0, 256, ws_need, 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_detect_sinks(_desc(tokens=0), 256, 2.0, 4, 256, 0, 256, 64, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_detect_sinks_workspace_bytes(_desc(batch=0)) == 0
    # a sink list must be 4-byte aligned
    tb = K.kvq_tables()
    tb.sink_pos = 258
    ds = _desc(n_sink=2)
    assert K.kvq_encode(ds, 256, tb, _packed(ds, sink=256), 0) == K.KVQ_ERR_ALIGN
    # dynamic codebooks: IsoQuant rotations only; tables and the ext field required
    dd = _desc(rot="iso", quant="codebook_dyn", bits=3)
    assert K.kvq_calibrate_codebook_workspace_bytes(_desc()) == 0  # not an IsoQuant rotation
    nb = K.kvq_calibrate_codebook_workspace_bytes(dd)
    assert nb >= 2 * 8 * 1 * 128 * 8
    t = K.kvq_tables()
    assert K.kvq_calibrate_codebook(dd, 256, t, 256, 256, 256, nb, 0) == K.KVQ_ERR_INVALID  # no qL/qR
    t.qL, t.qR = 256, 256
    assert K.kvq_calibrate_codebook(dd, 256, t, 256, 256, 256, nb - 8, 0) == K.KVQ_ERR_INVALID
    assert K.kvq_calibrate_codebook(dd, 256, t, 260, 256, 256, nb, 0) == K.KVQ_ERR_ALIGN
    assert K.kvq_calibrate_codebook(_desc(), 256, t, 256, 256, 256, nb, 0) == K.KVQ_ERR_UNSUPPORTED
    t.codebook = 256
    p = _packed(dd, norm=256)
    assert K.kvq_encode(dd, 256, t, p, 0) == K.KVQ_ERR_INVALID  # no wide codebook / scales / masks
    t.codebook_wide, t.ch_scale, t.ch_wide = 256, 256, 256
    assert K.kvq_encode(dd, 256, t, p, 0) == K.KVQ_ERR_INVALID  # no ext field
    assert K.kvq_packed_bytes(dd, K.KVQ_FIELD_EXT) == 2 * 8 * 16 * 2
    assert K.kvq_packed_bytes(_desc(), K.KVQ_FIELD_EXT) == 0
    assert K.kvq_lloyd_max_codebook(np.zeros(32, np.float32).ctypes.data, 5, 1) == K.KVQ_OK
    assert K.kvq_lloyd_max_codebook(np.zeros(64, np.float32).ctypes.data, 6, 1) == K.KVQ_ERR_INVALID


@pytest.mark.parametrize("bits", [2, 3, 4, 5])
def test_unit_normal_codebook_matches_oracle(orc, bits):
    """The N(0,1) levels (head_dim 1) that the dynamic codebooks scale, up to
    the 5-bit wide codebook of 4-bit codes, bit-equal to the oracle's."""
    host = np.zeros(1 << bits, np.float32)
    assert K.kvq_lloyd_max_codebook(host.ctypes.data, bits, 1) == K.KVQ_OK
    assert np.array_equal(host, orc.codebook(bits, 1))
