"""Seeded synthetic inputs and workload definitions.

This module is shared by the tests, the smoke check and the benchmark. It
holds only shapes, parameters and seeded random draws (numpy PCG64) -- none
of the method's arithmetic -- so that the CUDA path and the CPU oracle can
consume identical bytes while sharing no code.

Distributions follow the workloads described on the pages: fp16 K/V drawn
from N(0,1) with a few strongly scaled outlier channels (the channel-wise
outliers that motivate the outlier-aware rotation of "RotateKV: Accurate and
Robust 2-Bit KV Cache Quantization for LLMs via Outlier-Aware Adaptive
Rotations", abstract), heavy-tailed Student-t vectors for the IsoQuant batch
("KV缓存压缩技术：IsoQuant在大语言模型中的应用", §7: batch 8192, d = 128), and
seeded unit quaternions for its 4-D blocks (§2.1). No dataset is used.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np

_CHUNK = 1 << 24  # elements drawn per numpy call (bounds host memory)


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int  # tokens encoded (prefill) / cache slots for scoring
    D: int = 128
    rot: str = "fwht_head"  # none | fwht_head | fwht_group | iso
    quant: str = "minmax"  # minmax | codebook
    bits: int = 2
    group: int = 128
    group_heads: int = 1
    rope_k: bool = True
    n_sink: int = 0
    perm: bool = False
    dist: str = "normal_outliers"  # normal_outliers | student_t
    outliers: tuple = ("pairs", 0.01, 10.0, 50.0)
    seed: int = 0
    Hq: int = 0  # query heads for scoring (0: no score)
    append: int = 0  # tokens appended after the prefill (decode step)
    extra: dict = field(default_factory=dict)

    @property
    def n_vectors(self) -> int:
        return self.B * self.H * self.T


WORKLOADS = {
    # 1 layer, batch 1, 8 heads x 128, 256 tokens; 4 outlier channels x20 per
    # head; FWHT over head_dim; 4-bit min-max, group 128.
    "tiny": Workload("tiny", B=1, H=8, T=256, bits=4, group=128, outliers=("per_head", 4, 20.0, 20.0),
                     seed=1),
    # Llama-2-7B-shaped MHA layer: batch 8, 32 heads, 4096 tokens; 1 % of the
    # (head, channel) pairs scaled by U[10, 50]; abs-max permutation; 2-bit
    # group 64; first 4 tokens kept in fp16.
    "llama2_7b_mha": Workload("llama2_7b_mha", B=8, H=32, T=4096, bits=2, group=64, n_sink=4, perm=True,
                              seed=2),
    # Llama-3-8B-shaped GQA layer: batch 4, 8 KV heads, 32768 tokens; FWHT
    # over the 8 heads x 128 = 1024 channels before RoPE; 2-bit group 128.
    "llama3_8b_gqa": Workload("llama3_8b_gqa", B=4, H=8, T=32768, rot="fwht_group", group_heads=8, bits=2,
                              group=128, seed=3),
    # IsoQuant-style batch: 8192 x 2048 vectors of d = 128, Student-t(4);
    # 3-bit Lloyd-Max codebook for N(0, 1/128).
    "isoquant_batch": Workload("isoquant_batch", B=8192, H=1, T=2048, rot="iso", quant="codebook", bits=3,
                               rope_k=False, dist="student_t", seed=4),
    # The same batch through the 3-D sandwich q v q* (3-channel blocks, a
    # 2-channel tail turned in its plane).
    "isoquant_so3_batch": Workload("isoquant_so3_batch", B=8192, H=1, T=2048, rot="iso3", quant="codebook",
                                   bits=3, rope_k=False, dist="student_t", seed=4),
    # The IsoQuant batch with dynamic codebooks, on keys with outlier
    # channels (3 % of the channels scaled by U[10, 50], the channel-wise
    # outliers the per-channel statistics are for): 3-bit, SO(4) blocks.
    "isoquant_dyn_batch": Workload("isoquant_dyn_batch", B=8192, H=1, T=2048, rot="iso", quant="codebook_dyn",
                                   bits=3, rope_k=False, outliers=("pairs", 0.03, 10.0, 50.0), seed=5),
    # Decode step: batch 64, 32 heads, 8192-token 2-bit cache encoded as in
    # the Llama-2-7B workload, plus one appended token; fp32 scores.
    "decode_score": Workload("decode_score", B=64, H=32, T=8192, bits=2, group=64, n_sink=4, perm=True,
                             seed=5, Hq=32, append=1),
    # Decode step at the Llama-3-8B shape: 8 KV heads, 32 query heads (GQA
    # 4:1), 32768 cached tokens + 1 appended, head-dim FWHT, 2-bit group 128.
    "llama3_8b_gqa_score": Workload("llama3_8b_gqa_score", B=4, H=8, T=32768, bits=2, group=128, n_sink=4,
                                    seed=6, Hq=32, append=1),
    # Decode-step attention at the same shape: K and V caches (values without
    # RoPE), one token appended to each, then softmax(q . k) . v.
    "llama3_8b_gqa_attend": Workload("llama3_8b_gqa_attend", B=4, H=8, T=32768, bits=2, group=128, n_sink=4,
                                     seed=7, Hq=32, append=1),
    # Decode-step attention at the Llama-2-7B shape (32 heads, MHA, 4096 cached
    # tokens + 1, 2-bit group 64, permutation, 4 sinks): two groups per record,
    # so the three-kernel form (scores, chunked sums, merge).
    "llama2_7b_mha_attend": Workload("llama2_7b_mha_attend", B=8, H=32, T=4096, bits=2, group=64, n_sink=4,
                                     perm=True, seed=8, Hq=32, append=1),
}


def scaled(w: Workload, **kw) -> Workload:
    """Same workload with some fields replaced (e.g. fewer tokens)."""
    return replace(w, **kw)


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream]))


def _normal_f16(rng, n: int) -> np.ndarray:
    out = np.empty(n, np.float16)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = rng.standard_normal(e - s, dtype=np.float32)
    return out


def _student_f16(rng, n: int, nu: float) -> np.ndarray:
    out = np.empty(n, np.float16)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        out[s:e] = rng.standard_t(nu, e - s)
    return out


def outlier_scales(H: int, D: int, spec, rng) -> np.ndarray:
    """[H][D] float32 multipliers (1 for ordinary channels)."""
    sc = np.ones((H, D), np.float32)
    kind = spec[0]
    if kind == "per_head":  # k channels per head, fixed factor
        _, k, lo, hi = spec
        for h in range(H):
            ch = rng.choice(D, size=k, replace=False)
            sc[h, ch] = rng.uniform(lo, hi, size=k) if hi > lo else lo
    elif kind == "pairs":  # a fraction of all (head, channel) pairs, U[lo, hi]
        _, frac, lo, hi = spec
        k = int(math.ceil(frac * H * D))
        idx = rng.choice(H * D, size=k, replace=False)
        sc.reshape(-1)[idx] = rng.uniform(lo, hi, size=k).astype(np.float32)
    elif kind == "none":
        pass
    else:
        raise ValueError(kind)
    return sc


def kv_tensor(w: Workload, which: str, T: Optional[int] = None, B: Optional[int] = None) -> np.ndarray:
    """fp16 [B][H][T][D] tensor for K ('k'), V ('v') or the tokens appended
    after a prefill ('k_append', 'v_append'; same outlier channels as K / V).
    A smaller T or B draws a smaller tensor with the same recipe."""
    T = w.T if T is None else T
    B = w.B if B is None else B
    stream = {"k": 1, "v": 2, "k_append": 3, "v_append": 4}[which]
    rng = _rng(w.seed, stream)
    n = B * w.H * T * w.D
    if w.dist == "student_t":
        x = _student_f16(rng, n, 4.0).reshape(B, w.H, T, w.D)
        return x
    x = _normal_f16(rng, n).reshape(B, w.H, T, w.D)
    sc = outlier_scales(w.H, w.D, w.outliers, _rng(w.seed, 10 + stream % 2))
    for h, c in zip(*np.nonzero(sc != 1.0)):
        x[:, h, :, c] = (x[:, h, :, c].astype(np.float32) * sc[h, c]).astype(np.float16)
    return x


def queries(w: Workload, B: Optional[int] = None) -> np.ndarray:
    """fp16 [B][Hq][D] query vectors, N(0,1) (taken as already RoPE'd)."""
    B = w.B if B is None else B
    rng = _rng(w.seed, 20)
    return _normal_f16(rng, B * w.Hq * w.D).reshape(B, w.Hq, w.D)


def unit_quaternions(n: int, seed: int, stream: int) -> np.ndarray:
    """[n][4] float32 (real, i, j, k): 4 iid N(0,1) normalised in float64."""
    g = _rng(seed, stream).standard_normal((n, 4))
    g /= np.linalg.norm(g, axis=1, keepdims=True)
    return g.astype(np.float32)


def iso_tables(w: Workload):
    """(qL, qR) for the IsoQuant rotation: one unit quaternion pair per 4-D block."""
    return unit_quaternions(w.D // 4, w.seed, 30), unit_quaternions(w.D // 4, w.seed, 31)


def iso3_tables(D: int, seed: int) -> np.ndarray:
    """[ceil(D/3)][4] float32 unit quaternions (real, i, j, k) for the 3-D
    sandwich: one per 3-channel block, drawn like unit_quaternions; when D mod
    3 = 2 the last entry, for the 2-channel tail, has zero i and j parts
    (real and k drawn N(0,1), normalised in float64)."""
    nb = D // 3
    n = nb + (1 if D % 3 else 0)
    g = _rng(seed, 32).standard_normal((n, 4))
    if D % 3 == 2:
        g[nb, 1:3] = 0.0
    g /= np.linalg.norm(g, axis=1, keepdims=True)
    return g.astype(np.float32)


def plant_massive(x: np.ndarray, n_tokens: int, seed: int, lo: float = 2000.0, hi: float = 6000.0,
                  head_frac: float = 0.25):
    """Massive activations on a few tokens, in place (the attention-sink tokens
    of "RotateKV: Accurate and Robust 2-Bit KV Cache Quantization for LLMs via
    Outlier-Aware Adaptive Rotations", abstract (iii)): per sequence, token 0
    and n_tokens - 1 other tokens drawn uniformly get, in a random quarter of
    the heads, one random channel set to +-U[lo, hi] (fp16). Returns the
    planted token indices per sequence (sorted)."""
    B, H, T, D = x.shape
    rng = _rng(seed, 50)
    planted = []
    for b in range(B):
        extra = rng.choice(np.arange(1, T), size=min(n_tokens - 1, T - 1), replace=False) if T > 1 else []
        toks = sorted({0, *[int(t) for t in extra]})
        for t in toks:
            heads = rng.choice(H, size=max(1, int(round(head_frac * H))), replace=False)
            for h in heads:
                c = int(rng.integers(D))
                x[b, h, t, c] = np.float16(rng.uniform(lo, hi) * (1 if rng.random() < 0.5 else -1))
        planted.append(toks)
    return planted


def random_perm(H: int, D: int, seed: int) -> np.ndarray:
    """[H][D] int16, a seeded random permutation per head (any permutation
    exercises the permutation step; calibrated ones are computed elsewhere)."""
    rng = _rng(seed, 40)
    return np.stack([rng.permutation(D) for _ in range(H)]).astype(np.int16)


def positions(t0: int, T: int) -> np.ndarray:
    return np.arange(t0, t0 + T, dtype=np.int64)


def kv_tensor_device(w: Workload, which: str, device, T: Optional[int] = None, B: Optional[int] = None):
    """Large tensors drawn on the GPU with torch's seeded generator (same
    recipe as kv_tensor, different stream): fp16 [B][H][T][D]. Student-t(4)
    is z0 / sqrt((z1^2 + z2^2 + z3^2 + z4^2) / 4) with iid standard normals."""
    import torch
    T = w.T if T is None else T
    B = w.B if B is None else B
    stream = {"k": 1, "v": 2, "k_append": 3, "v_append": 4}[which]
    g = torch.Generator(device=device)
    g.manual_seed(w.seed * 1000 + stream)
    n = B * w.H * T * w.D
    out = torch.empty(n, dtype=torch.float16, device=device)
    chunk = 1 << 25
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        if w.dist == "student_t":
            z = torch.randn((5, e - s), generator=g, device=device)
            out[s:e] = (z[0] / torch.sqrt((z[1:] ** 2).sum(0) / 4.0)).half()
        else:
            out[s:e] = torch.randn(e - s, generator=g, device=device).half()
    out = out.view(B, w.H, T, w.D)
    if w.dist != "student_t":
        sc = outlier_scales(w.H, w.D, w.outliers, _rng(w.seed, 10 + stream % 2))
        for h, c in zip(*np.nonzero(sc != 1.0)):
            out[:, h, :, c] = (out[:, h, :, c].float() * float(sc[h, c])).half()
    return out
