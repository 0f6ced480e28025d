"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and compare them with the rules
below.

Codes: bit-exact, except that a code may differ by one level where the
oracle's pre-quantization value lies within 1e-5 (relative) of the decision
boundary between the two levels; such excused elements may be at most 1e-4
of all elements. fp16 scale/zero and sinks: bit-exact.
Reconstruction: max-abs 1e-3 against the oracle's fp64 decode of the same
codes (the GPU's), and the fp16 output equals the fp32 output rounded.
Scores: |s_gpu - s_orc| <= 1e-3 * scale * sum_j |q_j khat_j| (relative error
in the L1 magnitude of the dot product; fp32 accumulation on the GPU).
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass

import numpy as np

EXCUSE_REL = 1e-5
EXCUSE_FRAC = 1e-4
RECON_ABS = 1e-3
# Rows of extreme magnitude (edge-case tests only): fp32 rounding in the
# inverse transform is ~2^-24 * sqrt(log2 N) * ||x_row||, so those rows get
# RECON_ABS + RECON_ROW_REL * ||x_row||_2 instead of the plain 1e-3.
RECON_ROW_REL = 2.0 ** -20
SCORE_REL = 1e-3

ORC_ROT = {"none": 0, "fwht_head": 1, "fwht_group": 2, "iso": 3}
ORC_Q = {"minmax": 0, "codebook": 1}


@dataclass
class CodeReport:
    n: int
    mismatched: int
    excused: int
    unexcused: int
    sz_mismatch: int

    @property
    def ok(self) -> bool:
        return self.unexcused == 0 and self.sz_mismatch == 0 and self.excused <= EXCUSE_FRAC * self.n


# Every code comparison made in this process, as (test id, CodeReport): the
# session summary (conftest.py) prints the mismatched and excused counts per
# test, so the excused fraction is reported, not only bounded.
REPORTS = []


def _record(rep: "CodeReport") -> "CodeReport":
    REPORTS.append((os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0], rep))
    return rep


def unpack_all(codes: np.ndarray, D: int, bits: int) -> np.ndarray:
    """[..., D*bits/8] bytes -> [..., D] codes (LSB-first bit stream)."""
    flat = codes.reshape(-1, D * bits // 8)
    bitsarr = np.unpackbits(flat, axis=1, bitorder="little")  # [N, D*bits]
    bitsarr = bitsarr.reshape(-1, D, bits).astype(np.uint32)
    w = (1 << np.arange(bits, dtype=np.uint32))
    return (bitsarr * w).sum(axis=2).astype(np.uint8).reshape(*codes.shape[:-1], D)


def compare_minmax(gpu_codes, orc_codes, gpu_sz, orc_sz, pre, D, bits, group) -> CodeReport:
    cg = unpack_all(gpu_codes, D, bits).astype(np.int32)
    co = unpack_all(orc_codes, D, bits).astype(np.int32)
    szm = int(np.sum(np.any(gpu_sz.view(np.uint16) != orc_sz.view(np.uint16), axis=-1)))
    diff = cg != co
    n_mis = int(diff.sum())
    exc = 0
    if n_mis:
        ng = D // group
        S = orc_sz[..., 0].view(np.float16).astype(np.float64)
        Z = orc_sz[..., 1].view(np.float16).astype(np.float64)
        S = np.repeat(S.reshape(*S.shape[:-1], ng, 1), group, axis=-1).reshape(cg.shape)
        Z = np.repeat(Z.reshape(*Z.shape[:-1], ng, 1), group, axis=-1).reshape(cg.shape)
        k = np.minimum(cg, co)
        beta = Z + (k + 0.5) * S
        v = pre.astype(np.float64)
        near = np.abs(v - beta) <= EXCUSE_REL * np.maximum(np.abs(v), S)
        ok = diff & (np.abs(cg - co) == 1) & near
        exc = int(ok.sum())
    return _record(CodeReport(cg.size, n_mis, exc, n_mis - exc, szm))


def compare_codebook(gpu_codes, orc_codes, pre, cb, D, bits) -> CodeReport:
    cg = unpack_all(gpu_codes, D, bits).astype(np.int32)
    co = unpack_all(orc_codes, D, bits).astype(np.int32)
    diff = cg != co
    n_mis = int(diff.sum())
    exc = 0
    if n_mis:
        beta = 0.5 * (cb[1:].astype(np.float64) + cb[:-1].astype(np.float64))
        k = np.minimum(cg, co)
        kk = np.clip(k, 0, beta.size - 1)
        v = pre.astype(np.float64)
        sigma = 1.0 / math.sqrt(D)
        near = np.abs(v - beta[kk]) <= EXCUSE_REL * np.maximum(np.abs(v), sigma)
        ok = diff & (np.abs(cg - co) == 1) & near
        exc = int(ok.sum())
    return _record(CodeReport(cg.size, n_mis, exc, n_mis - exc, 0))


def recon_tolerance(ref, row_rel=0.0):
    """Per-element decode tolerance broadcast over [..., D]."""
    if not row_rel:
        return RECON_ABS
    return RECON_ABS + row_rel * np.linalg.norm(ref, axis=-1, keepdims=True)


def score_tolerance(q, khat, scale):
    """Per-score bound SCORE_REL * |scale| * sum_j |q_j khat_j| (fp64)."""
    return SCORE_REL * abs(scale) * np.abs(q.astype(np.float64)) @ np.abs(khat.astype(np.float64))
