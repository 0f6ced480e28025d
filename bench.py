"""Benchmark: fp16-KV GB/s of encode / decode / score on the Llama-3-8B-shaped
KV-cache layer, and the HBM roofline fraction of the dominant kernel.

One step = one pass of the whole path over one layer's KV cache
(batch 4, 8 KV heads x 128, 32768 tokens, fp16, synthetic):
  encode K, encode V   grouped-head FWHT over 8 heads x 128 channels, RoPE on K,
                       2-bit min-max, group 128
  decode K, decode V   the exact inverse (fp16 out)
  append               encode one new token per sequence into the decode cache
                       (head-dim FWHT, 2-bit group 128, 4 fp16 sinks)
  score                q . K^T for 32 query heads (GQA 4:1) over the 32769 cached
                       tokens, straight from the packed cache
value = fp16-equivalent KV bytes represented by the step's kernels / step time.

Usage: python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Under torchrun each rank runs its own copy of the workload on its own GPU
(weak scaling, no collective on the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "fp16-KV GB/s for encode/decode/score and % of B200 HBM roofline"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 512 << 20


SPEC_HBM_GBS = 8000.0  # B200 HBM3e specification (context beside the measured copy bandwidth)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _config(n_gpus):
    wg, ws = W.WORKLOADS["llama3_8b_gqa"], W.WORKLOADS["llama3_8b_gqa_score"]
    return {
        "workload": "llama3_8b_gqa",
        "batch": wg.B, "kv_heads": wg.H, "head_dim": wg.D, "tokens": wg.T, "q_heads": ws.Hq,
        "kv": "K and V fp16, N(0,1) + 1% outlier channels x U[10,50] (synthetic)",
        "encode_decode": "fwht over 8 heads x 128, RoPE(K) after it, 2-bit min-max group 128",
        "score_cache": "fwht over head_dim, 2-bit group 128, 4 fp16 sinks, 32768 + 1 appended tokens",
        "l2": "no flush: every step streams ~1.4 GB (11x the 126 MB L2), so each kernel's inputs "
              "were evicted by the kernels before it",
        "parallelism": f"replicas x{n_gpus} (batch-sharded, no data-path collective)",
    }


# ---------------------------------------------------------------- clocks
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
               0x10: "sync_boost"}

    def __init__(self, dev_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- workload
class Step:
    """Device buffers and launches of one step of the Llama-3-8B-shaped
    layer (through the C ABI)."""

    workload = "llama3_8b_gqa"

    def __init__(self, device):
        import torch
        from kv_cache_rotation_b200 import torch_api as TA
        self.torch, self.TA = torch, TA
        wg, ws = W.WORKLOADS["llama3_8b_gqa"], W.WORKLOADS["llama3_8b_gqa_score"]
        self.wg, self.ws = wg, ws
        B, H, T, D = wg.B, wg.H, wg.T, wg.D
        self.k_host = W.kv_tensor(wg, "k")
        self.v_host = W.kv_tensor(wg, "v")
        self.k = torch.from_numpy(self.k_host).to(device)
        self.v = torch.from_numpy(self.v_host).to(device)
        self.dk = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=wg.bits, group=wg.group,
                               group_heads=wg.group_heads, rope=1, rot="fwht_group")
        self.dv = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=wg.bits, group=wg.group,
                               group_heads=wg.group_heads, rope=0, rot="fwht_group")
        self.tk = TA.make_tables(rope_cs=TA.rope_table(T + 1, D, device=device))
        self.tv = TA.make_tables()
        self.pk, self.pv = TA.alloc_packed(self.dk, device), TA.alloc_packed(self.dv, device)
        self.ok = torch.empty((B, H, T, D), dtype=torch.float16, device=device)
        self.ov = torch.empty((B, H, T, D), dtype=torch.float16, device=device)
        # decode-step cache: prefill (untimed) + one appended token per step
        self.sc = ScoreCache(ws, device)
        torch.cuda.synchronize(device)
        # accounting
        rb, ng = D * wg.bits // 8, D // wg.group
        nvec = B * H * T
        self.alg = {
            "encode_k": nvec * (2 * D + rb + 4 * ng),
            "encode_v": nvec * (2 * D + rb + 4 * ng),
            "decode_k": nvec * (rb + 4 * ng + 2 * D),
            "decode_v": nvec * (rb + 4 * ng + 2 * D),
            "append": self.sc.alg_append,
            "score": self.sc.alg_score,
        }
        self.fp16_equiv = {
            "encode_k": nvec * 2 * D, "encode_v": nvec * 2 * D, "decode_k": nvec * 2 * D, "decode_v": nvec * 2 * D,
            "append": self.sc.fp16_append, "score": self.sc.fp16_score,
        }
        self.tokens = {"encode_k": B * T, "encode_v": B * T, "decode_k": B * T, "decode_v": B * T, "append": B}
        self.kernels = {"encode_k": "k_encode_group", "encode_v": "k_encode_group", "decode_k": "k_decode_group",
                        "decode_v": "k_decode_group", "append": "k_encode_head", "score": "k_score_mma"}
        self.fp32_ops = {n: nvec * D * fp32_ops_per_element("fwht_group", n, wg.group_heads, D)
                         for n in ("encode_k", "encode_v", "decode_k", "decode_v")}
        self.names = list(self.alg)
        self.host_in = [self.k_host, self.v_host, self.sc.app_host, self.sc.q_host]
        self.dev_in = [self.k, self.v, self.sc.app, self.sc.q]
        self.dev_out = [self.pk.codes, self.pk.scale_zero, self.pv.codes, self.pv.scale_zero, self.ok, self.ov,
                        self.sc.scores]

    def launches(self):
        TA = self.TA
        return [
            TA.bind_encode(self.dk, self.k, self.tk, self.pk),
            TA.bind_encode(self.dv, self.v, self.tv, self.pv),
            TA.bind_decode(self.dk, self.pk, self.tk, self.ok),
            TA.bind_decode(self.dv, self.pv, self.tv, self.ov),
            self.sc.append,
            self.sc.score,
        ]


class ScoreCache:
    """A prefilled head-variant cache (untimed) plus the decode-step launches:
    append one token per sequence, then score every cached slot. `which` =
    "v" builds the value cache of the same shape (no RoPE)."""

    def __init__(self, ws, device, which="k"):
        import torch
        from kv_cache_rotation_b200 import torch_api as TA
        self.TA = TA
        D = ws.D
        Ts = ws.T
        self.n_tok = Ts + ws.append
        cap = self.n_tok
        rope = 1 if which == "k" else 0
        common = dict(batch=ws.B, heads=ws.H, head_dim=D, t_cap=cap, bits=ws.bits, group=ws.group, rope=rope,
                      n_sink=ws.n_sink, rot="fwht_head")
        self.d_pre = TA.make_desc(tokens=Ts, t0=0, **common)
        self.d_app = TA.make_desc(tokens=ws.append, t0=Ts, **common)
        perm = (torch.from_numpy(W.random_perm(ws.H, D, ws.seed + (which == "v"))).to(device) if ws.perm
                else None)
        self.tables = TA.make_tables(perm=perm, rope_cs=TA.rope_table(cap, D, device=device) if rope else None)
        self.packed = TA.alloc_packed(self.d_pre, device)
        ks = torch.from_numpy(W.kv_tensor(ws, which)).to(device)
        TA.encode(self.d_pre, ks, self.tables, self.packed)
        del ks
        self.app_host = W.kv_tensor(ws, which + "_append", T=ws.append)
        self.app = torch.from_numpy(self.app_host).to(device)
        self.q_host = W.queries(ws)
        self.q = torch.from_numpy(self.q_host).to(device)
        self.scores = torch.empty((ws.B, ws.Hq, self.n_tok), dtype=torch.float32, device=device)
        self.scale = 1.0 / math.sqrt(D)
        rb, ng = D * ws.bits // 8, D // ws.group
        self.alg_append = ws.B * ws.H * ws.append * (2 * D + rb + 4 * ng)
        self.alg_score = (ws.B * ws.H * (self.n_tok - ws.n_sink) * (rb + 4 * ng) + ws.B * ws.H * ws.n_sink * D * 2
                          + ws.B * ws.Hq * D * 2 + ws.B * ws.Hq * self.n_tok * 4)
        self.fp16_append = ws.B * ws.H * ws.append * 2 * D
        self.fp16_score = ws.B * ws.H * self.n_tok * 2 * D
        self.append = TA.bind_encode(self.d_app, self.app, self.tables, self.packed)
        self.score = TA.bind_score(self.d_pre, self.q, self.packed, self.tables, self.n_tok, self.scale, self.scores)
        self.alg_cache = (ws.B * ws.H * (self.n_tok - ws.n_sink) * (rb + 4 * ng) + ws.B * ws.H * ws.n_sink * D * 2)


class AttendStep:
    """Decode-step attention: append one token to the K and the V cache, then
    out = softmax(q . k) . v over every slot (the Llama-3-8B shape by default;
    the Llama-2-7B shape runs the three-kernel form)."""

    # K and V caches are 75 MB (Llama-3-8B) or 84 MB (Llama-2-7B), less than the 126 MB L2: flush it before every step
    l2_flush = True

    def __init__(self, device, workload="llama3_8b_gqa_attend"):
        import torch
        from kv_cache_rotation_b200 import torch_api as TA
        self.workload = workload
        ws = W.WORKLOADS[self.workload]
        fused = ws.group == 128 and ws.bits in (2, 4)
        # two appends, then the fused attention kernel and its merge, or the scores, the chunk sums and the merge
        self.kernels_per_step = 4 if fused else 5
        self.k = ScoreCache(ws, device, "k")
        self.v = ScoreCache(ws, device, "v")
        n = self.k.n_tok
        self.out = torch.empty((ws.B, ws.Hq, ws.D), dtype=torch.float32, device=device)
        self.ws = TA.attend_workspace(self.k.d_pre, self.v.d_pre, ws.Hq, n, device=device)
        self.attend = TA.bind_attend(self.k.d_pre, self.v.d_pre, self.k.q, self.k.packed, self.k.tables,
                                     self.v.packed, self.v.tables, n, self.k.scale, self.out, self.ws)
        q_out = ws.B * ws.Hq * ws.D * (2 + 4)
        self.alg = {"append_k": self.k.alg_append, "append_v": self.v.alg_append,
                    "attend": self.k.alg_cache + self.v.alg_cache + q_out}
        self.fp16_equiv = {"append_k": self.k.fp16_append, "append_v": self.v.fp16_append,
                           "attend": 2 * self.k.fp16_score}
        self.kernels = {"append_k": "k_encode_head", "append_v": "k_encode_head",
                        "attend": "k_attend_fused" if fused else "k_attend_part"}
        self.fp32_ops = {}
        self.names = list(self.alg)
        torch.cuda.synchronize(device)

    def launches(self):
        return [self.k.append, self.v.append, self.attend]


class CalibrateStep:
    """Channel-permutation calibration of the Llama-3-8B GQA keys (head-dim
    variant: RoPE, then the abs-max over 4 x 32768 positions per head)."""

    workload = "llama3_8b_calibrate"
    kernels_per_step = 2  # abs-max and rank (plus a memset of the maxima)

    def __init__(self, device):
        import torch
        from kv_cache_rotation_b200 import torch_api as TA
        w = W.WORKLOADS["llama3_8b_gqa_score"]
        self.x = torch.from_numpy(W.kv_tensor(w, "k")).to(device)
        self.d = TA.make_desc(batch=w.B, heads=w.H, head_dim=w.D, tokens=w.T, bits=w.bits, group=w.group,
                              rope=1, n_sink=w.n_sink, rot="fwht_head")
        self.tb = TA.make_tables(rope_cs=TA.rope_table(w.T, w.D, device=device))
        self.perm = torch.empty((w.H, w.D), dtype=torch.int16, device=device)
        self.ws = TA.calibrate_workspace(self.d, device)
        self.call = TA.bind_calibrate(self.d, self.x, self.tb, self.perm, self.ws)
        nbytes = self.x.numel() * 2
        self.alg = {"calibrate": nbytes + self.perm.numel() * 2}
        self.fp16_equiv = {"calibrate": nbytes}
        self.kernels = {"calibrate": "k_absmax"}
        self.fp32_ops = {}
        self.names = list(self.alg)
        torch.cuda.synchronize(device)

    def launches(self):
        return [self.call]


class PairEnergyStep:
    """Exact per-pair RoPE energies and their ranking over the Llama-3-8B GQA
    keys (4 x 8 x 32768 x 128)."""

    workload = "llama3_8b_pair_energy"
    kernels_per_step = 2  # energy and rank (plus a memset of the sums)

    def __init__(self, device):
        import torch
        from kv_cache_rotation_b200 import torch_api as TA
        w = W.WORKLOADS["llama3_8b_gqa_score"]
        self.x = torch.from_numpy(W.kv_tensor(w, "k")).to(device)
        self.d = TA.make_desc(batch=w.B, heads=w.H, head_dim=w.D, tokens=w.T, bits=w.bits, group=w.group)
        self.e = torch.empty((w.H, w.D // 2, 2), dtype=torch.uint64, device=device)
        self.r = torch.empty((w.H, w.D // 2), dtype=torch.int16, device=device)
        self.call = TA.bind_pair_energy(self.d, self.x, self.e, self.r)
        nbytes = self.x.numel() * 2
        self.alg = {"pair_energy": nbytes + self.e.numel() * 8 + self.r.numel() * 2}
        self.fp16_equiv = {"pair_energy": nbytes}
        self.kernels = {"pair_energy": "k_pair_energy"}
        self.fp32_ops = {}
        self.names = list(self.alg)
        torch.cuda.synchronize(device)

    def launches(self):
        return [self.call]


class SinkDetectStep:
    """Attention-sink detection over the Llama-2-7B-shaped key prefill (8 x 32
    heads x 4096 tokens x 128, with massive activations planted on 4 tokens
    per sequence): per-token maxima over all heads and channels, then the
    median, threshold tau = 8 and a list of at most 8 sinks per sequence."""

    workload = "llama2_7b_sink_detect"
    kernels_per_step = 2  # per-token maxima, then one selection CTA per sequence

    def __init__(self, device):
        import torch
        from kv_cache_rotation_b200 import torch_api as TA
        w = W.WORKLOADS["llama2_7b_mha"]
        x = W.kv_tensor(w, "k")
        W.plant_massive(x, 4, 11)
        self.x = torch.from_numpy(x).to(device)
        self.d = TA.make_desc(batch=w.B, heads=w.H, head_dim=w.D, tokens=w.T, bits=w.bits, group=w.group)
        self.sp = torch.empty((w.B, 8), dtype=torch.int32, device=device)
        self.cnt = torch.empty((w.B,), dtype=torch.int32, device=device)
        self.ws = TA.detect_sinks_workspace(self.d, device)
        self.call = TA.bind_detect_sinks(self.d, self.x, 8.0, self.sp, self.cnt, self.ws)
        nbytes = self.x.numel() * 2
        # x once, the per-token keys written and read back, the lists and counts
        self.alg = {"detect": nbytes + 2 * (w.B * w.T * 2) + self.sp.numel() * 4 + w.B * 4}
        self.fp16_equiv = {"detect": nbytes}
        self.kernels = {"detect": "k_token_absmax"}
        self.fp32_ops = {}
        self.names = list(self.alg)
        torch.cuda.synchronize(device)

    def launches(self):
        return [self.call]


class GroupScoreStep:
    """Decode-step scores over the headline layer's own grouped-head key cache
    (4 x 8 KV heads x 32768 slots, FWHT over the 8 heads before RoPE, 2-bit
    group 128) for 32 query heads (GQA 4:1): every slot is decoded, turned by
    RoPE and dotted with its query heads."""

    workload = "llama3_8b_gqa_group_score"

    def __init__(self, device):
        import torch
        from kv_cache_rotation_b200 import torch_api as TA
        wg, ws = W.WORKLOADS["llama3_8b_gqa"], W.WORKLOADS["llama3_8b_gqa_score"]
        B, H, T, D = wg.B, wg.H, wg.T, wg.D
        self.d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=wg.bits, group=wg.group,
                              group_heads=wg.group_heads, rope=1, rot="fwht_group")
        self.tb = TA.make_tables(rope_cs=TA.rope_table(T, D, device=device))
        self.pk = TA.alloc_packed(self.d, device)
        TA.encode(self.d, torch.from_numpy(W.kv_tensor(wg, "k")).to(device), self.tb, self.pk)
        self.q = torch.from_numpy(W.queries(ws)).to(device)
        self.scores = torch.empty((B, ws.Hq, T), dtype=torch.float32, device=device)
        self.call = TA.bind_score(self.d, self.q, self.pk, self.tb, T, 1.0 / math.sqrt(D), self.scores)
        rb, ng = D * wg.bits // 8, D // wg.group
        self.alg = {"score": B * H * T * (rb + 4 * ng) + B * ws.Hq * D * 2 + B * ws.Hq * T * 4}
        self.fp16_equiv = {"score": B * H * T * D * 2}
        self.kernels = {"score": "k_score_group"}
        self.fp32_ops = {}
        self.names = list(self.alg)
        torch.cuda.synchronize(device)

    def launches(self):
        return [self.call]


class EncDecStep:
    """Encode then decode of K (and V when `both`) for one workload."""

    def __init__(self, name, device, both=True, batch=None):
        import torch
        from kv_cache_rotation_b200 import torch_api as TA
        self.workload = name
        w = W.WORKLOADS[name] if batch is None else W.scaled(W.WORKLOADS[name], B=batch)
        self.TA = TA
        B, H, T, D = w.B, w.H, w.T, w.D
        iso = w.rot in ("iso", "iso3")
        tensors = ["k", "v"] if both and not iso else ["k"]
        self.items = []
        self.alg, self.fp16_equiv, self.kernels, self.fp32_ops = {}, {}, {}, {}
        self.tokens = {}
        kern = {"fwht_head": "head", "none": "head", "fwht_group": "group", "iso": "iso", "iso3": "iso"}[w.rot]
        for which in tensors:
            x = (W.kv_tensor_device(w, which, device) if iso else torch.from_numpy(W.kv_tensor(w, which)).to(device))
            rope = 1 if (which == "k" and w.rope_k) else 0
            d = TA.make_desc(batch=B, heads=H, head_dim=D, tokens=T, bits=w.bits, group=w.group,
                             group_heads=w.group_heads, rope=rope, n_sink=w.n_sink, rot=w.rot, quant=w.quant)
            perm = torch.from_numpy(W.random_perm(H, D, w.seed + len(which))).to(device) if w.perm else None
            if iso:
                qL, qR = W.iso_tables(w) if w.rot == "iso" else (W.iso3_tables(D, w.seed), None)
                qLd = torch.from_numpy(qL).to(device)
                qRd = torch.from_numpy(qR).to(device) if qR is not None else None
                if w.quant == "codebook_dyn":
                    # per-channel tables from the same tokens (untimed), then the
                    # quality of both codebooks on them
                    tb = TA.make_tables(qL=qLd, qR=qRd, codebook=TA.lloyd_max_codebook(w.bits, 1, device=device),
                                        codebook_wide=TA.lloyd_max_codebook(w.bits + 1, 1, device=device))
                    tb.ch_scale, tb.ch_wide = TA.calibrate_codebook(d, x, tb)
                    self.quality = self._snr(TA, d, x, tb, qLd, qRd, w, device)
                else:
                    tb = TA.make_tables(qL=qLd, qR=qRd, codebook=TA.lloyd_max_codebook(w.bits, D, device=device))
            else:
                tb = TA.make_tables(perm=perm, rope_cs=TA.rope_table(T, D, device=device) if rope else None)
            pk = TA.alloc_packed(d, device)
            out = torch.empty((B, H, T, D), dtype=torch.float16, device=device)
            self.items.append((which, d, x, tb, pk, out))
            nvec = B * H * T
            per_vec = D * w.bits // 8 + (4 * (D // w.group) if w.quant == "minmax" else 4)
            if w.quant == "codebook_dyn":
                per_vec += 2  # the outlier channels' top bits
            self.alg[f"encode_{which}"] = nvec * (2 * D + per_vec) + (B * H * w.n_sink * D * 2)
            self.alg[f"decode_{which}"] = nvec * (2 * D + per_vec)
            self.tokens[f"encode_{which}"] = self.tokens[f"decode_{which}"] = B * T
            self.fp16_equiv[f"encode_{which}"] = nvec * 2 * D
            self.fp16_equiv[f"decode_{which}"] = nvec * 2 * D
            self.kernels[f"encode_{which}"] = f"k_encode_{kern}"
            self.kernels[f"decode_{which}"] = f"k_decode_{kern}"
            for n in (f"encode_{which}", f"decode_{which}"):
                ops = fp32_ops_per_element(w.rot, n, w.group_heads, D, rope=rope)
                if ops:
                    self.fp32_ops[n] = nvec * D * ops
        self.names = list(self.alg)
        torch.cuda.synchronize(device)

    @staticmethod
    def _snr(TA, d, x, tb, qL, qR, w, device, rows=1 << 18):
        """SNR (dB) of the decode against the input on the first `rows` vectors,
        with the dynamic tables and with the fixed N(0, 1/D) codebook."""
        import torch
        n = min(rows, d.batch * d.heads * d.tokens)
        b = max(1, n // (d.heads * d.tokens))
        ds = TA.make_desc(batch=b, heads=d.heads, head_dim=d.head_dim, tokens=d.tokens, bits=d.bits, rot=d.rot,
                          quant=d.quant)
        xs = x[:b].contiguous()
        ref = xs.float()
        out = {}
        fixed = TA.make_tables(qL=qL, qR=qR, codebook=TA.lloyd_max_codebook(w.bits, d.head_dim, device=device))
        for name, q, t in (("dynamic", d.quant, tb), ("fixed", TA.QUANT["codebook"], fixed)):
            ds.quant = q
            pk = TA.alloc_packed(ds, device)
            y = torch.empty_like(ref)
            TA.encode(ds, xs, t, pk)
            TA.decode(ds, pk, t, y)
            out[f"snr_db_{name}"] = float(10 * torch.log10((ref ** 2).sum() / ((ref - y) ** 2).sum()))
        out["snr_sample_vectors"] = b * d.heads * d.tokens
        return out

    def launches(self):
        """One launch per entry of self.names, in the same order (encode then
        decode of each tensor)."""
        TA = self.TA
        fs = []
        for which, d, x, tb, pk, out in self.items:
            fs += [TA.bind_encode(d, x, tb, pk), TA.bind_decode(d, pk, tb, out)]
        assert len(fs) == len(self.names)
        return fs


class DecodeScoreStep:
    """Decode step of the batch-64 MHA cache: append one token, score all slots."""

    workload = "decode_score"

    def __init__(self, device):
        import torch
        self.sc = ScoreCache(W.WORKLOADS["decode_score"], device)
        self.alg = {"append": self.sc.alg_append, "score": self.sc.alg_score}
        self.fp16_equiv = {"append": self.sc.fp16_append, "score": self.sc.fp16_score}
        self.kernels = {"append": "k_encode_head", "score": "k_score_mma"}
        self.fp32_ops = {}
        self.names = list(self.alg)
        torch.cuda.synchronize(device)

    def launches(self):
        return [self.sc.append, self.sc.score]


class LiteralScoreStep:
    """Both forms of the decode-step score over one prefilled head-variant cache:
    the query-rotation kernel and the literal form that decodes every key
    (unpack, dequantize, inverse FWHT) before the dot product."""

    def __init__(self, workload, device):
        import torch
        self.workload = workload
        base = workload[:-len("_literal")]
        self.sc = ScoreCache(W.WORKLOADS[base], device)
        self.literal = self.sc.TA.bind_score(self.sc.d_pre, self.sc.q, self.sc.packed, self.sc.tables,
                                             self.sc.n_tok, self.sc.scale, self.sc.scores, literal=True)
        self.alg = {"score": self.sc.alg_score, "score_literal": self.sc.alg_score}
        self.fp16_equiv = {"score": self.sc.fp16_score, "score_literal": self.sc.fp16_score}
        self.kernels = {"score": "k_score_mma", "score_literal": "k_score_literal"}
        self.fp32_ops = {}
        self.names = list(self.alg)
        torch.cuda.synchronize(device)

    def launches(self):
        return [self.sc.score, self.literal]


def fp32_ops_per_element(rot, step, group_heads, D, rope=None):
    """Algorithmic fp32 operations per element of an encode/decode launch, in
    the oracle's order: FWHT log2(N) add/sub (N = D, or group_heads * D), RoPE
    2 (one mul and one fma per output, keys only), the quantizer 2 (sub + fma)
    or the dequantizer 2 (fma + the folded normalisation). Min/max compares run
    on the ALU pipe and are not counted. None for IsoQuant (norm, 4x4 blocks,
    codebook search)."""
    if rot in ("iso", "iso3"):
        return None
    n = D * (group_heads if rot == "fwht_group" else 1)
    fwht = 0 if rot == "none" else int(math.log2(n))
    if rope is None:
        rope = 1 if step.endswith("_k") else 0
    return fwht + 2 * rope + 2


def make_step(workload, device, batch=None):
    if workload == "llama3_8b_gqa":
        return Step(device)
    if workload == "decode_score":
        return DecodeScoreStep(device)
    if workload in ("llama3_8b_gqa_attend", "llama2_7b_mha_attend"):
        return AttendStep(device, workload)
    if workload == "llama3_8b_calibrate":
        return CalibrateStep(device)
    if workload == "llama3_8b_pair_energy":
        return PairEnergyStep(device)
    if workload == "llama3_8b_gqa_group_score":
        return GroupScoreStep(device)
    if workload == "llama2_7b_sink_detect":
        return SinkDetectStep(device)
    if workload.endswith("_score_literal"):
        return LiteralScoreStep(workload, device)
    return EncDecStep(workload, device, batch=batch)


def _kernel_sources_sha(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "kv_cache_rotation_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(f"{kernel}@{workload}") or j.get(kernel)
    if not e or e.get("bench_workload") != workload:
        return None
    if e.get("source_sha") != _kernel_sources_sha(e.get("sources", [])):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU oracle timing
def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class CpuSample:
    """The oracle on a bounded sample of the headline workload: the first
    `batches` sequences (all 8 KV heads), encode + decode of K and V (grouped
    FWHT) and the score of their 32 query heads, over a window of token
    positions. Inputs are drawn once; `run` times only the oracle calls. The
    work is split into independent (sequence, token range) items run by
    `threads` threads (each oracle call is plain C through ctypes, which
    releases the GIL, so the threads run in parallel on the host cores)."""

    def __init__(self, batches: int, tokens: int):
        import oracle
        self.oracle = oracle
        wg, ws = W.WORKLOADS["llama3_8b_gqa"], W.WORKLOADS["llama3_8b_gqa_score"]
        self.wg, self.ws, self.Bn, self.Tn = wg, ws, batches, tokens
        self.k = W.kv_tensor(W.scaled(wg, T=tokens, B=batches, seed=wg.seed * 1000), "k").view(np.uint16)
        self.v = W.kv_tensor(W.scaled(wg, T=tokens, B=batches, seed=wg.seed * 1000), "v").view(np.uint16)
        self.kwk = dict(rot=oracle.ROT_FWHT_GROUP, bits=wg.bits, group=wg.group, group_heads=wg.group_heads,
                        rope=1)
        self.kwv = dict(self.kwk, rope=0)
        self.kws = dict(rot=oracle.ROT_FWHT_HEAD, bits=ws.bits, group=ws.group, rope=1, n_sink=ws.n_sink)
        ks = W.kv_tensor(W.scaled(ws, T=tokens, B=batches, seed=ws.seed * 1000), "k").view(np.uint16)
        self.q = W.queries(ws, B=batches).view(np.uint16)
        cache = oracle.encode(ks, np.arange(tokens), **self.kws)  # the decode-step cache (untimed)
        self.caches = [{f: np.ascontiguousarray(a[b:b + 1]) for f, a in cache.items() if a is not None}
                       for b in range(batches)]

    def _item(self, b, lo, hi):
        o = self.oracle
        k = np.ascontiguousarray(self.k[b:b + 1, :, lo:hi])
        v = np.ascontiguousarray(self.v[b:b + 1, :, lo:hi])
        pos = np.arange(lo, hi)
        pk = o.encode(k, pos, **self.kwk)
        pv = o.encode(v, pos, **self.kwv)
        o.decode(pk, pos, k.shape, **self.kwk)
        o.decode(pv, pos, v.shape, **self.kwv)
        o.score(np.ascontiguousarray(self.q[b:b + 1]), self.caches[b], pos, H=self.ws.H, t_cap=self.Tn,
                scale=1 / math.sqrt(self.ws.D), **self.kws)

    def run(self, threads: int, lo: int = 0, hi: int = None):
        """Time the sample over token positions [lo, hi) of every sequence.
        Returns (fp16-equivalent bytes, seconds, description)."""
        import concurrent.futures as cf
        hi = self.Tn if hi is None else hi
        n_items = max(1, 4 * threads // self.Bn)  # token ranges per sequence (load balance)
        edges = np.linspace(lo, hi, n_items + 1).astype(int)
        items = [(b, int(a), int(c)) for b in range(self.Bn) for a, c in zip(edges[:-1], edges[1:]) if c > a]
        t0 = time.perf_counter()
        if threads == 1:
            for it in items:
                self._item(*it)
        else:
            with cf.ThreadPoolExecutor(max_workers=threads) as ex:
                list(ex.map(lambda it: self._item(*it), items))
        dt = time.perf_counter() - t0
        Tn = hi - lo
        nbytes = 5 * self.Bn * self.wg.H * Tn * self.wg.D * 2  # 4 encode/decode passes + the score's keys
        desc = (f"oracle (plain C), {threads} thread{'s' if threads > 1 else ''}: {self.Bn} of {self.wg.B} "
                f"sequences x {Tn} of {self.wg.T} tokens: encode+decode of K and V (grouped FWHT) and the "
                f"score of 32 query heads per sequence over those cache slots")
        return nbytes, dt, desc


def cpu_baseline():
    """The oracle on the host: all cores on all 4 sequences (the reported
    figure), and one thread on one sequence beside it. About 5 s of one core
    plus 22 s of CPU work spread over the cores."""
    cores = host_cores()
    one = CpuSample(1, W.WORKLOADS["llama3_8b_gqa"].T)
    b1, s1, d1 = one.run(1)
    allc = CpuSample(W.WORKLOADS["llama3_8b_gqa"].B, W.WORKLOADS["llama3_8b_gqa"].T)
    b, s, d = allc.run(cores)
    return {"value": b / s / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": d, "seconds": s,
            "single_thread": {"value": b1 / s1 / 1e9, "unit": UNIT, "cores": 1, "sample": d1, "seconds": s1}}


# ---------------------------------------------------------------- arms
def run_reference(args):
    """The oracle as the reference arm: each step is the all-core CPU sample
    over the next window of `--ref-tokens` token positions of all 4
    sequences (the same sample kind as the GPU line's cpu_baseline)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = _config(args.gpus)
    cores = host_cores()
    wg = W.WORKLOADS["llama3_8b_gqa"]
    smp = CpuSample(wg.B, wg.T)
    win = max(1, min(args.ref_tokens, wg.T))
    n_win = wg.T // win
    for i in range(args.warmup):
        smp.run(cores, 0, min(wg.T, 256))
    tot_b, tot_s = 0, 0.0
    desc = ""
    for i in range(args.steps):
        lo = (i % n_win) * win
        b, s, desc = smp.run(cores, lo, lo + win)
        tot_b += b
        tot_s += s
    value = tot_b / tot_s / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_s / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over all ranks (every rank receives it); x itself without a
    process group. Each rank times its own device; the job takes as long as the
    slowest rank."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step_per_rank: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: the bytes all ranks processed over the slowest rank's time."""
    return world * bytes_per_step_per_rank * steps / (max_ms / 1e3) / 1e9


def run_ours(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import kv_cache_rotation_b200 as K
    st = make_step(args.workload, dev, args.batch)
    launches = st.launches()
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        for f in launches:
            f()
    torch.cuda.synchronize(dev)
    assert K.kvq_check(0) == K.KVQ_OK

    nk = len(launches)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
    flush = getattr(st, "l2_flush", False)
    # read-based flush (a clean 512 MB sweep, 4x the L2): leaves no dirty lines for the next kernel to write back
    fbuf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev) if flush else None
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for s in range(args.steps):
            if flush:
                fbuf.sum()
            ev[s][0].record(stream)
            for i, f in enumerate(launches):
                f()
                ev[s][i + 1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    # with a flush the timed region is the steps alone (each step bracketed by its own events)
    total_ms = (sum(ev[s][0].elapsed_time(ev[s][nk]) for s in range(args.steps)) if flush
                else t_start.elapsed_time(t_end))
    per_kernel = {n: 0.0 for n in st.names}
    for s in range(args.steps):
        for i, n in enumerate(st.names):
            per_kernel[n] += ev[s][i].elapsed_time(ev[s][i + 1])
    status = K.kvq_check(0)
    total_ms = max_over_ranks(total_ms, dist, dev)

    fp16_step = sum(st.fp16_equiv.values())
    value = whole_job_gbs(world, fp16_step, args.steps, total_ms)
    peak, peak_kind = _peaks()
    kernels = {}
    for n in st.names:
        ms = per_kernel[n] / args.steps
        kernels[n] = {"ms": ms, "fp16_gbs": st.fp16_equiv[n] / (ms / 1e3) / 1e9,
                      "alg_gbs": st.alg[n] / (ms / 1e3) / 1e9,
                      "frac_of_measured_hbm": st.alg[n] / (ms / 1e3) / 1e9 / peak,
                      "frac_of_spec_8tbs": st.alg[n] / (ms / 1e3) / 1e9 / SPEC_HBM_GBS}
        tok = getattr(st, "tokens", {}).get(n)
        if tok:  # token positions of one tensor (B x T) processed per second
            kernels[n]["tokens_per_s"] = tok / (ms / 1e3)
    dom = max(st.names, key=lambda n: per_kernel[n])
    dom_ms = per_kernel[dom] / args.steps
    achieved = st.alg[dom] / (dom_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": _traffic_for(st.kernels[dom], args.workload), "kernel": st.kernels[dom],
                "kernel_step": dom, "alg_bytes_per_launch": st.alg[dom], "peak_kind": peak_kind}
    clocks = clk.summary()
    if dom in st.fp32_ops:
        # the same launch against the fp32 pipe: SMs x 128 fp32 lanes x max SM clock
        mhz = clocks.get("sm_max_mhz") or 1965
        alu_peak = torch.cuda.get_device_properties(dev).multi_processor_count * 128 * mhz * 1e6
        alu_ach = st.fp32_ops[dom] / (dom_ms / 1e3)
        roofline["alu"] = {"achieved": alu_ach / 1e12, "peak": alu_peak / 1e12, "unit": "T fp32-op/s",
                           "frac": alu_ach / alu_peak, "ops_per_launch": st.fp32_ops[dom]}
        roofline["alu_frac"] = alu_ach / alu_peak

    e2e_line = None
    if hasattr(st, "host_in"):
        # a second buffer set (same workload, same bytes) so one step's inputs can go in
        # while the previous step's results come out
        st2 = make_step(args.workload, dev, args.batch)
        e2e = run_e2e([(st, launches), (st2, st2.launches())], dev, stream, min(args.steps, args.e2e_steps),
                      args.warmup_e2e)
        del st2
        e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], dist, dev)
        e2e_line = {"value": whole_job_gbs(world, fp16_step, 1, e2e["ms_per_step"]), "unit": UNIT,
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "ms_per_step": e2e["ms_per_step"], "steps": e2e["steps"],
                    "pipelined": "two buffer sets; each step's copy-in overlaps the previous step's copy-out"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and args.workload == "llama3_8b_gqa":
        cpu = cpu_baseline()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": _config(world) if args.workload == "llama3_8b_gqa" else _other_config(args.workload, world),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e_line,
            "gpu_launches": getattr(st, "kernels_per_step", nk) * args.steps, "clocks": clocks, "kernels": kernels,
            "status": K.kvq_status_str(status),
        }
        if hasattr(st, "quality"):
            line["quality"] = st.quality
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0 if status == K.KVQ_OK else 1


def run_e2e(sets, dev, stream, steps, warmup):
    """The step through host buffers: every step copies its inputs in from pinned
    host memory and every result it produces back to pinned host memory, inside
    the timed region. Steps alternate between two device buffer sets, with the
    copies on their own streams, so step i+1's host-to-device copy overlaps step
    i's compute and device-to-host copy (PCIe runs both directions at once);
    events keep each buffer set's copy-in, kernels and copy-out in order."""
    import torch
    bufs = []
    for st, launches in sets:
        h_in = [torch.from_numpy(a).pin_memory() for a in st.host_in]
        h_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in st.dev_out]
        bufs.append((st, launches, h_in, h_out))
    h2d = sum(t.numel() * t.element_size() for t in bufs[0][2])
    d2h = sum(t.numel() * t.element_size() for t in bufs[0][3])
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    comp_done = [torch.cuda.Event() for _ in bufs]
    out_done = [torch.cuda.Event() for _ in bufs]

    def one(i):
        k = i % len(bufs)
        st, launches, h_in, h_out = bufs[k]
        s_in.wait_event(comp_done[k])  # the kernels of the last step on this set have read its inputs
        with torch.cuda.stream(s_in):
            for h, d in zip(h_in, st.dev_in):
                d.copy_(h, non_blocking=True)
        in_done = torch.cuda.Event()
        in_done.record(s_in)
        stream.wait_event(in_done)
        stream.wait_event(out_done[k])  # the last copy-out of this set's results has finished
        for f in launches:
            f()
        comp_done[k].record(stream)
        s_out.wait_event(comp_done[k])
        with torch.cuda.stream(s_out):
            for h, d in zip(h_out, st.dev_out):
                h.copy_(d, non_blocking=True)
        out_done[k].record(s_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(steps):
        one(i)
    for e in out_done:
        stream.wait_event(e)
    b.record(stream)
    torch.cuda.synchronize(dev)
    return {"ms_per_step": a.elapsed_time(b) / steps, "h2d": h2d, "d2h": d2h, "steps": steps,
            "buffer_sets": len(bufs)}


def _other_config(name, n_gpus):
    if name == "llama3_8b_pair_energy":
        w = W.WORKLOADS["llama3_8b_gqa_score"]
        return {"workload": name, "batch": w.B, "kv_heads": w.H, "head_dim": w.D, "tokens": w.T,
                "input": "keys fp16; exact 128-bit sums of each RoPE pair's squared norm, then the pair ranking",
                "l2": "no flush (the 268 MB input is larger than L2)", "parallelism": f"replicas x{n_gpus}"}
    if name == "llama3_8b_gqa_group_score":
        w = W.WORKLOADS["llama3_8b_gqa"]
        return {"workload": name, "batch": w.B, "kv_heads": w.H, "head_dim": w.D, "tokens": w.T, "q_heads": 32,
                "cache": "grouped-head FWHT over 8 heads x 128 before RoPE, 2-bit group 128 (the headline K cache)",
                "l2": "no flush (the 38 MB cache and 17 MB of scores are read / written once per step)",
                "parallelism": f"replicas x{n_gpus}"}
    if name == "llama2_7b_sink_detect":
        w = W.WORKLOADS["llama2_7b_mha"]
        return {"workload": name, "batch": w.B, "kv_heads": w.H, "head_dim": w.D, "tokens": w.T,
                "input": "keys fp16 with massive activations planted on 4 tokens per sequence",
                "tau": 8.0, "max_sinks": 8,
                "l2": "no flush (the 268 MB input is larger than L2)", "parallelism": f"replicas x{n_gpus}"}
    if name == "llama3_8b_calibrate":
        w = W.WORKLOADS["llama3_8b_gqa_score"]
        return {"workload": name, "batch": w.B, "kv_heads": w.H, "head_dim": w.D, "tokens": w.T,
                "input": "keys fp16, RoPE'd before the abs-max (head-dim variant)", "n_sink": w.n_sink,
                "l2": "no flush (the 268 MB input is larger than L2)", "parallelism": f"replicas x{n_gpus}"}
    if name.endswith("_score_literal"):
        c = _other_config(name[:-len("_literal")], n_gpus)
        c["workload"] = name
        c["forms"] = ("query rotation (k_score_mma) and the literal per-token decode + inverse FWHT "
                      "(k_score_literal) over the same cache, timed one after the other")
        return c
    w = W.WORKLOADS[name]
    return {"workload": name, "batch": w.B, "kv_heads": w.H, "head_dim": w.D, "tokens": w.T, "q_heads": w.Hq,
            "rotation": w.rot, "quant": w.quant, "bits": w.bits, "group": w.group, "n_sink": w.n_sink,
            "perm": w.perm, "l2": ("flushed before every step by a 512 MB read (outside the timed steps)"
                                   if name in ("llama3_8b_gqa_attend", "llama2_7b_mha_attend") else
                                   "no flush (inputs larger than L2)" if name != "tiny" else "L2-resident"),
            "parallelism": f"replicas x{n_gpus}"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--warmup-e2e", type=int, default=3)
    ap.add_argument("--ref-tokens", type=int, default=4096,
                    help="token positions (of each of the 4 sequences) per reference-arm step")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline leg")
    ap.add_argument("--workload", default="llama3_8b_gqa",
                    choices=["llama3_8b_gqa", "llama2_7b_mha", "isoquant_batch", "isoquant_so3_batch",
                             "isoquant_dyn_batch", "decode_score",
                             "llama3_8b_gqa_group_score", "llama2_7b_sink_detect",
                             "decode_score_literal", "llama3_8b_gqa_score_literal",
                             "llama3_8b_gqa_attend", "llama2_7b_mha_attend", "llama3_8b_calibrate",
                             "llama3_8b_pair_energy", "tiny"],
                    help="which workload a step runs (the headline line is llama3_8b_gqa)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the batch of an encode/decode workload (small profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
