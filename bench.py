"""Benchmark of the MiMo-V2-Flash hybrid attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload stack|swa|global|decode|chunked|decode_fp8|qkv] [--no-e2e] [--no-cpu-baseline]

One step = one pass of the whole hot path over the hybrid 8-layer attention
stack (hybrid_layer_pattern 0,1,1,1,1,1,0,1: 6 sliding-window layers with
8 KV heads, window 128 and sinks; 2 global layers with 4 KV heads):
  prefill  B4 x S32768, Hq 64, qk 192 / v 128, rotary 64, every layer;
  decode   B64, one new token per sequence, KV lengths ~ U[1024, 32768]
           (global layers: linear cache of 32768; sliding layers: 128-slot ring).
Inputs are synthetic N(0,1) bf16 drawn on the device, resident in HBM before
timing. Every step streams ~60 GB (far above the 126 MB L2), so no L2 flush
is added. `value` = unmasked attention FLOPs of the step / step time.

With --gpus N the script runs under torch.distributed (one process per GPU,
NCCL), every rank runs the same per-GPU workload (weak scaling; the layer has
no exchange step, so no collective sits on the data path), and the step time
is the max over ranks.

--impl reference times the fp64 CPU oracle (test infrastructure) on a bounded
sample of the same workload on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from global_attention_partial_b200 import synthetic  # noqa: E402

METRIC = "prefill attn TFLOP/s & % tensor peak; decode KV GB/s & % HBM peak (1 B200)"
FLOP_PER_PAIR = None  # 2 * (Dqk + Dv) per visible (query head, query, key) triple


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ counting
def visible_pairs(spec, S: int) -> int:
    """Visible (query, key) pairs of one head: S(S+1)/2 (global) or
    sum_i min(i+1, W) (sliding window)."""
    if spec.layer_type == 0:
        return S * (S + 1) // 2
    W = spec.window
    if S <= W:
        return S * (S + 1) // 2
    return W * (W + 1) // 2 + (S - W) * W


def prefill_flops(spec, B: int, S: int) -> float:
    return float(B) * spec.num_q_heads * visible_pairs(spec, S) * 2 * (spec.qk_dim + spec.v_dim)


def chunk_flops(spec, B: int, S: int, past: int) -> float:
    """FLOPs of a chunk of S tokens after `past` cached ones: token t sees
    past + t + 1 keys (global) or min(past + t + 1, W) (sliding)."""
    if spec.layer_type == 0:
        pairs = S * past + S * (S + 1) // 2
    else:
        pairs = sum(min(past + t + 1, spec.window) for t in range(S))
    return float(B) * spec.num_q_heads * pairs * 2 * (spec.qk_dim + spec.v_dim)


def qkv_flops(spec, B: int, S: int) -> float:
    """FLOPs of one layer's QKV projection: 2 per multiply-add of x W^T."""
    n = spec.num_q_heads * spec.qk_dim + spec.num_kv_heads * (spec.qk_dim + spec.v_dim)
    return 2.0 * B * S * n * spec.hidden_size


def prefill_bytes(spec, B: int, S: int) -> float:
    """Compulsory HBM bytes of one prefill layer: read Q, K, V, write O."""
    e = 2
    return float(B) * S * e * (spec.num_q_heads * spec.qk_dim + spec.num_kv_heads * (spec.qk_dim + spec.v_dim)
                               + spec.num_q_heads * spec.v_dim)


def decode_visible(spec, lens):
    return [min(L, spec.window) if spec.layer_type == 1 else L for L in lens]


def decode_flops(spec, lens) -> float:
    return float(sum(decode_visible(spec, lens))) * spec.num_q_heads * 2 * (spec.qk_dim + spec.v_dim)


def decode_bytes(spec, lens, cache_elem: int = 2) -> float:
    """Algorithmic HBM bytes of one decode layer: the visible cache K/V, the
    new q/k/v, the new token's cache write, the output and the sinks.
    cache_elem: bytes per cached element (2 bf16, 1 fp8)."""
    e = 2
    B = len(lens)
    kv_elems = spec.num_kv_heads * (spec.qk_dim + spec.v_dim)
    kv_row = kv_elems * cache_elem
    cache_read = sum(decode_visible(spec, lens)) * kv_row
    q_read = B * spec.num_q_heads * spec.qk_dim * e
    new_rw = B * kv_elems * e + B * kv_row
    out_w = B * spec.num_q_heads * spec.v_dim * e
    sinks = spec.num_q_heads * 4 if spec.has_sink else 0
    return float(cache_read + q_read + new_rw + out_w + sinks)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not self.uuid.startswith("GPU-"):
                self.uuid = "GPU-" + self.uuid
        except Exception:
            pass
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        for ln in out.strip().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# chunked prefill workload: the hybrid stack's last CHUNK_SEQ tokens after CHUNK_PAST cached ones
CHUNK_PAST, CHUNK_SEQ = 28672, 4096

# ------------------------------------------------------------------ workload
class StackWorkload:
    """Device-resident inputs, outputs, caches and workspaces of the step."""

    def __init__(self, kind: str, seed: int = 0, layers=None, batch=None, seq=None):
        """layers: indices of the workload's layers to keep (all by default);
        batch / seq: override the prefill batch and length (prefill and
        projection workloads), e.g. to profile one kernel on a smaller case."""
        import dataclasses
        import global_attention_partial_b200 as mimo
        self.mimo = mimo
        self.kind = kind
        dev = "cuda"
        pw = synthetic.HYBRID_PREFILL
        dw = synthetic.HYBRID_DECODE
        if kind == "swa":
            pw = synthetic.SWA_PREFILL
        elif kind == "global":
            pw = synthetic.GLOBAL_PREFILL
        if layers is not None:
            pw = dataclasses.replace(pw, layers=tuple(pw.layers[i] for i in layers if i < len(pw.layers)))
            dw = dataclasses.replace(dw, layers=tuple(dw.layers[i] for i in layers if i < len(dw.layers)))
        if batch is not None:
            pw = dataclasses.replace(pw, batch=batch)
        if seq is not None:
            pw = dataclasses.replace(pw, seq=seq)
        # seeds follow each layer's index in the full workload
        self.layer_ids = list(layers) if layers is not None else list(range(len(synthetic.HYBRID_PATTERN)))
        self.do_prefill = kind in ("stack", "swa", "global")
        self.do_decode = kind in ("stack", "decode", "decode_fp8")
        self.fp8 = kind == "decode_fp8"
        self.k_scale, self.v_scale = 1.0 / 16, 1.0 / 32
        self.do_chunked = kind == "chunked"
        self.do_qkv = kind == "qkv"
        self.pw, self.dw = pw, dw
        self.prefill_layers = []
        if self.do_prefill:
            B, S = pw.batch, pw.seq
            for li, spec in zip(self.layer_ids, pw.layers):
                q, k, v, sinks = synthetic.prefill_inputs(spec, B, S, seed=seed, layer=li, device=dev)
                sinks = sinks if spec.layer_type == 1 else None
                lay = mimo.make_layer(spec.layer_type, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim,
                                      spec.v_dim, spec.rotary_dim, spec.window, spec.theta,
                                      spec.hidden_size, sinks)
                out = torch.empty((B, S, spec.num_q_heads, spec.v_dim), dtype=torch.bfloat16, device=dev)
                need = mimo.mimo_attn_prefill_workspace_size(lay, mimo.BF16, B, S)
                ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
                self.prefill_layers.append(dict(spec=spec, lay=lay, q=q, k=k, v=v, sinks=sinks, out=out, ws=ws,
                                                need=need))
        # chunked: the stack's last 4096 tokens as a chunk after 28672 cached ones
        self.chunk_layers = []
        self.chunk_past, self.chunk_seq = CHUNK_PAST, CHUNK_SEQ
        if self.do_chunked:
            B, S, P = pw.batch, CHUNK_SEQ, CHUNK_PAST
            self.past_dev = torch.full((B,), P, dtype=torch.int32, device=dev)
            for li, spec in zip(self.layer_ids, pw.layers):
                q, k, v, kc, vc, sinks = synthetic.cached_prefill_inputs(spec, B, S, P + S, seed=seed, layer=li,
                                                                         device=dev)
                sinks = sinks if spec.layer_type == 1 else None
                lay = mimo.make_layer(spec.layer_type, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim,
                                      spec.v_dim, spec.rotary_dim, spec.window, spec.theta,
                                      spec.hidden_size, sinks)
                out = torch.empty((B, S, spec.num_q_heads, spec.v_dim), dtype=torch.bfloat16, device=dev)
                need = mimo.mimo_attn_prefill_cached_workspace_size(lay, mimo.BF16, B, S, P)
                ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
                self.chunk_layers.append(dict(spec=spec, lay=lay, q=q, k=k, v=v, kc=kc, vc=vc, out=out, ws=ws))
        # qkv: every layer's fused QKV projection of the stack's prefill tokens
        # (outputs and the cache write; x and the output buffers are shared
        # by the layers, each layer has its own weights and caches)
        self.qkv_layers = []
        if self.do_qkv:
            B, S = pw.batch, pw.seq
            spec0 = pw.layers[0]
            self.qkv_x, _ = synthetic.projection_inputs(spec0, B, S, seed=seed, layer=0, device=dev)
            self.qkv_q = torch.empty((B, S, spec0.num_q_heads, spec0.qk_dim), dtype=torch.bfloat16, device=dev)
            kv_heads = max(s.num_kv_heads for s in pw.layers)
            self.qkv_k = torch.empty((B, S, kv_heads, spec0.qk_dim), dtype=torch.bfloat16, device=dev)
            self.qkv_v = torch.empty((B, S, kv_heads, spec0.v_dim), dtype=torch.bfloat16, device=dev)
            for li, spec in zip(self.layer_ids, pw.layers):
                _, w = synthetic.projection_inputs(spec, 1, 1, seed=seed, layer=li, device=dev)
                lay = mimo.make_layer(spec.layer_type, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim,
                                      spec.v_dim, spec.rotary_dim, spec.window, spec.theta, spec.hidden_size, None)
                cap = spec.window if spec.layer_type == 1 else S
                kc = torch.empty((B, cap, spec.num_kv_heads, spec.qk_dim), dtype=torch.bfloat16, device=dev)
                vc = torch.empty((B, cap, spec.num_kv_heads, spec.v_dim), dtype=torch.bfloat16, device=dev)
                need = mimo.mimo_attn_qkv_project_workspace_size(lay, B, S, 0)
                ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
                self.qkv_layers.append(dict(spec=spec, lay=lay, w=w, kc=kc, vc=vc, cap=cap, ws=ws))
        self.decode_layers = []
        if self.do_decode:
            B = dw.batch
            self.lens = synthetic.decode_kv_lens(B, *dw.kv_len_range, seed=seed).tolist()
            lens_dev = torch.tensor(self.lens, dtype=torch.int32, device=dev)
            for li, spec in zip(self.layer_ids, dw.layers):
                q, kn, vn, kc, vc, sinks = synthetic.decode_inputs(spec, B, dw.seq, torch.tensor(self.lens),
                                                                   seed=seed, layer=100 + li, device=dev)
                sinks = sinks if spec.layer_type == 1 else None
                lay = mimo.make_layer(spec.layer_type, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim,
                                      spec.v_dim, spec.rotary_dim, spec.window, spec.theta,
                                      spec.hidden_size, sinks)
                cap = kc.shape[1]
                if self.fp8:  # E4M3 caches: the same N(0,1) values quantized with per-tensor scales
                    kc = mimo.quantize_fp8(kc, self.k_scale)
                    vc = mimo.quantize_fp8(vc, self.v_scale)
                    torch.cuda.synchronize()
                out = torch.empty((B, spec.num_q_heads, spec.v_dim), dtype=torch.bfloat16, device=dev)
                need = mimo.mimo_attn_decode_workspace_size(lay, mimo.BF16, B, cap)
                ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
                self.decode_layers.append(dict(spec=spec, lay=lay, q=q, kn=kn, vn=vn, kc=kc, vc=vc, sinks=sinks,
                                               out=out, ws=ws, need=need, cap=cap, lens=lens_dev))

    # units
    def prefill_flops(self):
        return sum(prefill_flops(L["spec"], self.pw.batch, self.pw.seq) for L in self.prefill_layers)

    def decode_flops(self):
        return sum(decode_flops(L["spec"], self.lens) for L in self.decode_layers)

    def qkv_flops(self):
        return sum(qkv_flops(L["spec"], self.pw.batch, self.pw.seq) for L in self.qkv_layers)

    def run_qkv_layer(self, L, stream):
        m = self.mimo
        st = m.mimo_attn_qkv_project(L["lay"], self.pw.batch, self.pw.seq, self.qkv_x, L["w"], None, 0, self.qkv_q,
                                     self.qkv_k, self.qkv_v, L["kc"], L["vc"], L["cap"], L["ws"], L["ws"].numel(),
                                     stream)
        if st != m.OK:
            raise m.MimoAttnError(st, "mimo_attn_qkv_project")

    def chunk_flops(self):
        return sum(chunk_flops(L["spec"], self.pw.batch, self.chunk_seq, self.chunk_past) for L in self.chunk_layers)

    def run_chunk_layer(self, L, stream):
        m = self.mimo
        st = m.mimo_attn_prefill_cached(L["lay"], m.BF16, self.pw.batch, self.chunk_seq, L["q"], L["k"], L["v"],
                                        self.past_dev, self.chunk_past, L["out"], L["kc"], L["vc"],
                                        L["kc"].shape[1], L["ws"], L["ws"].numel(), stream)
        if st != m.OK:
            raise m.MimoAttnError(st, "mimo_attn_prefill_cached")

    def decode_bytes(self):
        return sum(decode_bytes(L["spec"], self.lens, 1 if self.fp8 else 2) for L in self.decode_layers)

    def launches_per_step(self):
        # prefill: RoPE table + attention, plus the key pre-pass on global
        # layers (sliding layers rotate K inside the attention kernel)
        n = sum(3 if L["spec"].layer_type == 0 else 2 for L in self.prefill_layers)
        for L in self.chunk_layers:  # RoPE table + cache prep (1 global, 2 sliding) + attention
            n += 3 if L["spec"].layer_type == 0 else 4
        for L in self.decode_layers:
            n += 2 if L["need"] > 0 else 1  # split kernel (+ combine)
        n += 2 * len(self.qkv_layers)  # RoPE table + projection
        return n

    def run_prefill_layer(self, L, stream):
        m = self.mimo
        st = m.mimo_attn_prefill(L["lay"], m.BF16, self.pw.batch, self.pw.seq, L["q"], L["k"], L["v"], None,
                                 L["out"], None, None, 0, L["ws"], L["ws"].numel(), stream)
        if st != m.OK:
            raise m.MimoAttnError(st, "mimo_attn_prefill")

    def run_decode_layer(self, L, stream):
        m = self.mimo
        if self.fp8:
            st = m.mimo_attn_decode_fp8kv(L["lay"], self.dw.batch, L["q"], L["kn"], L["vn"], L["lens"], L["kc"],
                                          L["vc"], L["cap"], self.k_scale, self.v_scale, L["out"], L["ws"],
                                          L["ws"].numel(), stream)
            if st != m.OK:
                raise m.MimoAttnError(st, "mimo_attn_decode_fp8kv")
            return
        st = m.mimo_attn_decode(L["lay"], m.BF16, self.dw.batch, L["q"], L["kn"], L["vn"], L["lens"], L["kc"],
                                L["vc"], L["cap"], L["out"], L["ws"], L["ws"].numel(), stream)
        if st != m.OK:
            raise m.MimoAttnError(st, "mimo_attn_decode")

    def capture_decode(self):
        """Captures the decode stack (every layer's kernels) in one CUDA graph,
        as a serving loop replays it each step; the first, uncaptured pass sets
        the kernels' launch attributes."""
        if not self.decode_layers:
            return
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for L in self.decode_layers:
                self.run_decode_layer(L, side)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            cs = torch.cuda.current_stream()
            for L in self.decode_layers:
                self.run_decode_layer(L, cs)
        torch.cuda.synchronize()
        self.decode_graph = g

    def run_decode_stack(self, stream):
        if getattr(self, "decode_graph", None) is not None:
            self.decode_graph.replay()
        else:
            for L in self.decode_layers:
                self.run_decode_layer(L, stream)

    def step(self, stream, events=None):
        """One pass of the hot path. events: optional dict of lists collecting
        (start, end) CUDA events per call kind, recorded on `stream`."""
        for L in self.prefill_layers:
            kind = "prefill_global" if L["spec"].layer_type == 0 else "prefill_swa"
            if events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                self.run_prefill_layer(L, stream)
                e1.record(stream)
                events.setdefault(kind, []).append((e0, e1))
            else:
                self.run_prefill_layer(L, stream)
        for L in self.chunk_layers:
            kind = "chunk_global" if L["spec"].layer_type == 0 else "chunk_swa"
            if events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                self.run_chunk_layer(L, stream)
                e1.record(stream)
                events.setdefault(kind, []).append((e0, e1))
            else:
                self.run_chunk_layer(L, stream)
        for L in self.qkv_layers:
            kind = "qkv_global" if L["spec"].layer_type == 0 else "qkv_swa"
            if events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                self.run_qkv_layer(L, stream)
                e1.record(stream)
                events.setdefault(kind, []).append((e0, e1))
            else:
                self.run_qkv_layer(L, stream)
        if self.decode_layers:
            if events is not None:
                e0 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            self.run_decode_stack(stream)
            if events is not None:
                e1 = torch.cuda.Event(enable_timing=True)
                e1.record(stream)
                events.setdefault("decode_stack", []).append((e0, e1))


# ------------------------------------------------------------------ e2e
class HostInputs:
    """Pinned host buffers of every step input and result. Layers of the same
    shape share one pinned set (bounded host memory); each step still copies
    every layer's full inputs host->device and its full result back.

    The copies are pipelined with the compute, as a serving loop would: per
    prefill layer, its inputs go host->device on one copy stream, the layer
    runs on the compute stream once they have landed, and its output goes
    device->host on a second copy stream (the two directions use separate
    copy engines). The decode stack's inputs follow the prefill inputs, and
    its outputs are read back after it. Per-layer events keep the next step's
    copies off buffers still in use: a layer's inputs are overwritten only
    after its compute has read them, its output only after it was read back.
    Consecutive steps overlap the same way: the next step's first inputs go
    host->device while the previous step's last outputs come back."""

    def __init__(self, w: StackWorkload):
        self.w = w
        shared = {}

        def pinned_like(t, key, fill_from=None):
            k = (key, tuple(t.shape), t.dtype)
            if k not in shared:
                h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                if fill_from is not None:
                    h.copy_(fill_from)
                shared[k] = h
            return shared[k]

        # one unit per prefill layer, then one for the whole decode stack
        self.units = []
        for L in w.prefill_layers:
            ins = [(L[key], pinned_like(L[key], key, L[key])) for key in ("q", "k", "v")]
            outs = [(L["out"], pinned_like(L["out"], "out"))]
            self.units.append((L, ins, outs))
        if w.decode_layers:
            ins, outs = [], []
            for L in w.decode_layers:
                ins += [(L[key], pinned_like(L[key], "dec_" + key, L[key])) for key in ("q", "kn", "vn")]
                outs.append((L["out"], pinned_like(L["out"], "dec_out")))
            self.units.append((None, ins, outs))
        self.h2d = sum(h.numel() * h.element_size() for _, ins, _ in self.units for _, h in ins)
        self.d2h = sum(h.numel() * h.element_size() for _, _, outs in self.units for _, h in outs)
        self.pinned_bytes = sum(h.numel() * h.element_size() for h in shared.values())
        self.s_in = torch.cuda.Stream()
        self.s_out = torch.cuda.Stream()
        n = len(self.units)
        self.landed = [torch.cuda.Event() for _ in range(n)]
        self.computed = [torch.cuda.Event() for _ in range(n)]
        self.read_back = [torch.cuda.Event() for _ in range(n)]
        self.primed = False

    def step(self, stream, follows_step: bool = False):
        """One step; `stream` ends after the step's last read-back. Its
        copies start after the work already queued on `stream`, or, when it
        directly follows another step of this object (`follows_step`), as
        soon as the per-layer events of that step allow."""
        if not follows_step:
            start = torch.cuda.Event()
            start.record(stream)
            self.s_in.wait_event(start)
        for u, (L, ins, outs) in enumerate(self.units):
            with torch.cuda.stream(self.s_in):
                if self.primed:
                    self.s_in.wait_event(self.computed[u])
                for d, h in ins:
                    d.copy_(h, non_blocking=True)
                self.landed[u].record(self.s_in)
            with torch.cuda.stream(stream):  # (the decode graph replays on the current stream)
                stream.wait_event(self.landed[u])
                if self.primed:
                    stream.wait_event(self.read_back[u])
                if L is not None:
                    self.w.run_prefill_layer(L, stream)
                else:
                    self.w.run_decode_stack(stream)
                self.computed[u].record(stream)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.computed[u])
                for d, h in outs:
                    h.copy_(d, non_blocking=True)
                self.read_back[u].record(self.s_out)
        stream.wait_event(self.read_back[-1])
        self.primed = True


# ------------------------------------------------------------------ oracle
def host_cores() -> int:
    """Cores this process may run on (the oracle's thread count)."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.lower().startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _run_parallel(tasks, threads: int, seconds: float = None):
    """Runs the callables of `tasks` (an iterator; each returns its FLOPs) on
    `threads` host threads, until the iterator ends or, when `seconds` is
    given, until that much wall time has passed (tasks already started
    finish). The oracle's C routines release the GIL, so the threads run on
    separate cores. Returns (FLOPs, wall seconds, tasks run)."""
    from concurrent.futures import FIRST_COMPLETED, ThreadPoolExecutor, wait
    flops, n = 0.0, 0
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        live = set()
        it = iter(tasks)
        exhausted = False
        while True:
            while not exhausted and len(live) < 2 * threads and (
                    seconds is None or time.perf_counter() - t0 < seconds):
                try:
                    live.add(ex.submit(next(it)))
                except StopIteration:
                    exhausted = True
            if not live:
                break
            done, live = wait(live, return_when=FIRST_COMPLETED)
            for f in done:
                flops += f.result()
                n += 1
            if seconds is not None and time.perf_counter() - t0 >= seconds:
                exhausted = True
    return flops, time.perf_counter() - t0, n


class _OracleInputs:
    """Host copies of synthetic inputs for the oracle's timing runs, drawn
    once per layer kind before the clock starts (values N(0,1) rounded to
    bf16, as on the device)."""

    def __init__(self, seed: int):
        self.seed = seed
        self.cache = {}

    def get(self, key, shape, tid):
        if key not in self.cache:
            self.cache[key] = synthetic.normal(shape, seed=self.seed, tensor_id=tid,
                                               dtype=torch.bfloat16).double().numpy()
        return self.cache[key]


def _prefill_row_task(inp, spec, S, i, li):
    """One query row of one head: rotate its visible keys and the query, attend."""
    import oracle
    lo = 0 if spec.layer_type == 0 else max(0, i - spec.window + 1)
    k = inp.get(("k", spec.layer_type, S), (S, spec.qk_dim), 1000 + spec.layer_type)
    v = inp.get(("v", spec.layer_type, S), (S, spec.v_dim), 2000 + spec.layer_type)
    q = inp.get(("q", spec.layer_type), (64, spec.qk_dim), 3000 + spec.layer_type)

    def run():
        pos = np.arange(lo, i + 1, dtype=np.float64)
        kr = oracle.rope(k[lo:i + 1], spec.rotary_dim, spec.theta, pos)
        qr = oracle.rope(q[li % 64:li % 64 + 1], spec.rotary_dim, spec.theta, [float(i)])
        oracle.prefill_rows(qr, [i - lo], kr, v[lo:i + 1], spec.layer_type, spec.window,
                            1 / math.sqrt(spec.qk_dim), 0.5 if spec.has_sink else None, 0.7)
        return (i - lo + 1) * 2.0 * (spec.qk_dim + spec.v_dim)
    return run


def _decode_group_task(inp, spec, L, li, fp8, e4m3_of):
    """One KV group of one sequence: the G query heads against the cache."""
    import oracle
    cap = spec.window if spec.layer_type == 1 else 32768
    G = spec.num_q_heads // spec.num_kv_heads
    kc = inp.get(("kc", spec.layer_type), (cap, spec.qk_dim), 4000 + spec.layer_type)
    vc = inp.get(("vc", spec.layer_type), (cap, spec.v_dim), 5000 + spec.layer_type)
    q = inp.get(("dq", spec.layer_type), (G, spec.qk_dim), 6000 + spec.layer_type)
    kn = inp.get(("kn", spec.layer_type), (spec.qk_dim,), 7000 + spec.layer_type)
    vn = inp.get(("vn", spec.layer_type), (spec.v_dim,), 8000 + spec.layer_type)
    sinks = np.zeros(G) if spec.has_sink else None
    c = cap if spec.layer_type == 1 else L
    if fp8:
        for key, src, scale in ((("kc8", spec.layer_type), kc, 1 / 16), (("vc8", spec.layer_type), vc, 1 / 32)):
            if key not in inp.cache:
                inp.cache[key] = e4m3_of(src, scale)
        kc8, vc8 = inp.cache[("kc8", spec.layer_type)], inp.cache[("vc8", spec.layer_type)]

    def run():
        if fp8:
            oracle.decode_fp8kv(q, kn, vn, kc8[:c], vc8[:c], L, spec.rotary_dim, spec.theta, spec.layer_type,
                                spec.window, 1 / math.sqrt(spec.qk_dim), sinks, 0.7, 1 / 16, 1 / 32)
        else:
            oracle.decode(q, kn, vn, kc[:c], vc[:c], L, spec.rotary_dim, spec.theta, spec.layer_type,
                          spec.window, 1 / math.sqrt(spec.qk_dim), sinks, 0.7)
        n = min(L, spec.window) if spec.layer_type == 1 else L
        return G * n * 2.0 * (spec.qk_dim + spec.v_dim)
    return run


def oracle_sample(seconds: float, seed: int = 1, kind: str = "stack", threads: int = None):
    """Times the fp64 oracle, threaded over all host cores, on a bounded
    sample of the workload: for every prefill layer in turn, query rows at
    uniform positions against their whole visible key range; for every
    decode layer, one KV group of one sequence of uniform length. Inputs are
    drawn before the clock starts. Returns (unmasked FLOPs done, wall
    seconds, description, threads)."""
    import oracle
    oracle.build()
    threads = threads or host_cores()
    if kind not in ("stack", "swa", "global", "decode", "decode_fp8", "chunked", "qkv"):
        raise ValueError(f"no oracle sample for workload {kind!r}")
    rng = np.random.default_rng(seed)
    pw = {"stack": synthetic.HYBRID_PREFILL, "swa": synthetic.SWA_PREFILL, "global": synthetic.GLOBAL_PREFILL,
          "chunked": synthetic.HYBRID_PREFILL}.get(kind)
    dw = synthetic.HYBRID_DECODE if kind in ("stack", "decode", "decode_fp8") else None
    fp8 = kind == "decode_fp8"
    row_lo = CHUNK_PAST if kind == "chunked" else 0  # chunked: rows in the stack's last CHUNK_SEQ positions
    inp = _OracleInputs(seed)
    tables = {}

    def e4m3_of(x, scale):
        # the oracle's codes of bf16 values, through one table over all 65536 patterns
        if scale not in tables:
            with np.errstate(all="ignore"):
                quot = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32) / np.float32(scale)
            tables[scale] = oracle.e4m3_encode(np.nan_to_num(quot, nan=0.0).astype(np.float64))
        bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.int64) & 0xFFFF
        return tables[scale][bits]

    if kind == "qkv":
        from threadpoolctl import threadpool_limits
        spec = synthetic.HYBRID_PREFILL.layers[0]
        x16, w16 = synthetic.projection_inputs(spec, 1, 64, seed=seed, layer=0)
        x, w = x16[0].double().numpy(), w16.double().numpy()
        flops, rows = 0.0, 0
        with threadpool_limits(limits=threads):  # numpy's BLAS on every core
            t0 = time.perf_counter()
            while time.perf_counter() - t0 < seconds:
                oracle.qkv_project(x, w, np.arange(x.shape[0]), num_q_heads=spec.num_q_heads,
                                   num_kv_heads=spec.num_kv_heads, qk_dim=spec.qk_dim, v_dim=spec.v_dim,
                                   rotary_dim=spec.rotary_dim, theta=spec.theta)
                flops += 2.0 * x.shape[0] * w.shape[0] * x.shape[1]
                rows += x.shape[0]
            t = time.perf_counter() - t0
        return flops, t, (f"{rows} tokens of the global layer's QKV projection (all 13568 features, RoPE); fp64 "
                          f"oracle, numpy matmul on {threads} BLAS threads"), threads

    def tasks():
        n = 0
        while True:
            if pw is not None:
                for li, spec in enumerate(pw.layers):
                    yield _prefill_row_task(inp, spec, pw.seq, int(rng.integers(row_lo, pw.seq)), n + li)
            if dw is not None:
                for li, spec in enumerate(dw.layers):
                    L = int(rng.integers(dw.kv_len_range[0], dw.kv_len_range[1] + 1))
                    yield _decode_group_task(inp, spec, L, li, fp8, e4m3_of)
            n += 1

    # draw the inputs of every layer kind before the clock starts
    warm = tasks()
    for _ in range((len(pw.layers) if pw else 0) + (len(dw.layers) if dw else 0)):
        next(warm)
    flops, t, n = _run_parallel(tasks(), threads, seconds)
    what = []
    if pw is not None:
        what.append(f"prefill query rows at uniform positions{' in the chunk' if row_lo else ''} (all visible keys, "
                    f"every layer of the workload in turn)")
    if dw is not None:
        what.append(f"decode KV groups (one sequence of uniform length, all query heads of the group"
                    f"{', E4M3 caches' if fp8 else ''})")
    desc = f"{n} units: " + " + ".join(what) + f"; fp64 C oracle on {threads} threads ({cpu_model()})"
    return flops, t, desc, threads


# ------------------------------------------------------------------ traffic
def committed_traffic(kernel_tag: str, source: str, tokens: int):
    """Per-launch DRAM bytes from the committed ncu summary profiles/<kernel_tag>.md,
    valid only while the kernel's source file (csrc/<source>) still matches the
    hash recorded there. The summary gives the bytes of its capture and the
    tokens (batch x sequence) the captured launch processed; this kernel's
    traffic grows with the tokens (Q, K, V read once, O written once), so the
    capture is scaled to `tokens`."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    src = os.path.join(ROOT, "global_attention_partial_b200", "csrc", source)
    if not os.path.exists(path) or not os.path.exists(src):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    vals = {}
    for ln in open(path):
        if ":" in ln and ln.strip().startswith("- "):
            k, _, v = ln.strip()[2:].partition(":")
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != sha:
        return None
    try:
        return float(vals["dram_bytes_per_capture"]) * tokens / float(vals["tokens_per_capture"])
    except (KeyError, ValueError, ZeroDivisionError):
        return None


# ------------------------------------------------------------------ main
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        return dist, dist.get_rank(), world, local
    return None, 0, 1, 0


def barrier(dist, local):
    if dist is not None:
        dist.barrier(device_ids=[local])


def max_over_ranks(dist, x: float, device="cuda") -> float:
    """Max of x over all ranks (the step time of the slowest GPU)."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, units_per_rank: float, ms_max: float) -> float:
    """Whole-job throughput (weak scaling): every rank processes the same
    units; the job takes as long as the slowest rank. TFLOP/s for FLOP units."""
    return world * units_per_rank / (ms_max * 1e-3) / 1e12


def run_reference(args):
    """CPU oracle arm: rank 0 times the oracle, threaded over the host cores,
    on bounded samples of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if args.oracle_table:
        print(json.dumps(oracle_table(args)), flush=True)
        return
    per_step = float(os.environ.get("MIMO_REF_STEP_SECONDS", "6"))
    for _ in range(args.warmup):
        oracle_sample(min(per_step, 1.0), seed=99, kind=args.workload)
    flops_total, t_total, desc, threads = 0.0, 0.0, "", 1
    for s in range(args.steps):
        f, t, desc, threads = oracle_sample(per_step, seed=s, kind=args.workload)
        flops_total += f
        t_total += t
    value = flops_total / t_total / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * t_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args, reference=True),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
                             "cpu_model": cpu_model()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def oracle_table(args):
    """Wall time of the fp64 oracle over whole configurations, threaded over
    the host cores: the tiny fp32 pair, the SWA layer (B1 S4096), the global
    layer (B2 S8192) and the hybrid decode (B64, every layer) in full; the
    hybrid prefill stack (B4 S32768) on a sample of query rows, extrapolated
    by unmasked FLOPs (each row's cost is proportional to its visible keys).
    The inputs are the synthetic ones (CPU draws, bf16)."""
    import oracle
    oracle.build()
    threads = host_cores()
    res = {"cores": threads, "cpu_model": cpu_model(), "configs": {}}
    seed = 0

    def time_layer(spec, B, S, rows_per_head, dtype=torch.bfloat16, batches=None):
        """Times one layer in the oracle's own order (oracle.prefill_layer):
        rotate each (batch, KV head)'s keys once, then per (batch, query head)
        rotate the query rows and attend them. Both phases run on the thread
        pool. `batches` limits the timed sequences (the others are alike);
        rows_per_head(b, h) picks the rows (all, or a sample). Returns
        (estimated seconds for all B sequences and all rows, measured
        seconds, attention FLOPs done)."""
        Hq, G = spec.num_q_heads, spec.num_q_heads // spec.num_kv_heads
        nb = B if batches is None else batches
        q, k, v, sinks = synthetic.prefill_inputs(spec, nb, S, seed=seed, layer=0, dtype=dtype)
        sn = None if sinks is None else sinks.double().numpy()
        pos = np.arange(S, dtype=np.float64)
        scale = 1 / math.sqrt(spec.qk_dim)
        vs = oracle.v_scale(spec.hidden_size, Hq, spec.v_dim)
        k_rot = {}

        def rotate(b, kv):
            def run():
                k_rot[(b, kv)] = (oracle.rope(k[b, :, kv].double().numpy(), spec.rotary_dim, spec.theta, pos),
                                  v[b, :, kv].double().numpy())
                return 0.0
            return run

        def attend(b, h, rows):
            def run():
                kr, vv = k_rot[(b, h // G)]
                qr = oracle.rope(q[b, rows, h].double().numpy(), spec.rotary_dim, spec.theta, pos[rows])
                oracle.prefill_rows(qr, rows, kr, vv, spec.layer_type, spec.window, scale,
                                    None if sn is None else float(sn[h]), vs)
                lo = np.maximum(0, rows - spec.window + 1) if spec.layer_type == 1 else 0
                return float(np.sum(rows - lo + 1)) * 2 * (spec.qk_dim + spec.v_dim)
            return run

        _, t_rot, _ = _run_parallel([rotate(b, kv) for b in range(nb) for kv in range(spec.num_kv_heads)], threads)
        f, t_att, _ = _run_parallel([attend(b, h, rows_per_head(b, h)) for b in range(nb) for h in range(Hq)],
                                    threads)
        full = prefill_flops(spec, B, S)
        # key rotation: once per (batch, KV head), scaled to B sequences;
        # attention: proportional to FLOPs (each row costs its visible keys)
        return t_rot * B / nb + t_att * full / f, t_rot + t_att, f

    def record(name, mode, est, meas, done, full):
        res["configs"][name] = {"mode": mode, "oracle_s": est, "measured_s": meas, "flops_done": done,
                                "flops_full": full, "gflops_per_s": full / est / 1e9}

    # tiny fp32 pair, in full
    est = meas = done = full = 0.0
    for spec in synthetic.TINY_PAIR.layers:
        e, m, d = time_layer(spec, 1, 64, lambda b, h: np.arange(64), dtype=torch.float32)
        est, meas, done, full = est + e, meas + m, done + d, full + prefill_flops(spec, 1, 64)
    record("c0 tiny fp32 pair", "full", est, meas, done, full)
    # SWA layer B1 S4096, in full
    spec = synthetic.SWA_PREFILL.layers[0]
    e, m, d = time_layer(spec, 1, 4096, lambda b, h: np.arange(4096))
    record("c1 SWA B1 S4096", "full", e, m, d, prefill_flops(spec, 1, 4096))
    # global layer B2 S8192, in full (under a minute on 16 cores)
    spec = synthetic.GLOBAL_PREFILL.layers[0]
    rng = np.random.default_rng(1)
    e, m, d = time_layer(spec, 2, 8192, lambda b, h: np.arange(8192))
    record("c2 global B2 S8192", "full", e, m, d, prefill_flops(spec, 2, 8192))
    # hybrid stack B4 S32768: each layer kind timed on one sequence (the four
    # are alike), 8 uniform rows per head, extrapolated to its layers of the
    # stack (2 global, 6 sliding) over all 4 sequences
    est = meas = done = 0.0
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        e, m, d = time_layer(spec, 4, 32768, lambda b, h: np.sort(rng.integers(0, 32768, 8)), batches=1)
        n_layers = sum(1 for sp in synthetic.HYBRID_PREFILL.layers if sp.layer_type == lt)
        est, meas, done = est + n_layers * e, meas + m, done + d
    record("c3 hybrid stack B4 S32768", "sampled, extrapolated", est, meas, done,
           sum(prefill_flops(sp, 4, 32768) for sp in synthetic.HYBRID_PREFILL.layers))
    # hybrid decode B64, every layer and every KV group, in full
    dw = synthetic.HYBRID_DECODE
    lens = synthetic.decode_kv_lens(dw.batch, *dw.kv_len_range, seed=seed).tolist()
    inp = _OracleInputs(seed)
    tasks = [_decode_group_task(inp, spec, L, li, False, None) for li, spec in enumerate(dw.layers)
             for L in lens for _ in range(spec.num_kv_heads)]
    f, t, _ = _run_parallel(tasks, threads)
    record("c4 hybrid decode B64", "full", t, t, f, sum(decode_flops(spec, lens) for spec in dw.layers))
    return res


def workload_config(args, reference=False, kind=None):
    kind = kind or args.workload
    names = {"stack": f"{synthetic.HYBRID_PREFILL.name} + {synthetic.HYBRID_DECODE.name}",
             "swa": synthetic.SWA_PREFILL.name, "global": synthetic.GLOBAL_PREFILL.name,
             "decode": synthetic.HYBRID_DECODE.name,
             "decode_fp8": synthetic.HYBRID_DECODE.name.replace("bf16", "bf16 q/out, fp8 E4M3 KV cache"),
             "qkv": "hybrid 8-layer stack QKV projection (x W^T + RoPE + q/k/v and cache stores) bf16 B4 S32768 "
                    "hidden 4096 pattern 0,1,1,1,1,1,0,1",
             "chunked": f"hybrid 8-layer stack, chunk of {CHUNK_SEQ} tokens after {CHUNK_PAST} cached, bf16 B4 "
                        f"pattern 0,1,1,1,1,1,0,1"}
    pw = {"swa": synthetic.SWA_PREFILL, "global": synthetic.GLOBAL_PREFILL}.get(kind, synthetic.HYBRID_PREFILL)
    cfg = {"workload": names[kind], "prefill_batch": pw.batch, "prefill_seq": pw.seq,
           "decode_batch": synthetic.HYBRID_DECODE.batch,
           "kv_len_range": list(synthetic.HYBRID_DECODE.kv_len_range),
           "layers": ",".join(str(t) for t in pw.pattern),
           "parallelism": f"replicas x{args.gpus} (weak, no collective on the data path)",
           "l2": "no flush: each step streams ~60 GB of inputs, far above the 126 MB L2"}
    if kind in ("stack", "decode", "decode_fp8"):
        cfg["decode_launch"] = ("direct C-ABI calls, one per layer" if args.no_graph else
                                "the 8 layers' C-ABI calls captured once in a CUDA graph, replayed each step")
    if kind != "stack":
        cfg["l2"] = "inputs larger than L2" if kind != "swa" else "L2 flushed between steps (256 MB write)"
    if args.layers is not None and kind == args.workload:
        cfg["layer_subset"] = args.layers
    if (args.batch is not None or args.seq is not None) and kind == args.workload:
        cfg["prefill_override"] = {"batch": args.batch, "seq": args.seq}
    return cfg


def time_workload(w, steps, warmup, stream, dist=None, local=0, sample_clocks=False):
    """Warm-up, then `steps` timed steps bracketed by a barrier and a
    synchronize on both sides, CUDA events on `stream`. The SWA layer alone
    fits in L2, so its steps flush L2 first (a 256 MB write, outside the
    events). Returns (ms per step, max over ranks; per-call-kind event times;
    clocks or None)."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda") if w.kind == "swa" else None
    for _ in range(max(warmup, 0)):
        w.step(stream)
    torch.cuda.synchronize()
    if w.mimo.mimo_attn_get_device_error() != 0:
        raise RuntimeError(f"device error word set during the {w.kind} warm-up")
    sampler = ClockSampler(local) if sample_clocks else None
    if sampler:
        sampler.start()
    events = {}
    barrier(dist, local)
    torch.cuda.synchronize()
    step_events = []
    for _ in range(steps):
        if flush is not None:
            flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        w.step(stream, events)
        e1.record(stream)
        step_events.append((e0, e1))
    torch.cuda.synchronize()
    barrier(dist, local)
    clocks = sampler.stop() if sampler else None
    ms_local = sum(a.elapsed_time(b) for a, b in step_events) / steps
    ms = max_over_ranks(dist, ms_local)
    kinds = {k: [a.elapsed_time(b) for a, b in v] for k, v in events.items()}
    if w.mimo.mimo_attn_get_device_error() != 0:
        raise RuntimeError(f"device error word set while timing {w.kind}")
    return ms, kinds, clocks


def summarize(w, ms, kinds, steps, peaks, stream):
    """Step FLOPs, per-part rates and the roofline object of the workload's
    dominant kernel, from the CUDA-event times of time_workload."""
    pflops = w.prefill_flops() if w.do_prefill else 0.0
    dflops = w.decode_flops() if w.do_decode else 0.0
    cflops = w.chunk_flops() if w.do_chunked else 0.0
    qflops = w.qkv_flops() if w.do_qkv else 0.0
    step_flops = pflops + dflops + cflops + qflops
    sustained = peaks["bf16_tflops_sustained"]
    parts = {}
    roofline = None
    if w.do_prefill:
        ms_prefill = (sum(sum(v) for k, v in kinds.items() if k.startswith("prefill")) / steps)
        parts["prefill"] = {"ms": ms_prefill, "tflops": pflops / (ms_prefill * 1e-3) / 1e12,
                            "frac_of_tensor_peak": pflops / (ms_prefill * 1e-3) / 1e12 / sustained}
        for kind, lt in (("prefill_global", 0), ("prefill_swa", 1)):
            if kind not in kinds:
                continue
            specs = [L["spec"] for L in w.prefill_layers if L["spec"].layer_type == lt]
            per = statistics.mean(kinds[kind])
            f = prefill_flops(specs[0], w.pw.batch, w.pw.seq)
            byt = prefill_bytes(specs[0], w.pw.batch, w.pw.seq)
            parts[kind.replace("prefill_", "") + "_layer"] = {
                "ms_per_launch": per, "tflops": f / (per * 1e-3) / 1e12,
                "frac_of_tensor_peak": f / (per * 1e-3) / 1e12 / sustained,
                "gbs_compulsory": byt / (per * 1e-3) / 1e9,
                "frac_of_hbm_peak": byt / (per * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        dom = "prefill_global" if "prefill_global" in kinds else "prefill_swa"
        lt = 0 if dom == "prefill_global" else 1
        spec = [L["spec"] for L in w.prefill_layers if L["spec"].layer_type == lt][0]
        per = statistics.mean(kinds[dom])
        if lt == 0:
            ach = prefill_flops(spec, w.pw.batch, w.pw.seq) / (per * 1e-3) / 1e12
            roofline = {"bound": "tensor", "achieved": ach, "peak": sustained,
                        "unit": "TFLOP/s", "frac": ach / sustained,
                        "traffic": committed_traffic("prefill_ga_global", "prefill_ga.cu", w.pw.batch * w.pw.seq),
                        "kernel": f"prefill_ga_kernel (global layer, B{w.pw.batch} S{w.pw.seq} causal)",
                        "peak_kind": f"bf16 dense, sustained, {peaks['source']}"}
        else:
            ach = prefill_bytes(spec, w.pw.batch, w.pw.seq) / (per * 1e-3) / 1e9
            roofline = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / peaks["hbm_gbs"],
                        "traffic": committed_traffic("prefill_swa_sliding", "prefill_swa.cu", w.pw.batch * w.pw.seq),
                        "kernel": f"prefill_swa_kernel (sliding layer, B{w.pw.batch} S{w.pw.seq})",
                        "peak_kind": f"HBM copy, {peaks['source']}"}
    if w.do_chunked:
        for kind, lt in (("chunk_global", 0), ("chunk_swa", 1)):
            if kind not in kinds:
                continue
            specs = [L["spec"] for L in w.chunk_layers if L["spec"].layer_type == lt]
            per = statistics.mean(kinds[kind])
            f = chunk_flops(specs[0], w.pw.batch, w.chunk_seq, w.chunk_past)
            parts[kind + "_layer"] = {"ms_per_launch": per, "tflops": f / (per * 1e-3) / 1e12,
                                      "frac_of_tensor_peak": f / (per * 1e-3) / 1e12 / sustained}
        if "chunk_global_layer" in parts:
            ach = parts["chunk_global_layer"]["tflops"]
            roofline = {"bound": "tensor", "achieved": ach, "peak": sustained, "unit": "TFLOP/s",
                        "frac": ach / sustained, "traffic": None,
                        "kernel": "prefill_ga_kernel (global layer, chunk of 4096 after 28672 cached, B4)",
                        "peak_kind": f"bf16 dense, sustained, {peaks['source']}"}
    if w.do_qkv:
        for kind, lt in (("qkv_global", 0), ("qkv_swa", 1)):
            if kind not in kinds:
                continue
            spec = [L["spec"] for L in w.qkv_layers if L["spec"].layer_type == lt][0]
            per = statistics.mean(kinds[kind])
            f = qkv_flops(spec, w.pw.batch, w.pw.seq)
            parts[kind + "_layer"] = {"ms_per_launch": per, "tflops": f / (per * 1e-3) / 1e12,
                                      "frac_of_tensor_peak": f / (per * 1e-3) / 1e12 / sustained}
        key = "qkv_swa_layer" if "qkv_swa_layer" in parts else "qkv_global_layer"
        ach = parts[key]["tflops"]
        roofline = {"bound": "tensor", "achieved": ach, "peak": sustained, "unit": "TFLOP/s",
                    "frac": ach / sustained, "traffic": None,
                    "kernel": f"qkv_proj_kernel ({key[4:-6]} layer, B{w.pw.batch} S{w.pw.seq}, hidden 4096)",
                    "peak_kind": f"bf16 dense, sustained, {peaks['source']}"}
    if w.do_decode:
        per = statistics.mean(kinds["decode_stack"])
        byt = w.decode_bytes()
        parts["decode"] = {"ms_per_stack": per, "gbs": byt / (per * 1e-3) / 1e9,
                           "frac_of_hbm_peak": byt / (per * 1e-3) / 1e9 / peaks["hbm_gbs"],
                           "bytes_per_stack": byt,
                           "launch": "direct calls" if getattr(w, "decode_graph", None) is None else "CUDA graph"}
        if getattr(w, "decode_graph", None) is not None:
            # the same stack as back-to-back direct calls, outside the timed region
            d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            reps = 5
            d0.record(stream)
            for _ in range(reps):
                for L in w.decode_layers:
                    w.run_decode_layer(L, stream)
            d1.record(stream)
            torch.cuda.synchronize()
            per_d = d0.elapsed_time(d1) / reps
            parts["decode"]["ms_per_stack_direct_calls"] = per_d
            parts["decode"]["gbs_direct_calls"] = byt / (per_d * 1e-3) / 1e9
        if roofline is None:
            ach = byt / (per * 1e-3) / 1e9
            roofline = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / peaks["hbm_gbs"], "traffic": None,
                        "kernel": "decode_mma_kernel (%d-layer stack%s)" % (
                            len(w.decode_layers), ", fp8 KV cache" if w.fp8 else ""),
                        "peak_kind": f"HBM copy, {peaks['source']}"}
    return step_flops, parts, roofline


# The configurations and NEXT-row workloads timed after the headline step
# (outside its timed region), each reported under parts.configs.
EXTRA_PARTS = ("swa", "global", "decode", "decode_fp8", "chunked", "qkv")


def extra_parts(args, peaks, stream):
    out = {}
    for kind in EXTRA_PARTS:
        w = StackWorkload(kind)
        if not args.no_graph:
            w.capture_decode()
        steps = 20 if kind in ("swa", "global", "decode", "decode_fp8") else 3
        ms, kinds, _ = time_workload(w, steps, 3, stream)
        step_flops, parts, roofline = summarize(w, ms, kinds, steps, peaks, stream)
        out[kind] = {"workload": workload_config(args, kind=kind)["workload"], "ms_per_step": ms, "steps": steps,
                     "tflops": step_flops / (ms * 1e-3) / 1e12, "roofline": roofline, "parts": parts}
        del w
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["stack", "swa", "global", "decode", "chunked", "decode_fp8", "qkv"],
                    default="stack")
    ap.add_argument("--layers", type=lambda x: [int(i) for i in x.split(",")], default=None,
                    help="comma-separated layer indices of the workload to run (default: all), e.g. to profile one")
    ap.add_argument("--batch", type=int, default=None, help="override the prefill batch (prefill / qkv workloads)")
    ap.add_argument("--seq", type=int, default=None, help="override the prefill length (prefill / qkv workloads)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-parts", action="store_true",
                    help="skip timing the other configurations after the stack step")
    ap.add_argument("--no-graph", action="store_true", help="launch the decode layers one call at a time")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--oracle-table", action="store_true",
                    help="with --impl reference: time the oracle over whole configurations (minutes)")
    args = ap.parse_args()
    if args.workload in ("chunked", "decode_fp8", "qkv") or args.layers is not None or args.seq or args.batch:
        args.no_e2e = True  # NEXT-row and profiling runs: no host-buffer leg
    if args.impl == "reference":
        run_reference(args)
        return

    dist, rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    import global_attention_partial_b200 as mimo
    mimo.load()
    peaks = measured_peaks()
    w = StackWorkload(args.workload, layers=args.layers, batch=args.batch, seq=args.seq)
    if not args.no_graph:
        w.capture_decode()
    stream = torch.cuda.current_stream()

    # ---- timed region (device-resident inputs)
    ms, kinds, clocks = time_workload(w, args.steps, args.warmup, stream, dist, local, sample_clocks=True)
    step_flops, parts, roofline = summarize(w, ms, kinds, args.steps, peaks, stream)
    value = job_value(world, step_flops, ms)

    # ---- e2e through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        host = HostInputs(w)
        e2e_steps = max(1, min(args.steps, 5))
        host.step(stream)
        torch.cuda.synchronize()
        barrier(dist, local)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(e2e_steps):
            host.step(stream, follows_step=i > 0)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(dist, local)
        ms_e2e = max_over_ranks(dist, e0.elapsed_time(e1) / e2e_steps)
        e2e = {"value": job_value(world, step_flops, ms_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": host.h2d, "d2h_bytes_per_step": host.d2h, "ms_per_step": ms_e2e,
               "steps": e2e_steps,
               "overlap": "per layer: host->device copy, compute and device->host copy on three streams; "
                          "a step's first inputs go in while the previous step's last outputs come back"}
        del host

    if mimo.mimo_attn_get_device_error() != 0:
        raise RuntimeError("device error word set during the timed region")
    launches = w.launches_per_step() * args.steps
    del w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # ---- the other configurations, outside the timed region (rank-local, 1 GPU runs only)
    if args.workload == "stack" and world == 1 and not args.no_parts and args.layers is None:
        parts["configs"] = extra_parts(args, peaks, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, t, desc, threads = oracle_sample(args.cpu_seconds, kind=args.workload)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
               "seconds": t, "cpu_model": cpu_model()}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None,
                "dtype": "e4m3 KV cache, f16 mma, fp32 accumulate" if args.workload == "decode_fp8" else "bf16",
                "data": "synthetic", "config": workload_config(args),
                "roofline": roofline, "parts": parts, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clocks, "peaks": peaks}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
