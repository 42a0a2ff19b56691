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

    def __init__(self, kind: str, seed: int = 0):
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
            for li, spec in enumerate(pw.layers):
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
            for li, spec in enumerate(pw.layers):
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
            for li, spec in enumerate(pw.layers):
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
            for li, spec in enumerate(dw.layers):
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
        n = 3 * len(self.prefill_layers)  # RoPE table + K-prep + attention
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
    every layer's full inputs host->device and its full result back."""

    def __init__(self, w: StackWorkload):
        self.w = w
        self.items_in = []
        self.items_out = []
        shared = {}

        def pinned_like(t, key, fill_from=None):
            k = (key, tuple(t.shape), t.dtype)
            if k not in shared:
                h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                if fill_from is not None:
                    h.copy_(fill_from)
                shared[k] = h
            return shared[k]

        for L in w.prefill_layers:
            for key in ("q", "k", "v"):
                self.items_in.append((L[key], pinned_like(L[key], key, L[key])))
            self.items_out.append((L["out"], pinned_like(L["out"], "out")))
        for L in w.decode_layers:
            for key in ("q", "kn", "vn"):
                self.items_in.append((L[key], pinned_like(L[key], "dec_" + key, L[key])))
            self.items_out.append((L["out"], pinned_like(L["out"], "dec_out")))
        self.h2d = sum(h.numel() * h.element_size() for _, h in self.items_in)
        self.d2h = sum(h.numel() * h.element_size() for _, h in self.items_out)
        self.pinned_bytes = sum(h.numel() * h.element_size() for h in shared.values())

    def step(self, stream):
        with torch.cuda.stream(stream):
            for d, h in self.items_in:
                d.copy_(h, non_blocking=True)
            self.w.step(stream)
            for d, h in self.items_out:
                h.copy_(d, non_blocking=True)


# ------------------------------------------------------------------ oracle
def oracle_sample(seconds: float, seed: int = 1, kind: str = "stack"):
    """Times the fp64 oracle on a bounded sample of the workload: for every
    prefill layer, query rows at uniform positions against their whole
    visible key range; for every decode layer, one KV group of one sequence.
    Returns (unmasked FLOPs done, seconds, description)."""
    import oracle
    oracle.build()
    rng = np.random.default_rng(seed)
    flops, t_total, rows_done, groups_done = 0.0, 0.0, 0, 0
    if kind not in ("stack", "swa", "global", "decode", "decode_fp8", "chunked", "qkv"):
        raise ValueError(f"no oracle sample for workload {kind!r}")
    pw = {"stack": synthetic.HYBRID_PREFILL, "swa": synthetic.SWA_PREFILL, "global": synthetic.GLOBAL_PREFILL,
          "chunked": synthetic.HYBRID_PREFILL}.get(kind)
    dw = synthetic.HYBRID_DECODE if kind in ("stack", "decode", "decode_fp8") else None
    fp8 = kind == "decode_fp8"
    # chunked: query rows are the stack's last CHUNK_SEQ positions
    row_lo = CHUNK_PAST if kind == "chunked" else 0
    tables = {}

    def e4m3_of(x, scale):
        # the oracle's codes of bf16 values, through one table over all 65536 patterns
        if scale not in tables:
            with np.errstate(all="ignore"):
                quot = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32) / np.float32(scale)
            tables[scale] = oracle.e4m3_encode(np.nan_to_num(quot, nan=0.0).astype(np.float64))
        return tables[scale][x.view(torch.int16).numpy().astype(np.int64) & 0xFFFF]

    proj = None
    if kind == "qkv":
        spec = synthetic.HYBRID_PREFILL.layers[0]
        x16, w16 = synthetic.projection_inputs(spec, 1, 16, seed=seed, layer=0)
        proj = (spec, x16[0].double().numpy(), w16.double().numpy())
    t_start = time.perf_counter()
    while time.perf_counter() - t_start < seconds:
        if proj is not None:
            from threadpoolctl import threadpool_limits
            spec, x, w = proj
            with threadpool_limits(limits=1):  # one core, like the C oracle
                t0 = time.perf_counter()
                oracle.qkv_project(x, w, np.arange(x.shape[0]), num_q_heads=spec.num_q_heads,
                                   num_kv_heads=spec.num_kv_heads, qk_dim=spec.qk_dim, v_dim=spec.v_dim,
                                   rotary_dim=spec.rotary_dim, theta=spec.theta)
                t_total += time.perf_counter() - t0
            flops += 2.0 * x.shape[0] * w.shape[0] * x.shape[1]
            rows_done += x.shape[0]
        if pw is not None:
            for li, spec in enumerate(pw.layers):
                S = pw.seq
                i = int(rng.integers(row_lo, S))
                lo = 0 if spec.layer_type == 0 else max(0, i - spec.window + 1)
                n = i - lo + 1
                k = synthetic.normal((n, spec.qk_dim), seed=seed, tensor_id=1000 + li, dtype=torch.bfloat16)
                v = synthetic.normal((n, spec.v_dim), seed=seed, tensor_id=2000 + li, dtype=torch.bfloat16)
                q = synthetic.normal((1, spec.qk_dim), seed=seed, tensor_id=3000 + li, dtype=torch.bfloat16)
                pos = np.arange(lo, i + 1, dtype=np.float64)
                t0 = time.perf_counter()
                kr = oracle.rope(k.double().numpy(), spec.rotary_dim, spec.theta, pos)
                qr = oracle.rope(q.double().numpy(), spec.rotary_dim, spec.theta, [float(i)])
                oracle.prefill_rows(qr, [n - 1], kr, v.double().numpy(), spec.layer_type, spec.window,
                                    1 / math.sqrt(spec.qk_dim), 0.5 if spec.has_sink else None, 0.7)
                t_total += time.perf_counter() - t0
                flops += n * 2 * (spec.qk_dim + spec.v_dim)
                rows_done += 1
        if dw is not None:
            for li, spec in enumerate(dw.layers):
                L = int(rng.integers(dw.kv_len_range[0], dw.kv_len_range[1] + 1))
                cap = spec.window if spec.layer_type == 1 else L
                G = spec.num_q_heads // spec.num_kv_heads
                kc = synthetic.normal((cap, spec.qk_dim), seed=seed, tensor_id=4000 + li, dtype=torch.bfloat16)
                vc = synthetic.normal((cap, spec.v_dim), seed=seed, tensor_id=5000 + li, dtype=torch.bfloat16)
                q = synthetic.normal((G, spec.qk_dim), seed=seed, tensor_id=6000 + li, dtype=torch.bfloat16)
                kn = synthetic.normal((spec.qk_dim,), seed=seed, tensor_id=7000 + li, dtype=torch.bfloat16)
                vn = synthetic.normal((spec.v_dim,), seed=seed, tensor_id=8000 + li, dtype=torch.bfloat16)
                sinks = np.zeros(G) if spec.has_sink else None
                if fp8:
                    kc8, vc8 = e4m3_of(kc, 1 / 16), e4m3_of(vc, 1 / 32)
                    t0 = time.perf_counter()
                    oracle.decode_fp8kv(q.double().numpy(), kn.double().numpy(), vn.double().numpy(), kc8, vc8, L,
                                        spec.rotary_dim, spec.theta, spec.layer_type, spec.window,
                                        1 / math.sqrt(spec.qk_dim), sinks, 0.7, 1 / 16, 1 / 32)
                else:
                    t0 = time.perf_counter()
                    oracle.decode(q.double().numpy(), kn.double().numpy(), vn.double().numpy(), kc.double().numpy(),
                                  vc.double().numpy(), L, spec.rotary_dim, spec.theta, spec.layer_type, spec.window,
                                  1 / math.sqrt(spec.qk_dim), sinks, 0.7)
                t_total += time.perf_counter() - t0
                flops += G * (min(L, spec.window) if spec.layer_type == 1 else L) * 2 * (spec.qk_dim + spec.v_dim)
                groups_done += 1
    if proj is not None:
        desc = (f"{rows_done} tokens of the global layer's QKV projection (all 13568 features, RoPE); "
                f"fp64 oracle (numpy matmul on one BLAS thread)")
    else:
        desc = (f"{rows_done} prefill query rows (uniform positions{' in the chunk' if row_lo else ''}, all visible "
                f"keys, every layer of the stack) + {groups_done} decode KV groups (one sequence, all query heads "
                f"of the group{', E4M3 caches' if fp8 else ''}); fp64 C oracle, single thread")
    return flops, t_total, desc


# ------------------------------------------------------------------ traffic
def committed_traffic(kernel_tag: str, source: str):
    """Per-launch DRAM bytes from the committed ncu summary profiles/<kernel_tag>.md,
    valid only while the kernel's source file (csrc/<source>) still matches the
    hash recorded there."""
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
        return float(vals["dram_bytes_per_full_launch"])
    except (KeyError, ValueError):
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
    """CPU oracle arm: rank 0 times the oracle on bounded samples."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step = float(os.environ.get("MIMO_REF_STEP_SECONDS", "6"))
    for _ in range(args.warmup):
        oracle_sample(min(per_step, 1.0), seed=99, kind=args.workload)
    vals, flops_total, t_total, desc = [], 0.0, 0.0, ""
    for s in range(args.steps):
        f, t, desc = oracle_sample(per_step, seed=s, kind=args.workload)
        flops_total += f
        t_total += t
    value = flops_total / t_total / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * t_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(args, reference=True),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(args, reference=False):
    names = {"stack": f"{synthetic.HYBRID_PREFILL.name} + {synthetic.HYBRID_DECODE.name}",
             "swa": synthetic.SWA_PREFILL.name, "global": synthetic.GLOBAL_PREFILL.name,
             "decode": synthetic.HYBRID_DECODE.name,
             "decode_fp8": synthetic.HYBRID_DECODE.name.replace("bf16", "bf16 q/out, fp8 E4M3 KV cache"),
             "qkv": "hybrid 8-layer stack QKV projection (x W^T + RoPE + q/k/v and cache stores) bf16 B4 S32768 "
                    "hidden 4096 pattern 0,1,1,1,1,1,0,1",
             "chunked": f"hybrid 8-layer stack, chunk of {CHUNK_SEQ} tokens after {CHUNK_PAST} cached, bf16 B4 "
                        f"pattern 0,1,1,1,1,1,0,1"}
    cfg = {"workload": names[args.workload], "prefill_batch": synthetic.HYBRID_PREFILL.batch,
           "prefill_seq": synthetic.HYBRID_PREFILL.seq, "decode_batch": synthetic.HYBRID_DECODE.batch,
           "kv_len_range": list(synthetic.HYBRID_DECODE.kv_len_range), "layers": "0,1,1,1,1,1,0,1",
           "parallelism": f"replicas x{args.gpus} (weak, no collective on the data path)",
           "l2": "no flush: each step streams ~60 GB of inputs, far above the 126 MB L2"}
    if args.workload in ("stack", "decode", "decode_fp8"):
        cfg["decode_launch"] = ("direct C-ABI calls, one per layer" if args.no_graph else
                                "the 8 layers' C-ABI calls captured once in a CUDA graph, replayed each step")
    if args.workload != "stack":
        cfg["l2"] = "inputs larger than L2" if args.workload != "swa" else "L2 flushed between steps (256 MB write)"
    return cfg


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["stack", "swa", "global", "decode", "chunked", "decode_fp8", "qkv"], default="stack")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the decode layers one call at a time")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    if args.workload in ("chunked", "decode_fp8", "qkv"):  # NEXT-row measurements: no host-buffer leg
        args.no_e2e = True
    if args.impl == "reference":
        run_reference(args)
        return

    dist, rank, world, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    import global_attention_partial_b200 as mimo
    mimo.load()
    peaks = measured_peaks()
    w = StackWorkload(args.workload)
    if not args.no_graph:
        w.capture_decode()
    stream = torch.cuda.current_stream()
    flush = None
    if args.workload == "swa":
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    for _ in range(max(args.warmup, 0)):
        w.step(stream)
    torch.cuda.synchronize()
    if mimo.mimo_attn_get_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    # ---- timed region (device-resident inputs)
    sampler = ClockSampler(local)
    sampler.start()
    events = {}
    barrier(dist, local)
    torch.cuda.synchronize()
    step_events = []
    for _ in range(args.steps):
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
    clocks = sampler.stop()
    ms_local = sum(a.elapsed_time(b) for a, b in step_events) / args.steps
    ms = max_over_ranks(dist, ms_local)

    kinds = {k: [a.elapsed_time(b) for a, b in v] for k, v in events.items()}
    pflops = w.prefill_flops() if w.do_prefill else 0.0
    dflops = w.decode_flops() if w.do_decode else 0.0
    cflops = w.chunk_flops() if w.do_chunked else 0.0
    qflops = w.qkv_flops() if w.do_qkv else 0.0
    step_flops = pflops + dflops + cflops + qflops
    value = job_value(world, step_flops, ms)

    parts = {}
    roofline = None
    if w.do_prefill:
        ms_prefill = (sum(sum(v) for k, v in kinds.items() if k.startswith("prefill")) / args.steps)
        parts["prefill"] = {"ms": ms_prefill, "tflops": pflops / (ms_prefill * 1e-3) / 1e12,
                            "frac_of_tensor_peak": pflops / (ms_prefill * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"]}
        for kind, lt in (("prefill_global", 0), ("prefill_swa", 1)):
            if kind not in kinds:
                continue
            specs = [L["spec"] for L in w.prefill_layers if L["spec"].layer_type == lt]
            per = statistics.mean(kinds[kind])
            f = prefill_flops(specs[0], w.pw.batch, w.pw.seq)
            byt = prefill_bytes(specs[0], w.pw.batch, w.pw.seq)
            parts[kind.replace("prefill_", "") + "_layer"] = {
                "ms_per_launch": per, "tflops": f / (per * 1e-3) / 1e12,
                "frac_of_tensor_peak": f / (per * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"],
                "gbs_compulsory": byt / (per * 1e-3) / 1e9,
                "frac_of_hbm_peak": byt / (per * 1e-3) / 1e9 / peaks["hbm_gbs"]}
        dom = "prefill_global" if "prefill_global" in kinds else "prefill_swa"
        lt = 0 if dom == "prefill_global" else 1
        spec = [L["spec"] for L in w.prefill_layers if L["spec"].layer_type == lt][0]
        per = statistics.mean(kinds[dom])
        if lt == 0:
            ach = prefill_flops(spec, w.pw.batch, w.pw.seq) / (per * 1e-3) / 1e12
            roofline = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops_sustained"],
                        "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops_sustained"],
                        "traffic": committed_traffic("prefill_ga_global", "prefill_ga.cu"),
                        "kernel": "prefill_ga_kernel (global layer, B4 S32768 causal)",
                        "peak_kind": f"bf16 dense, sustained, {peaks['source']}"}
        else:
            ach = prefill_bytes(spec, w.pw.batch, w.pw.seq) / (per * 1e-3) / 1e9
            roofline = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / peaks["hbm_gbs"],
                        "traffic": committed_traffic("prefill_swa_sliding", "prefill_swa.cu"),
                        "kernel": "prefill_swa_kernel (sliding layer)", "peak_kind": f"HBM copy, {peaks['source']}"}
    if w.do_chunked:
        for kind, lt in (("chunk_global", 0), ("chunk_swa", 1)):
            specs = [L["spec"] for L in w.chunk_layers if L["spec"].layer_type == lt]
            per = statistics.mean(kinds[kind])
            f = chunk_flops(specs[0], w.pw.batch, w.chunk_seq, w.chunk_past)
            parts[kind + "_layer"] = {"ms_per_launch": per, "tflops": f / (per * 1e-3) / 1e12,
                                      "frac_of_tensor_peak": f / (per * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"]}
        ach = parts["chunk_global_layer"]["tflops"]
        roofline = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                    "frac": ach / peaks["bf16_tflops_sustained"], "traffic": None,
                    "kernel": "prefill_ga_kernel (global layer, chunk of 4096 after 28672 cached, B4)",
                    "peak_kind": f"bf16 dense, sustained, {peaks['source']}"}
    if w.do_qkv:
        for kind, lt in (("qkv_global", 0), ("qkv_swa", 1)):
            spec = [L["spec"] for L in w.qkv_layers if L["spec"].layer_type == lt][0]
            per = statistics.mean(kinds[kind])
            f = qkv_flops(spec, w.pw.batch, w.pw.seq)
            parts[kind + "_layer"] = {"ms_per_launch": per, "tflops": f / (per * 1e-3) / 1e12,
                                      "frac_of_tensor_peak": f / (per * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"]}
        ach = parts["qkv_swa_layer"]["tflops"]
        roofline = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                    "frac": ach / peaks["bf16_tflops_sustained"], "traffic": None,
                    "kernel": "qkv_proj_kernel (sliding layer: 14848 features, B4 S32768, hidden 4096)",
                    "peak_kind": f"bf16 dense, sustained, {peaks['source']}"}
    if w.do_decode:
        per = statistics.mean(kinds["decode_stack"])
        byt = w.decode_bytes()
        parts["decode"] = {"ms_per_stack": per, "gbs": byt / (per * 1e-3) / 1e9,
                           "frac_of_hbm_peak": byt / (per * 1e-3) / 1e9 / peaks["hbm_gbs"],
                           "bytes_per_stack": byt,
                           "launch": "direct calls" if getattr(w, "decode_graph", None) is None else "CUDA graph"}
        if getattr(w, "decode_graph", None) is not None:
            # the same stack as 8 back-to-back direct calls, outside the timed region
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
                        "kernel": "decode_mma_kernel (8-layer stack%s)" % (", fp8 KV cache" if w.fp8 else ""),
                        "peak_kind": f"HBM copy, {peaks['source']}"}

    # ---- e2e through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        host = HostInputs(w)
        e2e_steps = max(1, min(args.steps, 3))
        host.step(stream)
        torch.cuda.synchronize()
        barrier(dist, local)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            host.step(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(dist, local)
        ms_e2e = max_over_ranks(dist, e0.elapsed_time(e1) / e2e_steps)
        e2e = {"value": job_value(world, step_flops, ms_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": host.h2d, "d2h_bytes_per_step": host.d2h, "ms_per_step": ms_e2e,
               "steps": e2e_steps}
        del host

    if mimo.mimo_attn_get_device_error() != 0:
        raise RuntimeError("device error word set during the timed region")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, t, desc = oracle_sample(args.cpu_seconds, kind=args.workload)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle", "sample": desc,
               "seconds": t}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None,
                "dtype": "e4m3 KV cache, f16 mma, fp32 accumulate" if w.fp8 else "bf16", "data": "synthetic", "config": workload_config(args),
                "roofline": roofline, "parts": parts, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": w.launches_per_step() * args.steps, "clocks": clocks,
                "peaks": peaks}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
