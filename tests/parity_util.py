"""Shared helpers of the GPU parity tests: run the library through its C ABI
binding, run the fp64 oracle on the same input bits, compare."""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic
import oracle

BF16_MAX_ABS = 2e-2   # tolerances of the layer's parity bar (bf16 inputs)
BF16_MEAN_ABS = 2e-3
FP32_MAX_ABS = 1e-4   # fp32 inputs


@dataclass
class Cmp:
    max_abs: float
    mean_abs: float
    n: int

    def ok(self, dtype) -> bool:
        if dtype == torch.float32:
            return self.max_abs <= FP32_MAX_ABS
        return self.max_abs <= BF16_MAX_ABS and self.mean_abs <= BF16_MEAN_ABS


def compare(gpu: np.ndarray, ref: np.ndarray) -> Cmp:
    d = np.abs(gpu.astype(np.float64) - ref)
    assert np.all(np.isfinite(gpu)), "non-finite GPU output"
    return Cmp(float(d.max()), float(d.mean()), int(d.size))


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def lib_layer(spec: synthetic.LayerSpec, sinks: Optional[torch.Tensor], window=None, rotary=None):
    return mimo.make_layer(spec.layer_type, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim, spec.v_dim,
                           spec.rotary_dim if rotary is None else rotary,
                           spec.window if window is None else window, spec.theta, spec.hidden_size,
                           sinks if spec.layer_type == 1 else None)


def oracle_threads() -> int:
    """Host threads for the oracle: every core this process may use."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def oracle_prefill(spec, q, k, v, sinks, rows_by_b_h, positions=None, window=None, rotary=None):
    """Oracle outputs {(b, h): (rows, out[len(rows), Dv])} for the requested rows.

    The (batch, KV head) key rotations and the (batch, query head) row sets
    run on a thread pool: the oracle's C routines release the GIL, so each
    call runs on its own core. The calls and their arguments are the same as
    a plain loop's."""
    Hq, G = spec.num_q_heads, spec.num_q_heads // spec.num_kv_heads
    S = q.shape[1]
    W = spec.window if window is None else window
    r = spec.rotary_dim if rotary is None else rotary
    pos = np.arange(S, dtype=np.float64) if positions is None else f64(positions)
    scale = 1.0 / math.sqrt(spec.qk_dim)
    vs = oracle.v_scale(spec.hidden_size, Hq, spec.v_dim)
    sink_np = None if sinks is None else f64(sinks)
    pairs = sorted({(b, h // G) for (b, h) in rows_by_b_h})
    kv_host = {(b, kv): (f64(k[b, :, kv, :]), f64(v[b, :, kv, :])) for (b, kv) in pairs}
    q_host = {(b, h): f64(q[b, np.asarray(rows, dtype=np.int64), h, :]) for (b, h), rows in rows_by_b_h.items()}

    def rotate(key):
        kk, vv = kv_host[key]
        return key, (oracle.rope(kk, r, spec.theta, pos), vv)

    def attend(item):
        (b, h), rows = item
        kr, vv = k_rot[(b, h // G)]
        rows = np.asarray(rows, dtype=np.int64)
        qr = oracle.rope(q_host[(b, h)], r, spec.theta, pos[rows])
        sink = None if (sink_np is None or spec.layer_type == 0) else float(sink_np[h])
        return (b, h), (rows, oracle.prefill_rows(qr, rows, kr, vv, spec.layer_type, W, scale, sink, vs))

    with ThreadPoolExecutor(max_workers=oracle_threads()) as ex:
        k_rot = dict(ex.map(rotate, pairs))
        return dict(ex.map(attend, list(rows_by_b_h.items())))


def check_prefill(spec, B, S, dtype, *, seed=0, layer_idx=0, rows="all", heads=None, batches=None,
                  positions=None, window=None, rotary=None, n_random_rows=24, out_offset_elems=0):
    """Runs the library prefill and compares it with the oracle. Returns Cmp.
    out_offset_elems > 0 places the output that many elements past a 256-byte
    aligned allocation (8 bf16 = 16 bytes: 16- but not 32-byte aligned)."""
    q, k, v, sinks = synthetic.prefill_inputs(spec, B, S, seed=seed, layer=layer_idx, dtype=dtype, device="cuda")
    if spec.layer_type == 0:
        sinks = None
    lay = lib_layer(spec, sinks, window, rotary)
    out = None
    if out_offset_elems:
        n = B * S * spec.num_q_heads * spec.v_dim
        base = torch.empty(n + out_offset_elems, dtype=dtype, device="cuda")
        out = base[out_offset_elems:].view(B, S, spec.num_q_heads, spec.v_dim)
    out = mimo.prefill(lay, q, k, v, positions=positions, out=out)
    torch.cuda.synchronize()
    heads = range(spec.num_q_heads) if heads is None else heads
    batches = range(B) if batches is None else batches
    W = spec.window if window is None else window
    if rows == "all":
        row_list = list(range(S))
    else:
        rng = np.random.default_rng(seed + 17)
        fixed = {0, 1, W - 2, W - 1, W, W + 1, 126, 127, 128, 129, S // 2 - 1, S // 2, S - 2, S - 1}
        row_list = sorted({r for r in fixed if 0 <= r < S} | set(rng.integers(0, S, n_random_rows).tolist()))
    want = {(b, h): row_list for b in batches for h in heads}
    ref = oracle_prefill(spec, q, k, v, sinks, want, positions=positions, window=window, rotary=rotary)
    gpu = out.detach().cpu()
    diffs, refs = [], []
    for (b, h), (rr, o) in ref.items():
        diffs.append(f64(gpu[b, rr, h, :]))
        refs.append(o)
    return compare(np.concatenate(diffs), np.concatenate(refs)), out, (q, k, v, sinks)
