"""Seeded synthetic inputs for the MiMo-V2-Flash attention layer.

This module only draws random numbers and describes workload shapes; it holds
none of the layer's arithmetic. It is the one module that both the CUDA-path
callers and the oracle-side tests use, so both sides read the very same bits.

Values are N(0, 1), drawn by torch's seeded generator on the requested device
(Philox on CUDA, MT19937 on CPU) in float32 and then rounded to the element
type; each tensor has its own seed derived from (seed, tensor_id). KV lengths
for decode are uniform integers drawn on the CPU.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import torch

_MASK64 = (1 << 64) - 1


def _mix(seed: int, tensor_id: int) -> int:
    """splitmix64 finaliser over (seed, tensor_id) -> a 63-bit generator seed."""
    z = (seed * 0x9E3779B97F4A7C15 + tensor_id * 0xD1B54A32D192ED03 + 0x632BE59BD9B4E019) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    z ^= z >> 31
    return z & ((1 << 63) - 1)


def normal(shape, *, seed: int, tensor_id: int, dtype=torch.bfloat16, device="cpu", std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) tensor of `shape`, rounded to `dtype`, drawn on `device`."""
    g = torch.Generator(device=device)
    g.manual_seed(_mix(seed, tensor_id))
    x = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x if dtype == torch.float32 else x.to(dtype)


def uniform_int(n: int, lo: int, hi: int, *, seed: int, tensor_id: int) -> torch.Tensor:
    """n integers uniform in [lo, hi] (inclusive), int32, on the CPU."""
    g = torch.Generator(device="cpu")
    g.manual_seed(_mix(seed, tensor_id))
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64).to(torch.int32)


# tensor ids: layer l uses 16*l + role
ROLE_Q, ROLE_K, ROLE_V, ROLE_SINK, ROLE_KCACHE, ROLE_VCACHE, ROLE_KNEW, ROLE_VNEW, ROLE_LENS, ROLE_X, ROLE_WQKV = range(11)


def tensor_id(layer: int, role: int) -> int:
    return 16 * layer + role


@dataclass(frozen=True)
class LayerSpec:
    """Per-layer attention parameters (the config fields the pages name)."""
    layer_type: int          # 0 global, 1 sliding window (hybrid_layer_pattern entry)
    num_q_heads: int
    num_kv_heads: int
    qk_dim: int
    v_dim: int
    rotary_dim: int
    window: int              # sliding_window_size (SWA only)
    theta: float             # swa_rope_theta (SWA) or rope_theta (global)
    hidden_size: int
    has_sink: bool


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" or "decode"
    batch: int
    seq: int                  # prefill length; decode: cache capacity of global layers
    layers: Tuple[LayerSpec, ...]
    dtype: torch.dtype
    kv_len_range: Optional[Tuple[int, int]] = None
    pattern: Tuple[int, ...] = field(default_factory=tuple)


def mimo_layer(layer_type: int, *, hq=64, qk=192, dv=128, rot=64, window=128, hidden=4096,
               swa_kv=8, ga_kv=4, swa_theta=1e4, ga_theta=5e6) -> LayerSpec:
    """MiMo-V2-Flash-shaped layer: SWA layers get swa_theta, swa_kv heads and a
    sink; global layers get ga_theta and ga_kv heads, no sink."""
    if layer_type == 1:
        return LayerSpec(1, hq, swa_kv, qk, dv, rot, window, swa_theta, hidden, True)
    return LayerSpec(0, hq, ga_kv, qk, dv, rot, window, ga_theta, hidden, False)


HYBRID_PATTERN = (0, 1, 1, 1, 1, 1, 0, 1)

# The five synthetic workloads (shapes of the MiMo-V2-Flash attention layers).
TINY_PAIR = Workload(
    name="tiny SWA+global pair fp32 B1 S64 Hq4 Hkv2/1 qk48 v32 r16 W16",
    kind="prefill", batch=1, seq=64, dtype=torch.float32, pattern=(1, 0),
    layers=(LayerSpec(1, 4, 2, 48, 32, 16, 16, 1e4, 256, True),
            LayerSpec(0, 4, 1, 48, 32, 16, 16, 1e6, 256, False)))
SWA_PREFILL = Workload(
    name="SWA layer prefill bf16 B1 S4096 Hq64 Hkv8 qk192 v128 r64 W128",
    kind="prefill", batch=1, seq=4096, dtype=torch.bfloat16, pattern=(1,),
    layers=(mimo_layer(1),))
GLOBAL_PREFILL = Workload(
    name="global layer prefill bf16 B2 S8192 Hq64 Hkv4 qk192 v128 r64 causal",
    kind="prefill", batch=2, seq=8192, dtype=torch.bfloat16, pattern=(0,),
    layers=(mimo_layer(0),))
HYBRID_PREFILL = Workload(
    name="hybrid 8-layer stack prefill bf16 B4 S32768 pattern 0,1,1,1,1,1,0,1",
    kind="prefill", batch=4, seq=32768, dtype=torch.bfloat16, pattern=HYBRID_PATTERN,
    layers=tuple(mimo_layer(t) for t in HYBRID_PATTERN))
HYBRID_DECODE = Workload(
    name="hybrid 8-layer decode bf16 B64 L~U[1024,32768] pattern 0,1,1,1,1,1,0,1",
    kind="decode", batch=64, seq=32768, dtype=torch.bfloat16, pattern=HYBRID_PATTERN,
    kv_len_range=(1024, 32768), layers=tuple(mimo_layer(t) for t in HYBRID_PATTERN))

WORKLOADS: List[Workload] = [TINY_PAIR, SWA_PREFILL, GLOBAL_PREFILL, HYBRID_PREFILL, HYBRID_DECODE]


def prefill_inputs(spec: LayerSpec, batch: int, seq: int, *, seed: int, layer: int,
                   dtype=torch.bfloat16, device="cpu"):
    """(q, k, v, sinks) for one prefill layer; sinks is None without a sink."""
    q = normal((batch, seq, spec.num_q_heads, spec.qk_dim), seed=seed,
               tensor_id=tensor_id(layer, ROLE_Q), dtype=dtype, device=device)
    k = normal((batch, seq, spec.num_kv_heads, spec.qk_dim), seed=seed,
               tensor_id=tensor_id(layer, ROLE_K), dtype=dtype, device=device)
    v = normal((batch, seq, spec.num_kv_heads, spec.v_dim), seed=seed,
               tensor_id=tensor_id(layer, ROLE_V), dtype=dtype, device=device)
    sinks = None
    if spec.has_sink:
        sinks = normal((spec.num_q_heads,), seed=seed, tensor_id=tensor_id(layer, ROLE_SINK),
                       dtype=torch.float32, device=device)
    return q, k, v, sinks


def decode_inputs(spec: LayerSpec, batch: int, capacity: int, kv_lens: torch.Tensor, *, seed: int,
                  layer: int, dtype=torch.bfloat16, device="cpu"):
    """(q, k_new, v_new, k_cache, v_cache, sinks) for one decode layer.
    Cache entries are N(0,1) values taken as already-rotated keys."""
    cap = spec.window if spec.layer_type == 1 else capacity
    q = normal((batch, spec.num_q_heads, spec.qk_dim), seed=seed,
               tensor_id=tensor_id(layer, ROLE_Q), dtype=dtype, device=device)
    k_new = normal((batch, spec.num_kv_heads, spec.qk_dim), seed=seed,
                   tensor_id=tensor_id(layer, ROLE_KNEW), dtype=dtype, device=device)
    v_new = normal((batch, spec.num_kv_heads, spec.v_dim), seed=seed,
                   tensor_id=tensor_id(layer, ROLE_VNEW), dtype=dtype, device=device)
    k_cache = normal((batch, cap, spec.num_kv_heads, spec.qk_dim), seed=seed,
                     tensor_id=tensor_id(layer, ROLE_KCACHE), dtype=dtype, device=device)
    v_cache = normal((batch, cap, spec.num_kv_heads, spec.v_dim), seed=seed,
                     tensor_id=tensor_id(layer, ROLE_VCACHE), dtype=dtype, device=device)
    sinks = None
    if spec.has_sink:
        sinks = normal((spec.num_q_heads,), seed=seed, tensor_id=tensor_id(layer, ROLE_SINK),
                       dtype=torch.float32, device=device)
    return q, k_new, v_new, k_cache, v_cache, sinks


def cached_prefill_inputs(spec: LayerSpec, batch: int, seq: int, capacity: int, *, seed: int, layer: int,
                          dtype=torch.bfloat16, device="cpu"):
    """(q, k, v, k_cache, v_cache, sinks) for a chunk of `seq` tokens that
    continues a cache: the chunk as prefill_inputs draws it, and caches of
    N(0,1) values taken as already-rotated keys (a ring of `window` slots on a
    sliding layer)."""
    q, k, v, sinks = prefill_inputs(spec, batch, seq, seed=seed, layer=layer, dtype=dtype, device=device)
    cap = spec.window if spec.layer_type == 1 else capacity
    k_cache = normal((batch, cap, spec.num_kv_heads, spec.qk_dim), seed=seed,
                     tensor_id=tensor_id(layer, ROLE_KCACHE), dtype=dtype, device=device)
    v_cache = normal((batch, cap, spec.num_kv_heads, spec.v_dim), seed=seed,
                     tensor_id=tensor_id(layer, ROLE_VCACHE), dtype=dtype, device=device)
    return q, k, v, k_cache, v_cache, sinks


def decode_kv_lens(batch: int, lo: int, hi: int, *, seed: int) -> torch.Tensor:
    """KV lengths (counting the new token) uniform in [lo, hi], int32 on the CPU."""
    return uniform_int(batch, lo, hi, seed=seed, tensor_id=tensor_id(255, ROLE_LENS))


def projection_inputs(spec: LayerSpec, batch: int, seq: int, *, seed: int, layer: int, device="cpu"):
    """(x, w_qkv) for the QKV projection of one layer: hidden states x
    [batch, seq, hidden] N(0,1) and the stacked weight [Hq*Dqk + Hkv*(Dqk+Dv),
    hidden] N(0, 1/hidden) (the usual fan-in initialisation scale, so the
    projections come out near N(0,1)), both bf16."""
    x = normal((batch, seq, spec.hidden_size), seed=seed, tensor_id=tensor_id(layer, ROLE_X), device=device)
    n = spec.num_q_heads * spec.qk_dim + spec.num_kv_heads * (spec.qk_dim + spec.v_dim)
    w = normal((n, spec.hidden_size), seed=seed, tensor_id=tensor_id(layer, ROLE_WQKV), device=device,
               std=spec.hidden_size ** -0.5)
    return x, w
