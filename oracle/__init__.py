"""fp64 CPU oracle for the MiMo-V2-Flash hybrid attention layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers. The CUDA library never imports, links or runs anything here, and
nothing here imports the CUDA library.

The arithmetic lives in ``mimo_oracle.c`` (plain C, double precision, plain
loops). This module compiles it with gcc when needed, loads it with ctypes
and marshals numpy arrays; the composition helpers below only chain the C
steps in the pages' order (rotate Q and K at their positions, then attend),
see "Add Xiaomi MiMo-V2" (huggingface/transformers PR 45144), section
"Additional useful info", and "feat(models): add Xiaomi MiMo v2
(mimo_v2_flash) text model support" (lablup/mlxcel issue 842), section
"Architecture, verified against upstream".
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mimo_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

GLOBAL = 0
SWA = 1


def build(force: bool = False) -> str:
    """Compile mimo_oracle.c into liboracle.so next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.oracle_rope.argtypes = [dp, dp, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_double, dp]
        lib.oracle_rope.restype = ctypes.c_int
        lib.oracle_prefill_rows.argtypes = [dp, i64p, ctypes.c_int64, dp, dp, ctypes.c_int64,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int64, ctypes.c_double, ctypes.c_int,
                                            ctypes.c_double, ctypes.c_double, dp]
        lib.oracle_prefill_rows.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [dp, ctypes.c_int, dp, dp, dp, dp, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_double, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_double, dp, ctypes.c_double, dp]
        lib.oracle_decode.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_softmax_scale(qk_dim: int) -> float:
    """1/sqrt(qk_dim): the pages name no scale; the standard one is the reading."""
    return 1.0 / math.sqrt(qk_dim)


def v_scale(hidden_size: int, num_q_heads: int, v_dim: int) -> float:
    """The V rescale factor sqrt(hidden / (Hq * v_dim)) (PR 45144, Additional useful info)."""
    return math.sqrt(hidden_size / (num_q_heads * v_dim))


def rope(x, rotary_dim: int, theta: float, pos) -> np.ndarray:
    """Partial RoPE of the rows of x ([n, dim]) at positions pos ([n])."""
    x = _f64(x)
    squeeze = x.ndim == 1
    if squeeze:
        x = x[None, :]
    n, dim = x.shape
    p = _f64(np.broadcast_to(np.asarray(pos, dtype=np.float64), (n,)))
    y = np.empty_like(x)
    rc = _load().oracle_rope(_ptr(x), _ptr(y), n, dim, int(rotary_dim), float(theta), _ptr(p))
    if rc != 0:
        raise ValueError("oracle_rope: bad rotary_dim")
    return y[0] if squeeze else y


def prefill_rows(q_rot, rows: Sequence[int], k_rot, v, layer_type: int, window: int,
                 softmax_scale: float, sink: Optional[float], vscale: float) -> np.ndarray:
    """Output rows of one (batch, query head): q_rot [n, Dqk] at indices rows,
    against rotated keys k_rot [S, Dqk] and values v [S, Dv]."""
    q_rot = _f64(q_rot)
    k_rot = _f64(k_rot)
    v = _f64(v)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    n = r.shape[0]
    seq, qk_dim = k_rot.shape
    v_dim = v.shape[1]
    out = np.empty((n, v_dim), dtype=np.float64)
    has_sink = sink is not None
    rc = _load().oracle_prefill_rows(
        _ptr(q_rot), r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n, _ptr(k_rot), _ptr(v),
        seq, qk_dim, v_dim, int(layer_type), int(window), float(softmax_scale), int(has_sink),
        float(sink) if has_sink else 0.0, float(vscale), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_prefill_rows: bad argument")
    return out


def decode(q, k_new, v_new, k_cache, v_cache, L: int, rotary_dim: int, theta: float,
           layer_type: int, window: int, softmax_scale: float, sinks, vscale: float):
    """One decode step of one (batch, KV head). q: [n_q, Dqk] unrotated query
    heads of the group; k_new [Dqk], v_new [Dv] unrotated; k_cache [cap, Dqk]
    (rotated keys), v_cache [cap, Dv]. Returns (out [n_q, Dv], k_cache', v_cache')
    with the new token written into its slot."""
    q = _f64(q)
    if q.ndim == 1:
        q = q[None, :]
    n_q, qk_dim = q.shape
    k_new = _f64(k_new)
    v_new = _f64(v_new)
    kc = np.array(k_cache, dtype=np.float64, copy=True, order="C")
    vc = np.array(v_cache, dtype=np.float64, copy=True, order="C")
    cap = kc.shape[0]
    v_dim = vc.shape[1]
    out = np.empty((n_q, v_dim), dtype=np.float64)
    s = None if sinks is None else _f64(sinks)
    rc = _load().oracle_decode(
        _ptr(q), n_q, _ptr(k_new), _ptr(v_new), _ptr(kc), _ptr(vc), cap, int(L), qk_dim, v_dim,
        int(rotary_dim), float(theta), int(layer_type), int(window), float(softmax_scale),
        None if s is None else _ptr(s), float(vscale), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_decode: bad argument")
    return out, kc, vc


def prefill_layer(q, k, v, *, layer_type: int, num_kv_heads: int, rotary_dim: int, theta: float,
                  window: int, sinks, hidden_size: int, softmax_scale: Optional[float] = None,
                  positions=None, rows=None, heads=None, batches=None):
    """Whole-layer prefill in the pages' order: rotate Q and K (partial RoPE at
    each token's position), then attend per (batch, query head) row.

    q [B, S, Hq, Dqk], k [B, S, Hkv, Dqk], v [B, S, Hkv, Dv] (any float dtype,
    converted to double). rows/heads/batches restrict the computed outputs
    (the result holds NaN elsewhere). Returns out [B, S, Hq, Dv] in float64.
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B, S, Hq, Dqk = q.shape
    Dv = v.shape[3]
    G = Hq // num_kv_heads
    scale = default_softmax_scale(Dqk) if softmax_scale is None else softmax_scale
    vs = v_scale(hidden_size, Hq, Dv)
    pos = np.arange(S, dtype=np.float64) if positions is None else _f64(positions)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = range(Hq) if heads is None else heads
    batches = range(B) if batches is None else batches
    out = np.full((B, S, Hq, Dv), np.nan, dtype=np.float64)
    for b in batches:
        k_rot = {}
        for h in heads:
            kv = h // G
            if kv not in k_rot:
                k_rot[kv] = rope(k[b, :, kv, :], rotary_dim, theta, pos)
            q_rot = rope(q[b, rows, h, :], rotary_dim, theta, pos[rows])
            sink = None if sinks is None else float(np.asarray(sinks)[h])
            out[b, rows, h, :] = prefill_rows(q_rot, rows, k_rot[kv], v[b, :, kv, :], layer_type,
                                              window, scale, sink, vs)
    return out


def prefill_cached_layer(q, k, v, k_cache, v_cache, past_lens, *, layer_type: int, num_kv_heads: int,
                         rotary_dim: int, theta: float, window: int, sinks, hidden_size: int,
                         softmax_scale: Optional[float] = None, rows=None, heads=None, batches=None):
    """Prefill of a chunk that continues a cache (the cache-aware prefill of the
    rotating cache: lablup/mlxcel issue 842, "Implementation plan"). Token t
    of batch b sits at position P_b + t, P_b = past_lens[b]. Its keys are the
    cached ones (already rotated: a global cache holds position p in slot p, a
    sliding ring holds the last `window` positions in slots p mod window) and
    the chunk's own keys, rotated at their positions, up to itself, with the
    layer's mask (causal; window on sliding layers).

    q [B, S, Hq, Dqk], k [B, S, Hkv, Dqk], v [B, S, Hkv, Dv] (unrotated);
    k_cache [B, cap, Hkv, Dqk], v_cache [B, cap, Hkv, Dv] (cap = window on a
    sliding layer). Returns (out [B, S, Hq, Dv], k_cache', v_cache') with the
    chunk's rotated keys and its values written into their slots, in token
    order (on a ring a later token takes the slot of an earlier one).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B, S, Hq, Dqk = q.shape
    Dv = v.shape[3]
    G = Hq // num_kv_heads
    kc = np.array(k_cache, dtype=np.float64, copy=True, order="C")
    vc = np.array(v_cache, dtype=np.float64, copy=True, order="C")
    scale = default_softmax_scale(Dqk) if softmax_scale is None else softmax_scale
    vs = v_scale(hidden_size, Hq, Dv)
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    heads = range(Hq) if heads is None else heads
    past = [int(x) for x in np.asarray(past_lens).reshape(-1)]
    out = np.full((B, S, Hq, Dv), np.nan, dtype=np.float64)
    for b in range(B):
        P = past[b]
        n = P + S
        pos_new = P + np.arange(S, dtype=np.float64)
        # keys and values over positions [0, P + S)
        K = np.zeros((n, num_kv_heads, Dqk))
        V = np.zeros((n, num_kv_heads, Dv))
        for p in range(P):
            if layer_type == GLOBAL:
                K[p], V[p] = kc[b, p], vc[b, p]
            elif p >= P - (window - 1):  # older positions are outside every query's window
                K[p], V[p] = kc[b, p % window], vc[b, p % window]
        for kv in range(num_kv_heads):
            K[P:, kv] = rope(k[b, :, kv, :], rotary_dim, theta, pos_new)
        V[P:] = _f64(v[b])
        if batches is None or b in batches:
            for h in heads:
                kv = h // G
                q_rot = rope(q[b, rows, h, :], rotary_dim, theta, pos_new[rows])
                sink = None if sinks is None else float(np.asarray(sinks)[h])
                out[b, rows, h, :] = prefill_rows(q_rot, P + rows, K[:, kv, :], V[:, kv, :], layer_type,
                                                  window, scale, sink, vs)
        for t in range(S):
            p = P + t
            slot = p if layer_type == GLOBAL else p % window
            kc[b, slot], vc[b, slot] = K[p], V[p]
    return out, kc, vc


# ------------------------------------------------------ fp8 (e4m3) KV cache
# The OCP 8-bit floating point format E4M3 ("OCP 8-bit Floating Point
# Specification", FP8 E4M3): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
# bits; exponent field 0 holds the subnormals m * 2^-9; S.1111.111 is NaN and
# there is no infinity, so the largest finite magnitude is 1.75 * 2^8 = 448.
# The cache stores code c for a value x as c = e4m3(x / scale) (round to
# nearest, ties to even mantissa, saturating at +-448) and reads scale *
# e4m3_value(c). A reading: the pages only mention "one quant" for this
# model, without a format or a scale granularity; per-tensor scales with
# saturation are the plainest choice.

def e4m3_value(code) -> np.ndarray:
    """Value of each E4M3 code (uint8 array-like), NaN for the two NaN codes."""
    c = np.asarray(code, dtype=np.int64)
    s = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.power(2.0, e - 7.0))
    nan = (e == 15) & (m == 7)
    return np.where(nan, np.nan, s * mag)


_E4M3_POS = e4m3_value(np.arange(0, 127))  # the 127 non-negative finite codes 0x00..0x7E, increasing


def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 code of each finite x (round to nearest, ties to the code
    with an even mantissa, |x| > 448 saturating to +-448)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 448.0)
    d = np.abs(a[..., None] - _E4M3_POS)  # distance to every non-negative code
    best = np.argmin(d, axis=-1)
    # ties: argmin takes the lower code; move to the upper one when it is
    # equally near and has the even mantissa
    upper = np.minimum(best + 1, 126)
    du = np.take_along_axis(d, upper[..., None], axis=-1)[..., 0]
    db = np.take_along_axis(d, best[..., None], axis=-1)[..., 0]
    pick_upper = (du == db) & (upper != best) & ((upper & 1) == 0)
    code = np.where(pick_upper, upper, best)
    return np.where(np.signbit(x), code | 0x80, code).astype(np.uint8)


def decode_fp8kv(q, k_new, v_new, k_codes, v_codes, L: int, rotary_dim: int, theta: float, layer_type: int,
                 window: int, softmax_scale: float, sinks, vscale: float, k_scale: float, v_scale: float):
    """One decode step of one (batch, KV head) over an E4M3 cache. q [n_q, Dqk],
    k_new [Dqk], v_new [Dv] unrotated; k_codes [cap, Dqk], v_codes [cap, Dv]
    uint8. The new token's rotated key and its value are quantized into their
    slot first (as the cache keeps them); the query then attends the cache's
    values (scale * code value) over its visible positions, exactly as
    decode() does for a bf16 cache. Returns (out [n_q, Dv], k_codes', v_codes')."""
    q = _f64(q)
    if q.ndim == 1:
        q = q[None, :]
    kc = np.array(k_codes, dtype=np.uint8, copy=True)
    vc = np.array(v_codes, dtype=np.uint8, copy=True)
    cap = kc.shape[0]
    if L < 1 or (layer_type == GLOBAL and L > cap) or (layer_type == SWA and cap != window):
        raise ValueError("decode_fp8kv: bad length or capacity")
    pos = float(L - 1)
    slot = (L - 1) % window if layer_type == SWA else L - 1
    kc[slot] = e4m3_encode(rope(_f64(k_new)[None, :], rotary_dim, theta, [pos])[0] / k_scale)
    vc[slot] = e4m3_encode(_f64(v_new) / v_scale)
    K = np.zeros((L, kc.shape[1]))
    V = np.zeros((L, vc.shape[1]))
    lo = max(0, L - window) if layer_type == SWA else 0
    for p in range(lo, L):
        sl = p % window if layer_type == SWA else p
        K[p] = k_scale * e4m3_value(kc[sl])
        V[p] = v_scale * e4m3_value(vc[sl])
    q_rot = rope(q, rotary_dim, theta, np.full(q.shape[0], pos))
    out = np.empty((q.shape[0], V.shape[1]))
    for r in range(q.shape[0]):
        s = None if sinks is None else float(np.asarray(sinks)[r])
        out[r] = prefill_rows(q_rot[r:r + 1], [L - 1], K, V, layer_type, window, softmax_scale, s, vscale)[0]
    return out, kc, vc


def qkv_project(x, w_qkv, positions, *, num_q_heads: int, num_kv_heads: int, qk_dim: int, v_dim: int,
                rotary_dim: int, theta: float):
    """The step before attention: the token's hidden state x ([T, hidden])
    times the stacked projection weight w_qkv ([Hq*Dqk + Hkv*Dqk + Hkv*Dv,
    hidden]: the rows of W_q, then W_k, then W_v, each in the [out, in]
    layout of a linear layer, no bias), split into query, key and value heads;
    queries and keys then get the layer's partial RoPE at the token's
    position, values are left as they are (PR 45144, "Additional useful
    info": partial RoPE, decoupled V head dim). Returns q [T, Hq, Dqk],
    k [T, Hkv, Dqk] (both rotated) and v [T, Hkv, Dv]."""
    x = _f64(x)
    w = _f64(w_qkv)
    T = x.shape[0]
    nq, nk, nv = num_q_heads * qk_dim, num_kv_heads * qk_dim, num_kv_heads * v_dim
    if w.shape != (nq + nk + nv, x.shape[1]):
        raise ValueError("qkv_project: weight shape")
    y = x @ w.T  # one product per (token, output feature)
    pos = np.asarray(positions, dtype=np.float64).reshape(T)
    q = y[:, :nq].reshape(T, num_q_heads, qk_dim)
    k = y[:, nq:nq + nk].reshape(T, num_kv_heads, qk_dim)
    v = y[:, nq + nk:].reshape(T, num_kv_heads, v_dim).copy()
    q_rot = rope(q.reshape(T * num_q_heads, qk_dim), rotary_dim, theta,
                 np.repeat(pos, num_q_heads)).reshape(T, num_q_heads, qk_dim)
    k_rot = rope(k.reshape(T * num_kv_heads, qk_dim), rotary_dim, theta,
                 np.repeat(pos, num_kv_heads)).reshape(T, num_kv_heads, qk_dim)
    return q_rot, k_rot, v


def cache_write(k_cache, v_cache, k, v, positions, *, layer_type: int, window: int):
    """Stores each token's (rotated) key and value in its cache slot, tokens
    in order, so a later token that maps to the same slot wins: slot = position
    in a global layer's linear cache, position mod window in a sliding
    layer's ring (issue 842, "Implementation plan": rotating cache).
    k_cache/v_cache [cap, Hkv, D]; k/v [T, Hkv, D]. Returns new arrays."""
    kc = _f64(k_cache).copy()
    vc = _f64(v_cache).copy()
    for t, p in enumerate(np.asarray(positions).reshape(-1)):
        slot = int(p) % window if layer_type == SWA else int(p)
        kc[slot] = k[t]
        vc[slot] = v[t]
    return kc, vc
