"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test ties one step of the oracle to a closed form, an invariant the pages
or the mathematics fix, or a library routine it must reduce to (torch SDPA in
float64, torch.softmax). The plausible mistakes each one catches are named in
its docstring. No GPU is used.

Pages: "Add Xiaomi MiMo-V2" (huggingface/transformers PR 45144), section
"Additional useful info"; "feat(models): add Xiaomi MiMo v2 (mimo_v2_flash)
text model support" (lablup/mlxcel issue 842), section "Architecture,
verified against upstream".
"""
import cmath
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

RNG = np.random.default_rng(1234)


def rnd(*shape):
    return RNG.standard_normal(shape)


# ---------------------------------------------------------------- RoPE pins

def test_rope_rotary_dim_zero_is_identity():
    """rotary_dim 0 leaves Q/K untouched (an invariant the layer's config fixes)."""
    x = rnd(7, 48)
    y = oracle.rope(x, 0, 1e4, np.arange(7) * 37.0)
    assert np.array_equal(x, y)


def test_rope_position_zero_is_identity():
    x = rnd(5, 192)
    y = oracle.rope(x, 64, 5e6, np.zeros(5))
    assert np.array_equal(x, y)


def test_rope_preserves_pair_norms():
    """A rotation keeps |(x_j, x_{j+r/2})| and leaves dims >= r alone; catches a
    scale error or a wrong partner index."""
    x = rnd(9, 192)
    pos = RNG.integers(0, 40000, 9).astype(np.float64)
    y = oracle.rope(x, 64, 1e4, pos)
    half = 32
    nx = x[:, :half] ** 2 + x[:, half:64] ** 2
    ny = y[:, :half] ** 2 + y[:, half:64] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-13, atol=1e-13)
    assert np.array_equal(x[:, 64:], y[:, 64:])
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)


@pytest.mark.parametrize("r,theta", [(64, 1e4), (16, 1e6), (64, 5e6), (2, 10.0)])
def test_rope_position_one_closed_form(r, theta):
    """At position 1, pair j turns by theta^(-2j/r): written as a complex product
    (a + i b) * exp(i * phi) with cmath. Catches a wrong sign, a wrong pairing
    (interleaved vs half-split) or a frequency denominator other than r."""
    dim = max(r, 8) + 6
    x = rnd(dim)
    y = oracle.rope(x, r, theta, 1.0)
    half = r // 2
    for j in range(half):
        z = complex(x[j], x[j + half]) * cmath.exp(1j * theta ** (-2.0 * j / r))
        assert abs(y[j] - z.real) < 1e-14 and abs(y[j + half] - z.imag) < 1e-14
    assert np.array_equal(y[r:], x[r:])


def test_rope_relative_position_property():
    """<R(p)q, R(s)k> depends only on p - s (shift all positions by c)."""
    q = rnd(192)
    k = rnd(192)
    for p, s, c in [(5, 2, 100), (3000, 17, 12345), (0, 0, 7)]:
        a = oracle.rope(q, 64, 1e4, p) @ oracle.rope(k, 64, 1e4, s)
        b = oracle.rope(q, 64, 1e4, p + c) @ oracle.rope(k, 64, 1e4, s + c)
        assert abs(a - b) < 1e-10


def test_rope_rejects_odd_or_oversized_rotary_dim():
    with pytest.raises(ValueError):
        oracle.rope(rnd(8), 3, 1e4, 1.0)
    with pytest.raises(ValueError):
        oracle.rope(rnd(8), 10, 1e4, 1.0)


# ------------------------------------------------------- attention pins

def _layer(q, k, v, **kw):
    return oracle.prefill_layer(q, k, v, **kw)


def _sdpa(q, k, v, mask=None, causal=False, scale=None):
    """torch SDPA in float64; q [B,S,Hq,D] layout converted to [B,H,S,D]."""
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3) for a in (q, k, v))
    o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, is_causal=causal, scale=scale,
                                       enable_gqa=True)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("B,S,Hq,Hkv,D,Dv", [(1, 37, 4, 1, 48, 32), (2, 64, 8, 2, 24, 40),
                                            (1, 1, 2, 2, 16, 8)])
def test_global_layer_matches_sdpa_causal(B, S, Hq, Hkv, D, Dv):
    """Global layer, rotary 0, V scale 1, no sink == torch SDPA(is_causal, GQA).
    Catches a mask off by one, a transposed operand, a wrong softmax scale
    (SDPA's default is 1/sqrt(D)) and a wrong KV-head mapping (SDPA's GQA
    repeats each KV head for consecutive query heads)."""
    q, k, v = rnd(B, S, Hq, D), rnd(B, S, Hkv, D), rnd(B, S, Hkv, Dv)
    out = _layer(q, k, v, layer_type=0, num_kv_heads=Hkv, rotary_dim=0, theta=1e4, window=0,
                 sinks=None, hidden_size=Hq * Dv)
    ref = _sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_rotated_global_layer_matches_sdpa_on_rotated_inputs():
    """With rotary on, the layer equals SDPA on pre-rotated q/k (RoPE is pinned
    above), so rotation happens at each token's own position."""
    B, S, Hq, Hkv, D, Dv = 1, 50, 4, 2, 48, 16
    q, k, v = rnd(B, S, Hq, D), rnd(B, S, Hkv, D), rnd(B, S, Hkv, Dv)
    pos = np.arange(S, dtype=np.float64)
    qr = np.stack([oracle.rope(q[0, :, h], 16, 1e6, pos) for h in range(Hq)], axis=1)[None]
    kr = np.stack([oracle.rope(k[0, :, h], 16, 1e6, pos) for h in range(Hkv)], axis=1)[None]
    out = _layer(q, k, v, layer_type=0, num_kv_heads=Hkv, rotary_dim=16, theta=1e6, window=0,
                 sinks=None, hidden_size=Hq * Dv)
    np.testing.assert_allclose(out, _sdpa(qr, kr, v, causal=True), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("S,W", [(64, 16), (33, 1), (20, 7), (5, 9)])
def test_swa_layer_without_sink_matches_sdpa_band_mask(S, W):
    """Sliding window, no sink == SDPA with the band mask 0 <= i-j < W (W keys
    including the query). Catches a window of W+1 or W-1 keys."""
    B, Hq, Hkv, D, Dv = 1, 4, 2, 48, 32
    q, k, v = rnd(B, S, Hq, D), rnd(B, S, Hkv, D), rnd(B, S, Hkv, Dv)
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    mask = (j <= i) & (i - j < W)
    out = _layer(q, k, v, layer_type=1, num_kv_heads=Hkv, rotary_dim=0, theta=1e4, window=W,
                 sinks=None, hidden_size=Hq * Dv)
    np.testing.assert_allclose(out, _sdpa(q, k, v, mask=mask), rtol=1e-11, atol=1e-12)


def test_window_at_least_seq_with_minus_inf_sink_equals_global():
    """Invariant: window >= seq_len and a -inf sink reduce SWA to global attention."""
    B, S, Hq, Hkv, D, Dv = 2, 40, 4, 2, 48, 32
    q, k, v = rnd(B, S, Hq, D), rnd(B, S, Hkv, D), rnd(B, S, Hkv, Dv)
    common = dict(num_kv_heads=Hkv, rotary_dim=16, theta=1e4, hidden_size=256)
    g = _layer(q, k, v, layer_type=0, window=0, sinks=None, **common)
    for W in (S, S + 5):
        s = _layer(q, k, v, layer_type=1, window=W, sinks=np.full(Hq, -np.inf), **common)
        np.testing.assert_allclose(s, g, rtol=1e-13, atol=1e-14)


def test_sink_matches_softmax_over_augmented_scores():
    """The sink joins the denominator only: softmax over [scores, sink] with
    the sink column dropped (torch.softmax in float64). Catches a sink that
    is scaled by the softmax scale, given a value, or left out."""
    S, D, Dv, W = 30, 16, 8, 6
    q, k, v = rnd(1, S, 1, D), rnd(1, S, 1, D), rnd(1, S, 1, Dv)
    sink = np.array([0.7])
    out = _layer(q, k, v, layer_type=1, num_kv_heads=1, rotary_dim=0, theta=1e4, window=W,
                 sinks=sink, hidden_size=Dv)
    tq, tk, tv = (torch.from_numpy(a[0, :, 0]) for a in (q, k, v))
    scores = tq @ tk.T / math.sqrt(D)
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    scores = scores.masked_fill(~((j <= i) & (i - j < W)), float("-inf"))
    aug = torch.cat([scores, torch.full((S, 1), 0.7, dtype=torch.float64)], dim=1)
    p = torch.softmax(aug, dim=1)[:, :S]
    np.testing.assert_allclose(out[0, :, 0], (p @ tv).numpy(), rtol=1e-12, atol=1e-13)


def test_minus_inf_sink_is_plain_softmax():
    S, D, Dv = 25, 48, 32
    q, k, v = rnd(1, S, 2, D), rnd(1, S, 1, D), rnd(1, S, 1, Dv)
    kw = dict(layer_type=1, num_kv_heads=1, rotary_dim=16, theta=1e4, window=8, hidden_size=64)
    a = _layer(q, k, v, sinks=np.full(2, -np.inf), **kw)
    b = _layer(q, k, v, sinks=None, **kw)
    np.testing.assert_array_equal(a, b)


def test_single_key_closed_form():
    """One KV position: o = beta * v without a sink, and
    o = beta * v * e^x / (e^x + e^s) with one, x = <q~, k~> / sqrt(D)."""
    D, Dv, Hq = 48, 32, 4
    q, k, v = rnd(1, 1, Hq, D), rnd(1, 1, 1, D), rnd(1, 1, 1, Dv)
    hidden = 1000
    beta = math.sqrt(hidden / (Hq * Dv))
    out = _layer(q, k, v, layer_type=0, num_kv_heads=1, rotary_dim=16, theta=1e4, window=0,
                 sinks=None, hidden_size=hidden)
    for h in range(Hq):
        np.testing.assert_allclose(out[0, 0, h], beta * v[0, 0, 0], rtol=1e-14)
    sinks = np.array([0.3, -2.0, 4.0, 0.0])
    out = _layer(q, k, v, layer_type=1, num_kv_heads=1, rotary_dim=16, theta=1e4, window=3,
                 sinks=sinks, hidden_size=hidden)
    for h in range(Hq):
        x = float(q[0, 0, h] @ k[0, 0, 0]) / math.sqrt(D)  # position 0: no rotation
        w = math.exp(x) / (math.exp(x) + math.exp(sinks[h]))
        np.testing.assert_allclose(out[0, 0, h], beta * w * v[0, 0, 0], rtol=1e-12)


def test_zero_query_closed_form():
    """q = 0 gives equal scores: o = beta * sum(v_visible) / (n + e^s)."""
    S, D, Dv, W = 12, 16, 4, 5
    q = np.zeros((1, S, 1, D))
    k, v = rnd(1, S, 1, D), rnd(1, S, 1, Dv)
    s = 1.3
    out = _layer(q, k, v, layer_type=1, num_kv_heads=1, rotary_dim=8, theta=1e4, window=W,
                 sinks=np.array([s]), hidden_size=4 * Dv)
    beta = 2.0
    for i in range(S):
        lo = max(0, i - W + 1)
        n = i - lo + 1
        ref = beta * v[0, lo:i + 1, 0].sum(axis=0) / (n + math.exp(s))
        np.testing.assert_allclose(out[0, i, 0], ref, rtol=1e-13, atol=1e-15)


def test_v_scale_multiplies_output():
    """hidden = Hq*Dv gives beta = 1; any other hidden scales the output by
    sqrt(hidden/(Hq*Dv)) (a multiplication, not a division)."""
    S, Hq, D, Dv = 20, 4, 48, 32
    q, k, v = rnd(1, S, Hq, D), rnd(1, S, 2, D), rnd(1, S, 2, Dv)
    kw = dict(layer_type=1, num_kv_heads=2, rotary_dim=16, theta=1e4, window=7,
              sinks=np.array([0.1, 0.2, -0.3, 1.0]))
    a = _layer(q, k, v, hidden_size=Hq * Dv, **kw)
    b = _layer(q, k, v, hidden_size=9 * Hq * Dv, **kw)
    np.testing.assert_allclose(b, 3.0 * a, rtol=1e-12, atol=1e-14)
    assert oracle.v_scale(4096, 64, 128) == pytest.approx(math.sqrt(0.5))
    assert oracle.v_scale(256, 4, 32) == pytest.approx(math.sqrt(2.0))


def test_gqa_equals_replicated_mha():
    """Replicating each KV head G times (contiguous grouping) and running MHA
    gives the GQA result; catches a strided (h % Hkv) head mapping."""
    S, Hq, Hkv, D, Dv = 24, 8, 2, 32, 16
    q, k, v = rnd(1, S, Hq, D), rnd(1, S, Hkv, D), rnd(1, S, Hkv, Dv)
    kw = dict(layer_type=1, rotary_dim=16, theta=1e4, window=9, sinks=rnd(Hq), hidden_size=512)
    a = _layer(q, k, v, num_kv_heads=Hkv, **kw)
    G = Hq // Hkv
    b = _layer(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), num_kv_heads=Hq, **kw)
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-15)


def test_positions_shift_leaves_output_unchanged():
    """Shifting every RoPE position by c changes nothing (relative property)."""
    S, Hq, D, Dv = 30, 2, 48, 8
    q, k, v = rnd(1, S, Hq, D), rnd(1, S, 1, D), rnd(1, S, 1, Dv)
    kw = dict(layer_type=0, num_kv_heads=1, rotary_dim=16, theta=1e4, window=0, sinks=None,
              hidden_size=64)
    a = _layer(q, k, v, **kw)
    b = _layer(q, k, v, positions=np.arange(S) + 4321.0, **kw)
    np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-10)


# ---------------------------------------------------------------- decode pins

def _rotated_cache(k, v, L, cap, layer_type, window, r, theta):
    """Cache holding positions 0..L-2 of k (rotated) / v, laid out per the
    cache rule: slot p (global) or p mod window (ring)."""
    kc = rnd(cap, k.shape[1])  # stale garbage in unused slots
    vc = rnd(cap, v.shape[1])
    for p in range(L - 1):
        slot = p % window if layer_type == 1 else p
        kc[slot] = oracle.rope(k[p], r, theta, p)
        vc[slot] = v[p]
    return kc, vc


@pytest.mark.parametrize("layer_type,L,W", [(0, 1, 0), (0, 37, 0), (1, 1, 8), (1, 5, 8),
                                           (1, 8, 8), (1, 9, 8), (1, 30, 8)])
def test_decode_equals_prefill_last_row(layer_type, L, W):
    """Decode of token L-1 equals row L-1 of prefill over L tokens. For the
    ring this pins the W-slot ring (new token + W-1 previous) to the W-key
    window of prefill."""
    Hq, D, Dv, r, theta = 4, 48, 32, 16, 1e4
    q, k, v = rnd(1, L, Hq, D), rnd(1, L, 1, D), rnd(1, L, 1, Dv)
    sinks = rnd(Hq) if layer_type == 1 else None
    pre = _layer(q, k, v, layer_type=layer_type, num_kv_heads=1, rotary_dim=r, theta=theta,
                 window=W, sinks=sinks, hidden_size=256)
    cap = W if layer_type == 1 else L + 3
    kc, vc = _rotated_cache(k[0, :, 0], v[0, :, 0], L, cap, layer_type, W, r, theta)
    out, kc2, vc2 = oracle.decode(q[0, L - 1], k[0, L - 1, 0], v[0, L - 1, 0], kc, vc, L, r, theta,
                                  layer_type, W, 1 / math.sqrt(D), sinks, oracle.v_scale(256, Hq, Dv))
    np.testing.assert_allclose(out, pre[0, L - 1], rtol=1e-12, atol=1e-13)
    slot = (L - 1) % W if layer_type == 1 else L - 1
    np.testing.assert_allclose(kc2[slot], oracle.rope(k[0, L - 1, 0], r, theta, L - 1), rtol=1e-15)
    assert np.array_equal(vc2[slot], v[0, L - 1, 0])
    others = [s for s in range(cap) if s != slot]
    assert np.array_equal(kc2[others], kc[others]) and np.array_equal(vc2[others], vc[others])


def test_decode_ring_slot_permutation_invariance():
    """Softmax is order-free: permuting the ring slots that hold the W-1 older
    positions leaves the output unchanged."""
    W, L, D, Dv = 16, 50, 48, 32
    q, kn, vn = rnd(2, D), rnd(D), rnd(Dv)
    kc, vc = rnd(W, D), rnd(W, Dv)
    args = (L, 16, 1e4, 1, W, 1 / math.sqrt(D), np.array([0.2, -1.0]), 0.5)
    a, _, _ = oracle.decode(q, kn, vn, kc, vc, *args)
    new_slot = (L - 1) % W
    others = [s for s in range(W) if s != new_slot]
    perm = list(others)
    RNG.shuffle(perm)
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[others] = kc[perm]
    vc2[others] = vc[perm]
    b, _, _ = oracle.decode(q, kn, vn, kc2, vc2, *args)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def test_decode_rejects_bad_lengths():
    D, Dv = 8, 4
    with pytest.raises(ValueError):
        oracle.decode(rnd(1, D), rnd(D), rnd(Dv), rnd(4, D), rnd(4, Dv), 5, 4, 1e4, 0, 0, 1.0, None, 1.0)
    with pytest.raises(ValueError):
        oracle.decode(rnd(1, D), rnd(D), rnd(Dv), rnd(4, D), rnd(4, Dv), 0, 4, 1e4, 0, 0, 1.0, None, 1.0)
    with pytest.raises(ValueError):  # ring capacity must equal the window
        oracle.decode(rnd(1, D), rnd(D), rnd(Dv), rnd(4, D), rnd(4, Dv), 3, 4, 1e4, 1, 5, 1.0, None, 1.0)


# --------------------------------------------------- prefill continuing a cache

def _chunk_layer(layer_type, W):
    return dict(layer_type=layer_type, num_kv_heads=2, rotary_dim=16, theta=1e4 if layer_type else 1e6,
                window=W, hidden_size=256)


@pytest.mark.parametrize("layer_type,W", [(0, 0), (1, 4), (1, 16)])
def test_cached_prefill_with_empty_cache_is_plain_prefill(layer_type, W):
    """With no past tokens the chunk is a whole sequence: prefill_layer's
    output, and the cache holds the rotated keys / values in their slots.
    Catches a position offset applied twice or a wrong slot."""
    B, S, Hq, D, Dv = 2, 11, 4, 48, 32
    q, k, v = rnd(B, S, Hq, D), rnd(B, S, 2, D), rnd(B, S, 2, Dv)
    sinks = rnd(Hq) if layer_type else None
    kw = _chunk_layer(layer_type, W)
    cap = S if layer_type == 0 else W
    out, kc, vc = oracle.prefill_cached_layer(q, k, v, np.zeros((B, cap, 2, D)), np.zeros((B, cap, 2, Dv)),
                                              [0, 0], sinks=sinks, **kw)
    ref = oracle.prefill_layer(q, k, v, sinks=sinks, **kw)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)
    for b in range(B):
        for p in range(S):
            if layer_type == 1 and p < S - W:
                continue  # overwritten by a later token of the ring
            slot = p if layer_type == 0 else p % W
            for kv in range(2):
                kr = oracle.rope(k[b, p, kv], 16, kw["theta"], [float(p)])
                np.testing.assert_allclose(kc[b, slot, kv], kr, rtol=0, atol=1e-14)
                assert np.array_equal(vc[b, slot, kv], v[b, p, kv])


@pytest.mark.parametrize("layer_type,W,S1,S2", [(0, 0, 7, 9), (0, 0, 1, 1), (1, 4, 6, 7), (1, 8, 3, 20),
                                                (1, 8, 20, 3), (1, 16, 5, 5)])
def test_two_chunks_equal_one_shot(layer_type, W, S1, S2):
    """Prefilling S1 tokens, then continuing with S2 from the resulting cache,
    gives the one-shot prefill's last S2 rows, for sliding layers also when a
    chunk is longer than the window (ring wrap). Ties the cached path to the
    plain prefill, which is pinned to SDPA; catches an off-by-one in the
    positions, the window or the ring slot."""
    B, Hq, D, Dv = 2, 4, 48, 32
    S = S1 + S2
    q, k, v = rnd(B, S, Hq, D), rnd(B, S, 2, D), rnd(B, S, 2, Dv)
    sinks = rnd(Hq) if layer_type else None
    kw = _chunk_layer(layer_type, W)
    cap = S if layer_type == 0 else W
    kc0, vc0 = np.zeros((B, cap, 2, D)), np.zeros((B, cap, 2, Dv))
    _, kc1, vc1 = oracle.prefill_cached_layer(q[:, :S1], k[:, :S1], v[:, :S1], kc0, vc0, [0, 0],
                                              sinks=sinks, **kw)
    out2, _, _ = oracle.prefill_cached_layer(q[:, S1:], k[:, S1:], v[:, S1:], kc1, vc1, [S1, S1],
                                             sinks=sinks, **kw)
    ref = oracle.prefill_layer(q, k, v, sinks=sinks, **kw)
    np.testing.assert_allclose(out2, ref[:, S1:], rtol=0, atol=1e-12)


@pytest.mark.parametrize("layer_type,W,P", [(0, 0, 0), (0, 0, 13), (1, 8, 3), (1, 8, 21)])
def test_one_token_chunk_equals_decode(layer_type, W, P):
    """A one-token chunk is a decode step: same output, same cache afterwards
    (oracle.decode counts the new token in L = P + 1)."""
    Hq, D, Dv = 4, 48, 32
    kw = _chunk_layer(layer_type, W)
    cap = 32 if layer_type == 0 else W
    kc, vc = rnd(1, cap, 2, D), rnd(1, cap, 2, Dv)
    q, k, v = rnd(1, 1, Hq, D), rnd(1, 1, 2, D), rnd(1, 1, 2, Dv)
    sinks = rnd(Hq) if layer_type else None
    out, kc2, vc2 = oracle.prefill_cached_layer(q, k, v, kc, vc, [P], sinks=sinks, **kw)
    for kv in range(2):
        hs = slice(2 * kv, 2 * kv + 2)
        o, kcd, vcd = oracle.decode(q[0, 0, hs], k[0, 0, kv], v[0, 0, kv], kc[0, :, kv], vc[0, :, kv], P + 1,
                                    16, kw["theta"], layer_type, W, 1 / math.sqrt(D),
                                    None if sinks is None else sinks[hs], oracle.v_scale(256, Hq, Dv))
        np.testing.assert_allclose(out[0, 0, hs], o, rtol=0, atol=1e-13)
        np.testing.assert_allclose(kc2[0, :, kv], kcd, rtol=0, atol=1e-14)
        np.testing.assert_allclose(vc2[0, :, kv], vcd, rtol=0, atol=0)


# ------------------------------------------------------------- fp8 KV cache

def test_e4m3_values_closed_forms():
    """Codes of the OCP E4M3 definition: largest finite 448 (0x7E), smallest
    normal 2^-6 (0x08), smallest subnormal 2^-9 (0x01), 1.0 (0x38), sign bit,
    and the two NaN codes. Catches a wrong bias or subnormal scale."""
    v = oracle.e4m3_value(np.arange(256))
    assert v[0x7E] == 448.0 and v[0x08] == 2.0 ** -6 and v[0x01] == 2.0 ** -9 and v[0x07] == 7 * 2.0 ** -9
    assert v[0x38] == 1.0 and v[0x39] == 1.125 and v[0xB8] == -1.0 and v[0x00] == 0.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF]) and np.isfinite(np.delete(v, [0x7F, 0xFF])).all()
    pos = v[:127]
    assert np.all(np.diff(pos) > 0)  # codes 0x00..0x7E increase


def test_e4m3_encode_round_trip_ties_and_saturation():
    """Every finite code round-trips; halfway values go to the even mantissa;
    magnitudes beyond 448 saturate; values between codes go to the nearer."""
    v = oracle.e4m3_value(np.arange(256))
    finite = [c for c in range(256) if not np.isnan(v[c])]
    assert np.array_equal(oracle.e4m3_encode(v[finite]), np.array(finite, dtype=np.uint8))
    assert list(oracle.e4m3_encode([1.0625, 1.1875, 1.9375, 2.0 ** -10, 3 * 2.0 ** -11])) == [0x38, 0x3A, 0x40, 0x00, 0x01]
    assert list(oracle.e4m3_encode([448.0, 465.0, 1e6, -1e6])) == [0x7E, 0x7E, 0x7E, 0xFE]
    # a value that rounds to zero keeps its sign, as an IEEE-style conversion does
    assert list(oracle.e4m3_encode([0.0, -0.0, -1e-9, 1e-9])) == [0x00, 0x80, 0x80, 0x00]
    x = RNG.uniform(-400, 400, 2000)
    got = oracle.e4m3_value(oracle.e4m3_encode(x))
    nearest = np.array([v[finite][np.argmin(np.abs(v[finite] - xi))] for xi in x])
    np.testing.assert_array_equal(np.abs(got - x), np.abs(nearest - x))


@pytest.mark.parametrize("layer_type,L,W", [(0, 1, 0), (0, 40, 0), (1, 3, 8), (1, 30, 8)])
def test_fp8_decode_equals_bf16_decode_on_representable_values(layer_type, L, W):
    """When every cached value and the new token's rotated key and value are
    exactly scale * (an E4M3 value), the fp8 path is the plain decode: same
    output, and the codes written decode to the values decode() stores."""
    Hq, D, Dv, r, theta = 2, 16, 8, 0, 1e4  # r = 0: the new key needs no rotation to stay representable
    ks, vs = 0.5, 2.0
    v = oracle.e4m3_value(np.arange(0, 0x7E))
    cap = W if layer_type == 1 else L + 2
    kc_codes = RNG.integers(0, 0x70, (cap, D)).astype(np.uint8)
    vc_codes = RNG.integers(0, 0x70, (cap, Dv)).astype(np.uint8)
    kn = ks * RNG.choice(v[:0x70], D) * RNG.choice([-1, 1], D)
    vn = vs * RNG.choice(v[:0x70], Dv) * RNG.choice([-1, 1], Dv)
    q = rnd(Hq, D)
    sinks = rnd(Hq) if layer_type == 1 else None
    args = (L, r, theta, layer_type, W, 1 / math.sqrt(D), sinks, 0.7)
    o8, kc2, vc2 = oracle.decode_fp8kv(q, kn, vn, kc_codes, vc_codes, *args, ks, vs)
    o16, kc16, vc16 = oracle.decode(q, kn, vn, ks * oracle.e4m3_value(kc_codes), vs * oracle.e4m3_value(vc_codes), *args)
    np.testing.assert_allclose(o8, o16, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(ks * oracle.e4m3_value(kc2), kc16)
    np.testing.assert_array_equal(vs * oracle.e4m3_value(vc2), vc16)


# ------------------------------------------------- QKV projection step pins

def test_qkv_project_brute_force_at_position_zero():
    """At position 0 RoPE is the identity, so every output is one dot product
    of the token's hidden state with one weight row, written out as a loop:
    query head h, dim d is row h*Dqk + d; key head j is row Hq*Dqk + j*Dqk + d;
    value head j is row (Hq + Hkv)*Dqk + j*Dv + d. Catches a transposed
    weight and the q/k/v blocks in the wrong order."""
    T, hidden, Hq, Hkv, Dqk, Dv = 3, 5, 2, 1, 4, 2
    x = rnd(T, hidden)
    w = rnd(Hq * Dqk + Hkv * Dqk + Hkv * Dv, hidden)
    q, k, v = oracle.qkv_project(x, w, np.zeros(T), num_q_heads=Hq, num_kv_heads=Hkv, qk_dim=Dqk, v_dim=Dv,
                                 rotary_dim=2, theta=1e4)

    def dot(t, row):
        return sum(x[t, i] * w[row, i] for i in range(hidden))

    for t in range(T):
        for h in range(Hq):
            for d in range(Dqk):
                assert abs(q[t, h, d] - dot(t, h * Dqk + d)) < 1e-12
        for j in range(Hkv):
            for d in range(Dqk):
                assert abs(k[t, j, d] - dot(t, Hq * Dqk + j * Dqk + d)) < 1e-12
            for d in range(Dv):
                assert abs(v[t, j, d] - dot(t, (Hq + Hkv) * Dqk + j * Dv + d)) < 1e-12


def test_qkv_project_rope_closed_form():
    """Selection weights (W_q = I, W_k = 2I, W_v = the first Dv rows of I)
    make the projections the hidden state itself, so the outputs at position
    p are the rotation written out: pair (j, j + r/2) of the first r dims
    turns by p * theta^(-2j/r); the rest and V pass through. Catches a wrong
    pairing, sign or frequency in the projection's RoPE, and a rotated V."""
    D, Dv, r, theta, p = 8, 4, 4, 100.0, 3.0
    x = rnd(1, D)
    w = np.concatenate([np.eye(D), 2 * np.eye(D), np.eye(D)[:Dv]])
    q, k, v = oracle.qkv_project(x, w, [p], num_q_heads=1, num_kv_heads=1, qk_dim=D, v_dim=Dv,
                                 rotary_dim=r, theta=theta)
    for j in range(r // 2):
        phi = p * theta ** (-2 * j / r)
        a, b = x[0, j], x[0, j + r // 2]
        z = complex(a, b) * cmath.exp(1j * phi)
        assert abs(q[0, 0, j] - z.real) < 1e-12 and abs(q[0, 0, j + r // 2] - z.imag) < 1e-12
        assert abs(k[0, 0, j] - 2 * z.real) < 1e-12 and abs(k[0, 0, j + r // 2] - 2 * z.imag) < 1e-12
    np.testing.assert_array_equal(q[0, 0, r:], x[0, r:])
    np.testing.assert_array_equal(v[0, 0], x[0, :Dv])


@pytest.mark.parametrize("layer_type", [0, 1])
def test_qkv_then_attention_without_rope_is_the_layer(layer_type):
    """Projection outputs are already rotated, so attention over them with
    rotary_dim 0 equals the layer (attention with RoPE) over the unrotated
    projections x W^T. Ties the projection's RoPE to the attention's own,
    independently pinned, and fixes how the two calls compose."""
    B, S, hidden, Hq, Hkv, Dqk, Dv, r, W = 1, 9, 6, 4, 2, 8, 4, 4, 3
    x = rnd(B * S, hidden)
    w = rnd(Hq * Dqk + Hkv * (Dqk + Dv), hidden)
    pos = np.arange(S, dtype=np.float64)
    q, k, v = oracle.qkv_project(x, w, pos, num_q_heads=Hq, num_kv_heads=Hkv, qk_dim=Dqk, v_dim=Dv,
                                 rotary_dim=r, theta=1e4)
    y = x @ w.T
    q0 = y[:, :Hq * Dqk].reshape(B, S, Hq, Dqk)
    k0 = y[:, Hq * Dqk:(Hq + Hkv) * Dqk].reshape(B, S, Hkv, Dqk)
    v0 = y[:, (Hq + Hkv) * Dqk:].reshape(B, S, Hkv, Dv)
    sinks = rnd(Hq) if layer_type == 1 else None
    kw = dict(layer_type=layer_type, num_kv_heads=Hkv, theta=1e4, window=W, sinks=sinks, hidden_size=64)
    want = oracle.prefill_layer(q0, k0, v0, rotary_dim=r, **kw)
    got = oracle.prefill_layer(q.reshape(B, S, Hq, Dqk), k.reshape(B, S, Hkv, Dqk), v.reshape(B, S, Hkv, Dv),
                               rotary_dim=0, **kw)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_cache_write_slots():
    """A global cache holds position p in slot p; a ring of W slots holds, in
    slot s, the latest token whose position is s mod W (later tokens
    overwrite earlier ones)."""
    T, W = 10, 4
    k = np.arange(T, dtype=np.float64).reshape(T, 1, 1) + 100
    v = -k
    kc, vc = oracle.cache_write(np.zeros((T, 1, 1)), np.zeros((T, 1, 1)), k, v, np.arange(T),
                                layer_type=0, window=W)
    assert list(kc[:, 0, 0]) == [100 + p for p in range(T)] and np.array_equal(vc, -kc)
    kc, vc = oracle.cache_write(np.zeros((W, 1, 1)), np.zeros((W, 1, 1)), k, v, np.arange(T),
                                layer_type=1, window=W)
    assert list(kc[:, 0, 0]) == [108, 109, 106, 107] and np.array_equal(vc, -kc)
