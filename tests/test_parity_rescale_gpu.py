"""GPU parity on inputs whose softmax maximum jumps, so the lazy rescaling runs.

With N(0, 1) inputs a row's maximum score is settled by its first key tile,
and the kernels' rescaling paths would go untested:

- the global prefill softmax moves its reference maximum, and rescales O,
  only when a key tile's maximum exceeds it by more than 2^8;
- the decode kernel does the same per 64-key tile;
- the split-KV combine merges partial results whose maxima differ by many
  orders of magnitude.

Construction. The last dimension (191, outside the rotated block) of every
query holds 1 and of every key 0, except for "spike" keys, which hold only
that dimension. A spike key's score is then the same for every query and
far above the others:

- a block of 400 keys [1900, 2300) scores 124/sqrt(192) ~ 8.95 nats;
- one key at 3500 scores 207/sqrt(192) ~ 14.94 nats.

Each jump exceeds the threshold: from a first-tile maximum of ~3.7 to 12.9
in log2 units, then from 12.9 to 21.6. The masses on either side of each
jump are of the same order, so a wrong correction factor moves the output by
tens of percent:

- first jump: ~2000 ordinary keys, ~e^8 in all, against e^8.95 per spike key;
- second jump: 400 x e^8.95 against e^14.94.

The split-KV boundary at key 2048 falls inside the block. The oracle is the
plain fp64 definition, which knows nothing of the threshold.
"""
import math

import numpy as np
import pytest
import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic
import oracle
from tests.parity_util import compare, f64, lib_layer, oracle_prefill

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
DIM = 191                  # last QK dim: not rotated (rotary dims are 0 .. 63)
BLOCK = (1900, 2300)       # spike block, score 124 / sqrt(192)
BLOCK_VALUE = 124.0        # exact in bf16
PEAK = 3500                # single spike, score 207 / sqrt(192)
PEAK_VALUE = 207.0         # exact in bf16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mimo.load()
    mimo.mimo_attn_get_device_error()  # clear


def _plant(q, keys, key_axis):
    """Sets dim DIM of every query to 1 and of every key to 0, then writes
    the spike keys (only dim DIM nonzero). keys: tensor with positions on
    `key_axis` (1 for [B, S, H, D] inputs and caches)."""
    q[..., DIM] = 1.0
    keys[..., DIM] = 0.0
    idx = [slice(None)] * keys.dim()
    idx[key_axis] = slice(*BLOCK)
    keys[tuple(idx)] = 0.0
    keys[tuple(idx[:-1] + [DIM])] = BLOCK_VALUE
    idx[key_axis] = PEAK
    keys[tuple(idx)] = 0.0
    keys[tuple(idx[:-1] + [DIM])] = PEAK_VALUE


def test_spike_scores_jump_past_the_threshold():
    """The construction's claims, checked on the numbers themselves."""
    s1 = BLOCK_VALUE / math.sqrt(192)
    s2 = PEAK_VALUE / math.sqrt(192)
    log2e = 1 / math.log(2)
    first_tile_max = 2.6 * log2e  # ~ max of 128 N(0, 1) scores, log2 units
    assert s1 * log2e - first_tile_max > 8
    assert (s2 - s1) * log2e > 8
    assert 0.1 < (BLOCK[1] - BLOCK[0]) * math.exp(s1) / math.exp(s2) < 10
    assert 0.1 < math.exp(s1) / (BLOCK[0] * math.exp(0.5)) < 10


@pytest.mark.parametrize("layer_type", [0, 1])
def test_prefill_with_spike_keys(layer_type):
    """Global layers: the lazy rescale of the online softmax. Sliding layers:
    scores ~15 nats above the rest inside the window, beside the sink."""
    spec = synthetic.mimo_layer(layer_type)
    B, S = 1, 4096 + 37
    q, k, v, sinks = synthetic.prefill_inputs(spec, B, S, seed=41, layer=layer_type, dtype=BF, device="cuda")
    _plant(q, k, key_axis=1)
    sinks = sinks if layer_type == 1 else None
    out = mimo.prefill(lib_layer(spec, sinks), q, k, v)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    rng = np.random.default_rng(7)
    fixed = {0, 127, 128, 1899, 1900, 1901, 1950, 2047, 2048, 2299, 2300, 2301, 2427, 2428,
             3499, 3500, 3501, 3627, 3628, 4000, S - 1}
    rows = sorted(fixed | set(rng.integers(1900, S, 16).tolist()))
    heads = (0, 1, 17, 30, 47, 63)
    ref = oracle_prefill(spec, q, k, v, sinks, {(0, h): rows for h in heads})
    gpu, want = [], []
    for (b, h), (rr, o) in ref.items():
        gpu.append(f64(out[b, rr, h, :]))
        want.append(o)
    c = compare(np.concatenate(gpu), np.concatenate(want))
    assert c.ok(BF), f"max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e} over {c.n}"


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_with_spike_keys(layer_type):
    """Decode over caches holding the spikes: the per-tile lazy rescale and,
    on global layers, a combine of splits whose maxima differ by ~10 nats
    (the block straddles the 2048-key split boundary). In sequence 1 the new
    token is the spike."""
    spec = synthetic.mimo_layer(layer_type)
    lens = [2000, 2100, 2300, 2301, 3400, 3501, 3700, 4100] if layer_type == 0 else [2000, 2301, 3502, 3600]
    B = len(lens)
    cap = 4100
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, sinks = synthetic.decode_inputs(spec, B, cap, kv_lens, seed=43, layer=layer_type,
                                                       dtype=BF, device="cuda")
    sinks = sinks if layer_type == 1 else None
    if layer_type == 0:
        _plant(q, kc, key_axis=1)
    else:
        # ring of W slots: slot p % W holds position p; spike the slots of the
        # positions in the window of each sequence's new token
        W = spec.window
        q[..., DIM] = 1.0
        kc[..., DIM] = 0.0
        for b, L in enumerate(lens):
            for p in range(max(0, L - W), L - 1):
                if BLOCK[0] <= p < BLOCK[1] or p == PEAK:
                    kc[b, p % W] = 0.0
                    kc[b, p % W, :, DIM] = PEAK_VALUE if p == PEAK else BLOCK_VALUE
    kn[..., DIM] = 0.0
    # one sequence whose new token is itself a spike (its key is rotated and
    # written by the kernel before use)
    kn[1] = 0.0
    kn[1, :, DIM] = PEAK_VALUE
    kc0, vc0 = kc.clone(), vc.clone()
    out = mimo.decode(lib_layer(spec, sinks), q, kn, vn, kv_lens.cuda(), kc, vc)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    G = spec.num_q_heads // spec.num_kv_heads
    vs = oracle.v_scale(spec.hidden_size, spec.num_q_heads, spec.v_dim)
    gpu, want = [], []
    for b, L in enumerate(lens):
        for kv in range(spec.num_kv_heads):
            hs = slice(kv * G, (kv + 1) * G)
            o, _, _ = oracle.decode(f64(q[b, hs]), f64(kn[b, kv]), f64(vn[b, kv]), f64(kc0[b, :, kv]),
                                    f64(vc0[b, :, kv]), L, spec.rotary_dim, spec.theta, spec.layer_type,
                                    spec.window, 1 / math.sqrt(spec.qk_dim),
                                    None if sinks is None else f64(sinks[hs]), vs)
            gpu.append(f64(out[b, hs]))
            want.append(o)
    c = compare(np.concatenate(gpu), np.concatenate(want))
    assert c.ok(BF), f"max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e} over {c.n}"


SINKS = (-math.inf, -30.0, 0.0, 12.0, 30.0)


def _extreme_sinks(spec):
    return torch.tensor([SINKS[h % len(SINKS)] for h in range(spec.num_q_heads)], dtype=torch.float32,
                        device="cuda")


def test_swa_prefill_extreme_sinks():
    """Sink logits of -inf (no sink), -30, 0, +12 and +30 nats: the sink may
    take all but ~e^-25 of the mass, or none. Every output of a ragged
    sequence, all heads."""
    spec = synthetic.mimo_layer(1)
    B, S = 1, 700
    q, k, v, _ = synthetic.prefill_inputs(spec, B, S, seed=47, layer=1, dtype=BF, device="cuda")
    sinks = _extreme_sinks(spec)
    out = mimo.prefill(lib_layer(spec, sinks), q, k, v)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    ref = oracle_prefill(spec, q, k, v, sinks, {(0, h): list(range(S)) for h in range(spec.num_q_heads)})
    gpu, want = [], []
    for (b, h), (rr, o) in ref.items():
        gpu.append(f64(out[b, rr, h, :]))
        want.append(o)
    c = compare(np.concatenate(gpu), np.concatenate(want))
    assert c.ok(BF), f"max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e} over {c.n}"


def test_swa_decode_extreme_sinks():
    spec = synthetic.mimo_layer(1)
    lens = [1, 2, 64, 65, 128, 129, 700]
    B, cap = len(lens), spec.window
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, _ = synthetic.decode_inputs(spec, B, cap, kv_lens, seed=53, layer=1, dtype=BF,
                                                   device="cuda")
    sinks = _extreme_sinks(spec)
    kc0, vc0 = kc.clone(), vc.clone()
    out = mimo.decode(lib_layer(spec, sinks), q, kn, vn, kv_lens.cuda(), kc, vc)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    G = spec.num_q_heads // spec.num_kv_heads
    vs = oracle.v_scale(spec.hidden_size, spec.num_q_heads, spec.v_dim)
    gpu, want = [], []
    for b, L in enumerate(lens):
        for kv in range(spec.num_kv_heads):
            hs = slice(kv * G, (kv + 1) * G)
            o, _, _ = oracle.decode(f64(q[b, hs]), f64(kn[b, kv]), f64(vn[b, kv]), f64(kc0[b, :, kv]),
                                    f64(vc0[b, :, kv]), L, spec.rotary_dim, spec.theta, spec.layer_type,
                                    spec.window, 1 / math.sqrt(spec.qk_dim), f64(sinks[hs]), vs)
            gpu.append(f64(out[b, hs]))
            want.append(o)
    c = compare(np.concatenate(gpu), np.concatenate(want))
    assert c.ok(BF), f"max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e} over {c.n}"


def _compare_rows(spec, out, q, k, v, sinks, rows, heads):
    ref = oracle_prefill(spec, q, k, v, sinks, {(0, h): rows for h in heads})
    gpu, want = [], []
    for (b, h), (rr, o) in ref.items():
        gpu.append(f64(out[b, rr, h, :]))
        want.append(o)
    return compare(np.concatenate(gpu), np.concatenate(want))


def test_single_tile_prefill_with_spike_keys():
    """An odd query-group size (12 query heads over 4 KV heads) takes the
    single-tile tensor-core kernel, whose online softmax has the same lazy
    rescale."""
    spec = synthetic.mimo_layer(0, hq=12, ga_kv=4)
    B, S = 1, 4096 + 37
    q, k, v, _ = synthetic.prefill_inputs(spec, B, S, seed=59, layer=0, dtype=BF, device="cuda")
    _plant(q, k, key_axis=1)
    out = mimo.prefill(lib_layer(spec, None), q, k, v)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    rows = sorted({0, 128, 1899, 1900, 1901, 2047, 2048, 2299, 2300, 3499, 3500, 3501, 4000, S - 1})
    c = _compare_rows(spec, out, q, k, v, None, rows, (0, 2, 3, 5, 11))
    assert c.ok(BF), f"max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e} over {c.n}"


def test_decode_fp8_with_spike_keys():
    """The fp8 (E4M3) decode over the planted global-layer cache. The keys are
    stored at k_scale 1/2 so the spikes stay representable (124 and 207 become
    the codes 256 and 416, i.e. 128 and 208)."""
    from tests.test_parity_fp8_gpu import _encode_on_device
    spec = synthetic.mimo_layer(0)
    k_scale, v_scale = 0.5, 1.0 / 32
    lens = [2000, 2100, 2301, 3501, 3700, 4100]
    B, cap = len(lens), 4100
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, _ = synthetic.decode_inputs(spec, B, cap, kv_lens, seed=61, layer=0, dtype=BF, device="cuda")
    _plant(q, kc, key_axis=1)
    kn[..., DIM] = 0.0
    kn[1] = 0.0
    kn[1, :, DIM] = PEAK_VALUE
    kc8 = torch.stack([_encode_on_device(kc[b], k_scale) for b in range(B)])
    vc8 = torch.stack([_encode_on_device(vc[b], v_scale) for b in range(B)])
    kc0, vc0 = kc8.clone(), vc8.clone()
    out = mimo.decode_fp8kv(lib_layer(spec, None), q, kn, vn, kv_lens.cuda(), kc8, vc8, k_scale, v_scale)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    G = spec.num_q_heads // spec.num_kv_heads
    vs = oracle.v_scale(spec.hidden_size, spec.num_q_heads, spec.v_dim)
    gpu, want = [], []
    for b, L in enumerate(lens):
        for kv in range(spec.num_kv_heads):
            hs = slice(kv * G, (kv + 1) * G)
            o, _, _ = oracle.decode_fp8kv(f64(q[b, hs]), f64(kn[b, kv]), f64(vn[b, kv]), kc0[b, :, kv].cpu().numpy(),
                                          vc0[b, :, kv].cpu().numpy(), L, spec.rotary_dim, spec.theta, 0,
                                          spec.window, 1 / math.sqrt(spec.qk_dim), None, vs, k_scale, v_scale)
            gpu.append(f64(out[b, hs]))
            want.append(o)
    c = compare(np.concatenate(gpu), np.concatenate(want))
    assert c.ok(BF), f"max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e} over {c.n}"


def test_prefill_continuing_cache_with_spike_keys():
    """A global-layer chunk after a cache that holds the spike block, with
    the single spike inside the chunk: the kernel reads the cache with a key
    offset per sequence."""
    spec = synthetic.mimo_layer(0)
    past, S = [2500, 1950], 1100
    B = len(past)
    cap = max(past) + S + 5
    q, k, v, kc, vc, _ = synthetic.cached_prefill_inputs(spec, B, S, cap, seed=67, layer=0, dtype=BF, device="cuda")
    q[..., DIM] = 1.0
    k[..., DIM] = 0.0
    kc[..., DIM] = 0.0
    for b, P in enumerate(past):
        for p0 in range(*BLOCK):           # block positions: in the cache or in the chunk
            if p0 < P:
                kc[b, p0] = 0.0
                kc[b, p0, :, DIM] = BLOCK_VALUE
            elif p0 - P < S:
                k[b, p0 - P] = 0.0
                k[b, p0 - P, :, DIM] = BLOCK_VALUE
        if 0 <= PEAK - P < S:
            k[b, PEAK - P] = 0.0
            k[b, PEAK - P, :, DIM] = PEAK_VALUE
    kc0, vc0 = kc.clone(), vc.clone()
    out = mimo.prefill_cached(lib_layer(spec, None), q, k, v, torch.tensor(past, dtype=torch.int32, device="cuda"),
                              kc, vc, max_past_len=max(past))
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    heads = [0, 1, 30, 63]
    ref, _, _ = oracle.prefill_cached_layer(
        f64(q), f64(k), f64(v), f64(kc0), f64(vc0), past, layer_type=0, num_kv_heads=spec.num_kv_heads,
        rotary_dim=spec.rotary_dim, theta=spec.theta, window=spec.window, sinks=None,
        hidden_size=spec.hidden_size, heads=heads)
    c = compare(f64(out)[:, :, heads].reshape(-1), ref[:, :, heads].reshape(-1))
    assert c.ok(BF), f"max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e} over {c.n}"
