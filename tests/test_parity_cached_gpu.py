"""GPU parity of the prefill that continues a cache (mimo_attn_prefill_cached)
against the fp64 oracle, through the C ABI.

Each case runs a chunk of S tokens after past_lens[b] cached tokens and
compares every output row of the checked heads and the updated caches: the
chunk's rotated keys (bf16 rounding of an fp32 rotation: the prefill bar) and
values (exact) in their slots, every other slot untouched. Bars as in
test_parity_gpu: bf16 max-abs <= 2e-2 and mean-abs <= 2e-3, fp32 <= 1e-4.
"""
import numpy as np
import pytest
import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic
import oracle
from tests.parity_util import compare, f64, lib_layer

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mimo.load()
    mimo.mimo_attn_get_device_error()  # clear


def _run(spec, past, S, *, dtype=BF, heads=None, seed=0, capacity=None):
    B = len(past)
    cap = capacity if capacity is not None else max(past) + S + 5
    q, k, v, kc, vc, sinks = synthetic.cached_prefill_inputs(spec, B, S, cap, seed=seed, layer=0, dtype=dtype,
                                                             device="cuda")
    sinks = sinks if spec.layer_type == 1 else None
    kc0, vc0 = kc.clone(), vc.clone()
    lay = lib_layer(spec, sinks)
    past_dev = torch.tensor(past, dtype=torch.int32, device="cuda")
    out = mimo.prefill_cached(lay, q, k, v, past_dev, kc, vc, max_past_len=max(past))
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    heads = list(range(spec.num_q_heads)) if heads is None else list(heads)
    ref, kc_ref, vc_ref = oracle.prefill_cached_layer(
        f64(q), f64(k), f64(v), f64(kc0), f64(vc0), past, layer_type=spec.layer_type,
        num_kv_heads=spec.num_kv_heads, rotary_dim=spec.rotary_dim, theta=spec.theta, window=spec.window,
        sinks=None if sinks is None else f64(sinks), hidden_size=spec.hidden_size, heads=heads)
    gpu = f64(out)
    c = compare(gpu[:, :, heads].reshape(-1), ref[:, :, heads].reshape(-1))
    assert c.ok(dtype), f"out: max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e}"
    # caches: written slots match the oracle, the rest is untouched
    kbar = 2e-2 if dtype == BF else 1e-5
    kc_g, vc_g = f64(kc), f64(vc)
    for b, P in enumerate(past):
        if spec.layer_type == 0:
            written = set(range(P, P + S))
        else:
            written = {(P + t) % spec.window for t in range(max(0, S - spec.window), S)}
        for slot in range(kc.shape[1]):
            if slot in written:
                assert np.max(np.abs(kc_g[b, slot] - kc_ref[b, slot])) <= kbar, (b, slot)
                assert np.array_equal(vc_g[b, slot], vc_ref[b, slot]), (b, slot)
            else:
                assert torch.equal(kc[b, slot], kc0[b, slot]) and torch.equal(vc[b, slot], vc0[b, slot]), (b, slot)
    return c


@pytest.mark.parametrize("past,S", [([0, 0], 130), ([1, 127], 1), ([100, 128], 7), ([300, 5], 200),
                                    ([129, 1000], 129)])
def test_global_chunk_continuing_cache(past, S):
    """Global layers (prefill_ga_kernel reading the linear cache): chunks of 1,
    ragged and multi-tile lengths after empty, short and long caches, mixed per
    sequence."""
    _run(synthetic.mimo_layer(0), past, S, heads=range(0, 64, 5), seed=S)


@pytest.mark.parametrize("past,S", [([0, 0], 100), ([5, 127], 16), ([128, 200], 17), ([1000, 3], 129),
                                    ([77, 4000], 300), ([250, 251], 1)])
def test_swa_chunk_continuing_cache(past, S):
    """Sliding layers (key window gathered from the ring, prefill_swa_kernel):
    caches shorter and longer than the window, chunks of 1 token, of a block
    (16), ragged, and longer than the window (the ring wraps within the
    chunk)."""
    _run(synthetic.mimo_layer(1), past, S, heads=range(0, 64, 5), seed=S + 1)


@pytest.mark.parametrize("layer_type", [0, 1])
def test_cached_fp32_cuda_core_path(layer_type):
    """fp32 tiny layers take the CUDA-core kernel with the same offsets."""
    spec = synthetic.TINY_PAIR.layers[0 if layer_type == 1 else 1]
    _run(spec, [0, 3, 20, 40], 23, dtype=torch.float32)


def test_chunks_equal_one_shot_prefill_on_gpu():
    """Two chunks through the library give the one-shot prefill's rows (the
    same property the oracle is pinned to, here end to end on the GPU)."""
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        B, S1, S2 = 2, 300, 200
        q, k, v, sinks = synthetic.prefill_inputs(spec, B, S1 + S2, seed=9, layer=0, device="cuda")
        sinks = sinks if lt == 1 else None
        lay = lib_layer(spec, sinks)
        full = mimo.prefill(lay, q, k, v)
        cap = spec.window if lt == 1 else S1 + S2
        kc = torch.zeros((B, cap, spec.num_kv_heads, spec.qk_dim), dtype=BF, device="cuda")
        vc = torch.zeros((B, cap, spec.num_kv_heads, spec.v_dim), dtype=BF, device="cuda")
        zeros = torch.zeros(B, dtype=torch.int32, device="cuda")
        o1 = mimo.prefill_cached(lay, q[:, :S1].contiguous(), k[:, :S1].contiguous(), v[:, :S1].contiguous(),
                                 zeros, kc, vc, max_past_len=0)
        o2 = mimo.prefill_cached(lay, q[:, S1:].contiguous(), k[:, S1:].contiguous(), v[:, S1:].contiguous(),
                                 zeros + S1, kc, vc, max_past_len=S1)
        torch.cuda.synchronize()
        c = compare(f64(torch.cat([o1, o2], dim=1)).reshape(-1), f64(full).reshape(-1))
        assert c.max_abs <= 2e-2 and c.mean_abs <= 2e-3, (lt, c)


def test_out_of_range_past_len_sets_device_error():
    """past_lens beyond max_past_len is reported in the device error word."""
    spec = synthetic.mimo_layer(0)
    q, k, v, kc, vc, _ = synthetic.cached_prefill_inputs(spec, 1, 8, 64, seed=1, layer=0, device="cuda")
    lay = lib_layer(spec, None)
    mimo.mimo_attn_get_device_error()
    mimo.prefill_cached(lay, q, k, v, torch.tensor([50], dtype=torch.int32, device="cuda"), kc, vc,
                        max_past_len=10)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() & mimo.DEVERR_KV_LEN
