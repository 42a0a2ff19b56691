"""The allocation-free decode entry point, mimo_attn_decode_static.

Some callers cannot allocate device memory at all: a host program whose own
memory pool owns the whole GPU, a plugin without an allocator, a loop that
must not pay cudaMalloc's implicit synchronisation. For them the library
keeps the split-KV partials of decode in a 16 MiB array built into the
library instead of a caller workspace. This test calls it through the C ABI
and checks it against mimo_attn_decode on calls in a row, since the shared
array keeps the previous call's contents. Both entry points run the same
kernels on the same inputs, so their outputs must be bit-identical (a
tolerance would hide a stale partial that shifts a result slightly). The
file name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic

pytestmark = pytest.mark.gpu


def _inputs(spec, lens, cap, seed, nan=False):
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, sinks = synthetic.decode_inputs(spec, len(lens), cap, kv_lens, seed=seed, layer=0,
                                                       device="cuda")
    if nan:
        for t in (q, kn, vn, kc, vc):
            t.fill_(float("nan"))
    return q, kn, vn, kc, vc, (sinks if spec.layer_type == 1 else None), kv_lens.cuda()


def _static(spec, lens, cap, seed, nan=False):
    """One mimo_attn_decode_static call; returns its output."""
    q, kn, vn, kc, vc, sinks, kv_lens = _inputs(spec, lens, cap, seed, nan)
    lay = mimo.make_layer(spec.layer_type, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim, spec.v_dim,
                          spec.rotary_dim, spec.window, spec.theta, spec.hidden_size, sinks)
    out = torch.empty((len(lens), spec.num_q_heads, spec.v_dim), dtype=torch.bfloat16, device="cuda")
    st = mimo.mimo_attn_decode_static(lay, mimo.BF16, len(lens), q, kn, vn, kv_lens, kc, vc, kc.shape[1], out)
    assert st == mimo.OK
    torch.cuda.synchronize()
    return out


def _both(spec, lens, cap, seed):
    q, kn, vn, kc, vc, sinks, kv_lens = _inputs(spec, lens, cap, seed)
    lay = mimo.make_layer(spec.layer_type, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim, spec.v_dim,
                          spec.rotary_dim, spec.window, spec.theta, spec.hidden_size, sinks)
    B = len(lens)
    cap_eff = kc.shape[1]
    # existing entry point, caller-provided workspace
    kc_a, vc_a = kc.clone(), vc.clone()
    out_a = torch.empty((B, spec.num_q_heads, spec.v_dim), dtype=torch.bfloat16, device="cuda")
    need = mimo.mimo_attn_decode_workspace_size(lay, mimo.BF16, B, cap_eff)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    st = mimo.mimo_attn_decode(lay, mimo.BF16, B, q, kn, vn, kv_lens, kc_a, vc_a, cap_eff, out_a, ws, ws.numel())
    assert st == mimo.OK
    # allocation-free entry point
    kc_b, vc_b = kc.clone(), vc.clone()
    out_b = torch.empty_like(out_a)
    st = mimo.mimo_attn_decode_static(lay, mimo.BF16, B, q, kn, vn, kv_lens, kc_b, vc_b, cap_eff, out_b)
    assert st == mimo.OK
    torch.cuda.synchronize()
    return need, (out_a, kc_a, vc_a), (out_b, kc_b, vc_b)


def _assert_same(a, b):
    """Bit-identical outputs, all finite (same kernels, same inputs)."""
    assert torch.isfinite(b.double()).all()
    assert torch.equal(a, b)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mimo.load()


def test_static_decode_matches_workspace_decode_two_calls_in_a_row():
    spec = synthetic.mimo_layer(0)  # global layer: several splits, so the array is used
    calls = [([1, 700, 5000, 8192, 3000, 1024, 1025, 6000], 11),
             ([8192, 20, 4097, 2048, 7777, 1, 512, 8000], 12)]
    for lens, seed in calls:
        need, (out_a, kc_a, vc_a), (out_b, kc_b, vc_b) = _both(spec, lens, 8192, seed)
        assert 0 < need <= 16 << 20
        _assert_same(out_a, out_b)
        assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)


def test_static_decode_single_split_layer():
    spec = synthetic.mimo_layer(1)  # sliding ring: one split, no partials
    need, (out_a, _, _), (out_b, _, _) = _both(spec, [1, 50, 128, 129, 4000], 0, 13)
    assert need == 0
    _assert_same(out_a, out_b)


def test_static_decode_ignores_stale_partials():
    """A first call at the array's capacity on all-NaN inputs leaves NaN in
    nearly every partial slot. Later calls of the same batch shape must read
    only what they wrote themselves: one with every length <= 2048 (one
    split per sequence, so no partial is read at all), then one with mixed
    lengths (several splits). A stale read would show as NaN or as a
    difference from mimo_attn_decode."""
    spec = synthetic.mimo_layer(0)
    B, cap = 120, 8192  # 120 x 64 heads x 4 splits x 130 floats = 15.97 MB of the 16 MiB
    lay0 = mimo.make_layer(0, 64, 4, 192, 128, 64, 0, spec.theta, 4096, None)
    assert 15 << 20 < mimo.mimo_attn_decode_workspace_size(lay0, mimo.BF16, B, cap) <= 16 << 20
    stale = _static(spec, [cap] * B, cap, seed=31, nan=True)
    assert torch.isnan(stale.double()).any()  # the array now holds non-finite partials
    rng = np.random.default_rng(5)
    short = rng.integers(1, 2049, B).tolist()
    mixed = rng.integers(1, cap + 1, B).tolist()
    for lens, seed in ((short, 32), (mixed, 33)):
        need, (out_a, kc_a, vc_a), (out_b, kc_b, vc_b) = _both(spec, lens, cap, seed)
        assert need > 15 << 20
        _assert_same(out_a, out_b)
        assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b)


def test_static_decode_rejects_sizes_beyond_the_array():
    """Partials above 16 MiB: a clear error, nothing launched, out untouched."""
    spec = synthetic.mimo_layer(0)
    lay = mimo.make_layer(0, 64, 4, 192, 128, 64, 0, spec.theta, 4096, None)
    B, cap = 64, 32768
    assert mimo.mimo_attn_decode_workspace_size(lay, mimo.BF16, B, cap) > 16 << 20
    q = torch.zeros((B, 64, 192), dtype=torch.bfloat16, device="cuda")
    kn = torch.zeros((B, 4, 192), dtype=torch.bfloat16, device="cuda")
    vn = torch.zeros((B, 4, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, 8, 4, 192), dtype=torch.bfloat16, device="cuda")  # never touched
    vc = torch.zeros((B, 8, 4, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.ones(B, dtype=torch.int32, device="cuda")
    out = torch.full((B, 64, 128), 5.0, dtype=torch.bfloat16, device="cuda")
    st = mimo.mimo_attn_decode_static(lay, mimo.BF16, B, q, kn, vn, lens, kc, vc, cap, out)
    torch.cuda.synchronize()
    assert st == mimo.ERR_WORKSPACE
    assert torch.all(out == 5.0)
