"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function include/mimo_attn.h declares, and rejects bad arguments with the
documented status before any launch."""
import ctypes
import math
import os
import re

import pytest

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import build as mimo_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mimo_build.build()
    return mimo.load()


def header_functions():
    text = open(os.path.join(ROOT, "include", "mimo_attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mimo_attn_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_function(lib):
    names = header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(mimo.EXPORTED)


def test_version_and_status_strings(lib):
    assert "sm_100a" in mimo.version()
    assert mimo.status_string(mimo.OK) == "ok"
    assert mimo.status_string(mimo.ERR_WORKSPACE).startswith("workspace")
    assert mimo.status_string(99) == "unknown status"


@pytest.mark.parametrize("f,d,want", [(1 / 3, 192, 64), (0.334, 192, 64), (0.5, 48, 24), (1 / 3, 48, 16),
                                      (0.0, 128, 0), (1.0, 128, 128), (-0.1, 64, -1),
                                      (float("nan"), 64, -1)])
def test_rotary_dim_is_int_of_product(lib, f, d, want):
    """int(partial_rotary_factor * head_dim), lablup/mlxcel issue 842."""
    got = mimo.rotary_dim(f, d)
    assert got == want
    if want >= 0:
        assert got == int(f * d)


def layer(**kw):
    base = dict(layer_type=mimo.SWA, num_q_heads=64, num_kv_heads=8, qk_dim=192, v_dim=128,
                rotary_dim=64, window=128, rope_theta=1e4, hidden_size=4096, sinks=None)
    base.update(kw)
    return mimo.make_layer(**base)


FAKE = 4096  # a 16-byte-aligned fake device address; never dereferenced (checks fail first)


def T(addr=FAKE):
    class _F:
        def is_contiguous(self):
            return True

        def data_ptr(self):
            return addr
    return _F()


def prefill_status(l, dtype=mimo.BF16, batch=1, seq=16, cache=None, cap=0, ws_bytes=1 << 30, q=None, stream=0):
    kc = vc = None
    if cache == "both":
        kc, vc = T(), T()
    elif cache == "k":
        kc = T()
    return mimo.mimo_attn_prefill(l, dtype, batch, seq, q or T(), T(), T(), None, T(), kc, vc, cap,
                                  T(), ws_bytes, stream)


def test_prefill_rejects_bad_layers(lib):
    bad = [dict(num_kv_heads=7), dict(num_q_heads=0), dict(rotary_dim=63), dict(rotary_dim=194),
           dict(rotary_dim=-2), dict(window=0), dict(layer_type=2), dict(qk_dim=191),
           dict(hidden_size=0), dict(rope_theta=0.0), dict(rope_theta=float("inf")),
           dict(layer_type=mimo.GLOBAL, sinks=T(8192))]
    mimo.mimo_attn_debug_fail_launches(True)
    try:
        for kw in bad:
            assert prefill_status(layer(**kw)) == mimo.ERR_INVALID_ARG, kw
        assert prefill_status(layer(qk_dim=258, rotary_dim=64)) == mimo.ERR_UNSUPPORTED
        assert prefill_status(layer(v_dim=512)) == mimo.ERR_UNSUPPORTED
    finally:
        mimo.mimo_attn_debug_fail_launches(False)


def test_prefill_rejects_bad_shapes_and_buffers(lib):
    mimo.mimo_attn_debug_fail_launches(True)
    try:
        l = layer()
        assert prefill_status(l, dtype=5) == mimo.ERR_INVALID_ARG
        assert prefill_status(l, batch=-1) == mimo.ERR_INVALID_ARG
        assert prefill_status(l, cache="k", cap=128) == mimo.ERR_INVALID_ARG       # one cache only
        assert prefill_status(l, cache="both", cap=64) == mimo.ERR_INVALID_ARG     # ring != window
        g = layer(layer_type=mimo.GLOBAL, num_kv_heads=4)
        assert prefill_status(g, cache="both", cap=8, seq=16) == mimo.ERR_INVALID_ARG  # cap < seq
        assert prefill_status(l, q=T(FAKE + 2)) == mimo.ERR_INVALID_ARG            # misaligned bf16
        assert prefill_status(l, ws_bytes=10) == mimo.ERR_WORKSPACE
        # empty problems are valid no-ops that launch nothing
        assert prefill_status(l, batch=0) == mimo.OK
        assert prefill_status(l, seq=0) == mimo.OK
        # well-formed arguments reach the launch step (the hook fails it)
        assert prefill_status(l) == mimo.ERR_CUDA
        # a global cache takes the rotated keys; the workspace then holds only the RoPE table
        assert prefill_status(g, cache="both", cap=16, ws_bytes=0) == mimo.ERR_WORKSPACE
        assert prefill_status(g, cache="both", cap=16, ws_bytes=16 * 32 * 8) == mimo.ERR_CUDA
    finally:
        mimo.mimo_attn_debug_fail_launches(False)


def decode_status(l, batch=2, cap=128, ws=1 << 30, dtype=mimo.BF16, lens=True):
    return mimo.mimo_attn_decode(l, dtype, batch, T(), T(), T(), T() if lens else None, T(), T(), cap,
                                 T(), T(), ws, 0)


def test_decode_argument_checks(lib):
    mimo.mimo_attn_debug_fail_launches(True)
    try:
        l = layer()
        assert decode_status(l, cap=64) == mimo.ERR_INVALID_ARG          # ring must equal window
        assert decode_status(l, lens=False) == mimo.ERR_INVALID_ARG
        assert decode_status(l, batch=0) == mimo.OK
        assert decode_status(l) == mimo.ERR_CUDA
        g = layer(layer_type=mimo.GLOBAL, num_kv_heads=4)
        assert decode_status(g, cap=0) == mimo.ERR_INVALID_ARG
        need = mimo.mimo_attn_decode_workspace_size(g, mimo.BF16, 64, 32768)
        assert need > 0
        assert decode_status(g, batch=64, cap=32768, ws=need - 1) == mimo.ERR_WORKSPACE
        assert decode_status(g, batch=64, cap=32768, ws=need) == mimo.ERR_CUDA
    finally:
        mimo.mimo_attn_debug_fail_launches(False)


def test_workspace_sizes(lib):
    l = layer()
    # RoPE table [S, r/2] (cos, sin); the sliding-window tensor-core kernel
    # rotates K itself, so bf16 needs no rotated copy of K ...
    assert mimo.mimo_attn_prefill_workspace_size(l, mimo.BF16, 1, 4096) == 4096 * 32 * 8
    # ... while fp32 (CUDA-core path) also takes the rotated keys [B, S, Hkv, Dqk]
    assert mimo.mimo_attn_prefill_workspace_size(l, mimo.FP32, 1, 4096) == 4096 * 32 * 8 + 4096 * 8 * 192 * 4
    assert mimo.mimo_attn_prefill_workspace_size(l, mimo.FP32, 1, 3) == 3 * 32 * 8 + 256 * math.ceil(3 * 8 * 192 * 4 / 256)
    # one split per sequence on the ring: no partials needed
    assert mimo.mimo_attn_decode_workspace_size(l, mimo.BF16, 64, 128) == 0
    g = layer(layer_type=mimo.GLOBAL, num_kv_heads=4)
    splits = 32768 // 2048
    assert mimo.mimo_attn_decode_workspace_size(g, mimo.BF16, 64, 32768) == 64 * 64 * splits * 130 * 4
    assert mimo.mimo_attn_prefill_workspace_size(layer(num_kv_heads=7), mimo.BF16, 1, 8) == 0


def test_layer_selection_from_config(lib):
    """hybrid_layer_pattern[idx] == 1 selects a sliding layer with its own
    theta, KV-head count, window and sink (lablup/mlxcel issue 842)."""
    cfg = dict(num_attention_heads=64, swa_num_key_value_heads=8, num_key_value_heads=4, head_dim=192,
               v_head_dim=128, partial_rotary_factor=1 / 3, sliding_window_size=128, rope_theta=5e6,
               swa_rope_theta=1e4, hidden_size=4096, sinks=T(8192))
    pattern = [0, 1, 1, 1, 1, 1, 0, 1]
    got = [mimo.layer_from_config(pattern, i, **cfg) for i in range(8)]
    for i, l in enumerate(got):
        if pattern[i] == 1:
            assert (l.layer_type, l.num_kv_heads, l.rope_theta, l.window) == (mimo.SWA, 8, 1e4, 128)
            assert l.sinks == 8192
        else:
            assert (l.layer_type, l.num_kv_heads, l.rope_theta) == (mimo.GLOBAL, 4, 5e6)
            assert l.sinks is None
        assert l.rotary_dim == 64 and l.qk_dim == 192 and l.v_dim == 128


def cached_status(l, batch=2, seq=16, max_past=100, cap=None, ws_bytes=1 << 30, past=True, caches=True):
    if cap is None:
        cap = l.window if l.layer_type == mimo.SWA else max_past + seq
    return mimo.mimo_attn_prefill_cached(l, mimo.BF16, batch, seq, T(), T(), T(), T() if past else None, max_past,
                                         T(), T() if caches else None, T() if caches else None, cap, T(),
                                         ws_bytes, 0)


def test_prefill_cached_argument_checks(lib):
    mimo.mimo_attn_debug_fail_launches(True)
    try:
        swa = layer()
        ga = layer(layer_type=mimo.GLOBAL, num_kv_heads=4)
        assert cached_status(swa, caches=False) == mimo.ERR_INVALID_ARG      # caches are required
        assert cached_status(swa, cap=64) == mimo.ERR_INVALID_ARG            # ring must equal the window
        assert cached_status(ga, cap=100 + 16 - 1) == mimo.ERR_INVALID_ARG   # cap < max_past + seq
        assert cached_status(ga, max_past=-1, cap=16) == mimo.ERR_INVALID_ARG
        assert cached_status(ga, past=False) == mimo.ERR_INVALID_ARG
        assert cached_status(ga, batch=0) == mimo.OK                         # empty problems are no-ops
        assert cached_status(swa, seq=0) == mimo.OK
        assert cached_status(ga, ws_bytes=10) == mimo.ERR_WORKSPACE
        assert cached_status(ga) == mimo.ERR_CUDA                            # reaches the launch step
        assert cached_status(swa) == mimo.ERR_CUDA
    finally:
        mimo.mimo_attn_debug_fail_launches(False)


def test_prefill_cached_workspace_sizes(lib):
    ga = layer(layer_type=mimo.GLOBAL, num_kv_heads=4)
    # global: only the RoPE table of positions 0 .. max_past + seq - 1
    assert mimo.mimo_attn_prefill_cached_workspace_size(ga, mimo.BF16, 4, 4096, 28672) == (28672 + 4096) * 32 * 8
    # sliding: the table, then key and value windows of round_up(W - 1, 16) + seq rows
    swa = layer()
    rows = 2 * (128 + 100) * 8
    want = 256 * math.ceil((50 + 100) * 32 * 8 / 256) + 256 * math.ceil(rows * 192 * 2 / 256) + \
        256 * math.ceil(rows * 128 * 2 / 256)
    assert mimo.mimo_attn_prefill_cached_workspace_size(swa, mimo.BF16, 2, 100, 50) == want
    w17 = layer(window=17)  # key offset round_up(16, 16) = 16
    rows = 1 * (16 + 10) * 8
    assert mimo.mimo_attn_prefill_cached_workspace_size(w17, mimo.FP32, 1, 10, 0) == \
        256 * math.ceil(10 * 32 * 8 / 256) + 256 * math.ceil(rows * 192 * 4 / 256) + 256 * math.ceil(rows * 128 * 4 / 256)
    assert mimo.mimo_attn_prefill_cached_workspace_size(ga, mimo.BF16, 1, 8, -1) == 0


def fp8_status(l, batch=2, cap=128, ws=1 << 30, ks=1.0, vs=1.0):
    return mimo.mimo_attn_decode_fp8kv(l, batch, T(), T(), T(), T(), T(), T(), cap, ks, vs, T(), T(), ws, 0)


def test_decode_fp8kv_argument_checks(lib):
    mimo.mimo_attn_debug_fail_launches(True)
    try:
        l = layer()
        assert fp8_status(l, cap=64) == mimo.ERR_INVALID_ARG                 # ring must equal window
        for bad in (0.0, -1.0, float("inf"), float("nan")):
            assert fp8_status(l, ks=bad) == mimo.ERR_INVALID_ARG
            assert fp8_status(l, vs=bad) == mimo.ERR_INVALID_ARG
        assert fp8_status(layer(qk_dim=128, rotary_dim=42)) == mimo.ERR_UNSUPPORTED
        assert fp8_status(layer(num_kv_heads=2)) == mimo.ERR_UNSUPPORTED  # G = 32 > 16
        assert fp8_status(l, batch=0) == mimo.OK
        assert fp8_status(l) == mimo.ERR_CUDA
        g = layer(layer_type=mimo.GLOBAL, num_kv_heads=4)
        need = mimo.mimo_attn_decode_fp8kv_workspace_size(g, 64, 32768)
        assert need == mimo.mimo_attn_decode_workspace_size(g, mimo.BF16, 64, 32768)
        assert fp8_status(g, batch=64, cap=32768, ws=need - 1) == mimo.ERR_WORKSPACE
        assert fp8_status(g, batch=64, cap=32768, ws=need) == mimo.ERR_CUDA
        assert mimo.mimo_attn_quantize_fp8(T(), T(), 10, 0.0, 0) == mimo.ERR_INVALID_ARG
        assert mimo.mimo_attn_quantize_fp8(None, T(), 10, 1.0, 0) == mimo.ERR_INVALID_ARG
        assert mimo.mimo_attn_quantize_fp8(None, None, 0, 1.0, 0) == mimo.OK
        assert mimo.mimo_attn_quantize_fp8(T(), T(), 10, 1.0, 0) == mimo.ERR_CUDA
    finally:
        mimo.mimo_attn_debug_fail_launches(False)


def qkv_status(l, batch=2, seq=64, past=True, max_past=10, caches=False, cap=None, ws=1 << 30, kv=True):
    if cap is None:
        cap = l.window if l.layer_type == mimo.SWA else max_past + seq
    return mimo.mimo_attn_qkv_project(l, batch, seq, T(), T(), T() if past else None, max_past, T(),
                                      T() if kv else None, T() if kv else None, T() if caches else None,
                                      T() if caches else None, cap, T(), ws, 0)


def test_qkv_project_argument_checks(lib):
    mimo.mimo_attn_debug_fail_launches(True)
    try:
        swa = layer()
        ga = layer(layer_type=mimo.GLOBAL, num_kv_heads=4)
        assert qkv_status(ga, past=False) == mimo.ERR_INVALID_ARG             # max_past without past_lens
        assert qkv_status(ga, past=False, max_past=0) == mimo.ERR_CUDA
        assert qkv_status(swa, caches=True, cap=64) == mimo.ERR_INVALID_ARG  # ring must equal the window
        assert qkv_status(ga, caches=True, cap=10 + 64 - 1) == mimo.ERR_INVALID_ARG
        assert qkv_status(ga, caches=True) == mimo.ERR_CUDA
        assert qkv_status(ga, max_past=-1) == mimo.ERR_INVALID_ARG
        assert qkv_status(layer(rotary_dim=32)) == mimo.ERR_UNSUPPORTED     # the epilogue rotates 64 or 0 dims
        assert qkv_status(layer(hidden_size=4000)) == mimo.ERR_UNSUPPORTED  # hidden not a multiple of 64
        assert qkv_status(layer(qk_dim=96, rotary_dim=32)) == mimo.ERR_UNSUPPORTED
        assert qkv_status(ga, batch=0) == mimo.OK
        assert qkv_status(ga, seq=0) == mimo.OK
        assert qkv_status(ga, ws=100) == mimo.ERR_WORKSPACE
        assert qkv_status(ga, kv=False) == mimo.ERR_CUDA
        assert qkv_status(swa) == mimo.ERR_CUDA
        # the RoPE table of positions 0 .. max_past + seq - 1
        assert mimo.mimo_attn_qkv_project_workspace_size(ga, 2, 64, 10) == 256 * math.ceil(74 * 32 * 8 / 256)
        assert mimo.mimo_attn_qkv_project_workspace_size(layer(rotary_dim=0), 2, 64, 10) == 0
    finally:
        mimo.mimo_attn_debug_fail_launches(False)


def test_python_conveniences_check_dtypes(lib):
    """decode_fp8kv wants uint8 caches and quantize_fp8 wants bf16 input; both
    refuse before touching the device."""
    import torch
    l = layer()
    q = torch.zeros((1, 64, 192), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mimo.decode_fp8kv(l, q, q[:, :8], q[:, :8, :128], torch.ones(1, dtype=torch.int32),
                          torch.zeros((1, 128, 8, 192), dtype=torch.bfloat16),
                          torch.zeros((1, 128, 8, 128), dtype=torch.uint8), 1.0, 1.0)
    with pytest.raises(ValueError):
        mimo.quantize_fp8(torch.zeros(8, dtype=torch.float32), 1.0)


def test_python_binding_refuses_host_tensors(lib):
    """Every pointer of the C ABI is a device pointer: the binding refuses
    tensors in host memory (and host sink logits) before any call."""
    import torch
    spec_q = torch.zeros((1, 16, 64, 192), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        mimo.prefill(layer(), spec_q, torch.zeros((1, 16, 8, 192), dtype=torch.bfloat16),
                     torch.zeros((1, 16, 8, 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        mimo.make_layer(mimo.SWA, 64, 8, 192, 128, 64, 128, 1e4, 4096, torch.zeros(64, dtype=torch.float32))
