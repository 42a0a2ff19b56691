"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Bars: bf16 inputs max-abs <= 2e-2 and mean-abs <= 2e-3; fp32 inputs max-abs
<= 1e-4. Small and ragged shapes are compared element by element; the large
workloads (SWA B1 S4096 in full, global B2 S8192 on sampled rows) at the
sizes and launch configuration the benchmark uses.
"""
import math

import numpy as np
import pytest
import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic
import oracle
from tests.parity_util import check_prefill, compare, f64, lib_layer

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    mimo.load()
    mimo.mimo_attn_get_device_error()  # clear


def _assert(c, dtype, what):
    assert c.ok(dtype), f"{what}: max_abs={c.max_abs:.3e} mean_abs={c.mean_abs:.3e} over {c.n}"


# ------------------------------------------------------------------ prefill

def test_tiny_pair_fp32_full():
    """Tiny SWA + global pair in fp32 (CUDA-core path), every output."""
    for li, spec in enumerate(synthetic.TINY_PAIR.layers):
        c, _, _ = check_prefill(spec, 1, 64, torch.float32, layer_idx=li)
        _assert(c, torch.float32, f"tiny layer {li}")


@pytest.mark.parametrize("layer_type", [0, 1])
@pytest.mark.parametrize("S", [1, 5, 16, 127, 128, 129, 300])
def test_tc_prefill_small_and_ragged_full(layer_type, S):
    """Tensor-core path, every output, sequence lengths around the tile sizes
    (128 rows; 16 positions x 8 heads on sliding layers)."""
    spec = synthetic.mimo_layer(layer_type)
    c, _, _ = check_prefill(spec, 2, S, BF, seed=S)
    _assert(c, BF, f"type {layer_type} S {S}")


@pytest.mark.parametrize("layer_type", [0, 1])
def test_tc_prefill_output_16_byte_aligned(layer_type):
    """An output that is 16- but not 32-byte aligned takes the 16-byte store
    path of the epilogue (32-byte aligned outputs use 256-bit stores)."""
    spec = synthetic.mimo_layer(layer_type)
    c, out, _ = check_prefill(spec, 2, 300, BF, seed=3, out_offset_elems=8)
    assert out.data_ptr() % 32 == 16
    _assert(c, BF, f"type {layer_type} 16-byte aligned output")


@pytest.mark.parametrize("window", [1, 2, 17, 129, 500])
def test_tc_prefill_windows(window):
    spec = synthetic.mimo_layer(1)
    c, _, _ = check_prefill(spec, 1, 400, BF, window=window, heads=range(0, 64, 3))
    _assert(c, BF, f"window {window}")


@pytest.mark.parametrize("rotary", [0, 2, 16, 32, 48, 64, 96, 192])
def test_tc_prefill_rotary_dims(rotary):
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        c, _, _ = check_prefill(spec, 1, 200, BF, rotary=rotary, heads=range(0, 64, 5))
        _assert(c, BF, f"rotary {rotary} type {lt}")


@pytest.mark.parametrize("hq,hkv_swa,hkv_ga", [(16, 16, 16), (32, 2, 2), (64, 64, 64), (8, 1, 1)])
def test_tc_prefill_gqa_shapes(hq, hkv_swa, hkv_ga):
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt, hq=hq, swa_kv=hkv_swa, ga_kv=hkv_ga)
        c, _, _ = check_prefill(spec, 1, 260, BF)
        _assert(c, BF, f"hq {hq} type {lt}")


def test_prefill_positions_shift():
    """Explicit RoPE positions (here 0..S-1 shifted by 40000) are honoured."""
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        pos = torch.arange(40000, 40000 + 150, dtype=torch.int32, device="cuda")
        c, _, _ = check_prefill(spec, 1, 150, BF, positions=pos, heads=range(0, 64, 7))
        _assert(c, BF, f"positions type {lt}")


def test_bf16_other_dims_cuda_core_path():
    """bf16 with head dims the tensor-core kernel does not take (CUDA-core path)."""
    spec = synthetic.LayerSpec(1, 8, 2, 64, 48, 32, 20, 1e4, 384, True)
    c, _, _ = check_prefill(spec, 2, 90, BF)
    _assert(c, BF, "bf16 64/48")


@pytest.mark.parametrize("B,S", [(3, 1000), (5, 777), (1, 2500)])
def test_swa_prefill_ring_runs_every_output(B, S):
    """Sliding layers with several KV-group runs per CTA and ring wrap-around
    (contiguous tile ranges cross (batch, KV head) boundaries)."""
    spec = synthetic.mimo_layer(1)
    c, _, _ = check_prefill(spec, B, S, BF, seed=B * 1000 + S, heads=range(0, 64, 3))
    _assert(c, BF, f"SWA B{B} S{S}")


@pytest.mark.parametrize("hq,hkv,window,S", [(32, 8, 64, 4790), (16, 8, 32, 9590), (8, 8, 16, 19000)])
def test_swa_prefill_staged_stores_other_head_groups(hq, hkv, window, S):
    """The sliding kernel's staged TMA-store epilogue (16 or more tiles per
    CTA) with 4, 2 and 1 query heads per KV group: a tile is then 32, 64 or 128
    positions of those heads, and each warp stores its 32 rows as a box of
    32 / heads positions. Ragged sequence ends; every row of a subset of
    heads, both batches."""
    spec = synthetic.mimo_layer(1, hq=hq, swa_kv=hkv, window=window)
    c, _, _ = check_prefill(spec, 2, S, BF, seed=hq + S, heads=range(0, hq, max(1, hq // 8)))
    _assert(c, BF, f"SWA Hq{hq} Hkv{hkv} W{window} B2 S{S}")
    assert mimo.mimo_attn_get_device_error() == 0


def test_swa_prefill_full_size_every_output():
    """Single SWA layer, B1 S4096 Hq64 Hkv8 qk192 v128 r64 W128: every output."""
    spec = synthetic.SWA_PREFILL.layers[0]
    c, _, _ = check_prefill(spec, 1, 4096, BF)
    _assert(c, BF, "SWA B1 S4096")


def test_global_prefill_full_size_sampled_rows():
    """Single global layer, B2 S8192 Hq64 Hkv4: all heads on sampled rows."""
    spec = synthetic.GLOBAL_PREFILL.layers[0]
    c, _, _ = check_prefill(spec, 2, 8192, BF, rows="sample", n_random_rows=16)
    _assert(c, BF, "global B2 S8192")


@pytest.mark.parametrize("layer_idx", [0, 1])
def test_hybrid_stack_full_size_sampled_rows(layer_idx):
    """The hybrid 8-layer stack's prefill at its full size, B4 S32768 (Hq 64,
    qk 192 / v 128, rotary 64), layer by layer as the benchmark runs it: layer
    0 is global (4 KV heads, rope_theta) and layer 1 sliding (8 KV heads,
    window 128, sinks), with the benchmark's seeds and launch path. Every
    batch and all 64 heads on rows {0, 1, 126..129, 16383, 16384, 32766,
    32767} plus 16 seeded random rows. Q alone is 3.2 GB here, so byte
    offsets pass 2^31 and the global kernel's grid is (256, 32, 4)."""
    wl = synthetic.HYBRID_PREFILL
    spec = wl.layers[layer_idx]
    assert spec.layer_type == (0 if layer_idx == 0 else 1)
    c, out, inputs = check_prefill(spec, wl.batch, wl.seq, BF, seed=0, layer_idx=layer_idx, rows="sample",
                                   n_random_rows=16)
    del out, inputs
    torch.cuda.empty_cache()
    _assert(c, BF, f"hybrid stack layer {layer_idx} B{wl.batch} S{wl.seq}")
    assert mimo.mimo_attn_get_device_error() == 0


def test_prefill_is_deterministic():
    spec = synthetic.mimo_layer(0)
    q, k, v, _ = synthetic.prefill_inputs(spec, 1, 700, seed=3, layer=0, dtype=BF, device="cuda")
    lay = lib_layer(spec, None)
    a = mimo.prefill(lay, q, k, v)
    b = mimo.prefill(lay, q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_prefill_writes_caches():
    """Global: rotated keys / values in slots 0..S-1 of a linear cache; SWA:
    the last `window` tokens in ring slot i mod window. Untouched slots keep
    their contents."""
    S = 300
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        q, k, v, sinks = synthetic.prefill_inputs(spec, 2, S, seed=5, layer=0, dtype=BF, device="cuda")
        sinks = sinks if lt == 1 else None
        cap = spec.window if lt == 1 else S + 37
        kc = torch.full((2, cap, spec.num_kv_heads, 192), 7.0, dtype=BF, device="cuda")
        vc = torch.full((2, cap, spec.num_kv_heads, 128), 7.0, dtype=BF, device="cuda")
        lay = lib_layer(spec, sinks)
        out = mimo.prefill(lay, q, k, v, k_cache=kc, v_cache=vc)
        ref_out = mimo.prefill(lay, q, k, v)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out)
        pos = np.arange(S, dtype=np.float64)
        for b in range(2):
            for kv in range(spec.num_kv_heads):
                kr = oracle.rope(f64(k[b, :, kv]), 64, spec.theta, pos)
                if lt == 0:
                    got_k, got_v, want_k, want_v = f64(kc[b, :S, kv]), vc[b, :S, kv], kr, v[b, :, kv]
                    assert torch.all(kc[b, S:] == 7.0) and torch.all(vc[b, S:] == 7.0)
                else:
                    toks = np.arange(S - spec.window, S)
                    slots = toks % spec.window
                    got_k, got_v = f64(kc[b, slots, kv]), vc[b, slots, kv]
                    want_k, want_v = kr[toks], v[b, toks, kv]
                assert np.max(np.abs(got_k - want_k)) <= 2e-2
                assert torch.equal(got_v, want_v)


# ------------------------------------------------------------------- decode

def _oracle_decode(spec, b, L, q, kn, vn, kc, vc, sinks):
    G = spec.num_q_heads // spec.num_kv_heads
    outs = []
    for kv in range(spec.num_kv_heads):
        hs = slice(kv * G, (kv + 1) * G)
        o, kc2, vc2 = oracle.decode(f64(q[b, hs]), f64(kn[b, kv]), f64(vn[b, kv]), f64(kc[b, :, kv]),
                                    f64(vc[b, :, kv]), L, spec.rotary_dim, spec.theta, spec.layer_type,
                                    spec.window, 1 / math.sqrt(spec.qk_dim),
                                    None if sinks is None else f64(sinks[hs]),
                                    oracle.v_scale(spec.hidden_size, spec.num_q_heads, spec.v_dim))
        outs.append((o, kc2, vc2))
    return outs


def _run_decode(spec, B, cap, lens, dtype=BF, seed=0):
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, sinks = synthetic.decode_inputs(spec, B, cap, kv_lens, seed=seed, layer=0, dtype=dtype,
                                                       device="cuda")
    sinks = sinks if spec.layer_type == 1 else None
    kc0, vc0 = kc.clone(), vc.clone()
    lay = lib_layer(spec, sinks)
    out = mimo.decode(lay, q, kn, vn, kv_lens.cuda(), kc, vc)
    torch.cuda.synchronize()
    return out, (q, kn, vn, kc0, vc0, sinks), (kc, vc)


def _check_decode(spec, out, inputs, caches, batches, lens, dtype=BF):
    q, kn, vn, kc0, vc0, sinks = inputs
    kc, vc = caches
    G = spec.num_q_heads // spec.num_kv_heads
    gpu, ref = [], []
    for b in batches:
        L = int(lens[b])
        res = _oracle_decode(spec, b, L, q, kn, vn, kc0, vc0, sinks)
        for kv, (o, kc2, vc2) in enumerate(res):
            gpu.append(f64(out[b, kv * G:(kv + 1) * G]))
            ref.append(o)
            slot = (L - 1) % spec.window if spec.layer_type == 1 else L - 1
            assert np.max(np.abs(f64(kc[b, slot, kv]) - kc2[slot])) <= (2e-2 if dtype == BF else 1e-5)
            assert np.array_equal(f64(vc[b, slot, kv]), vc2[slot])
        others = [s for s in range(kc.shape[1]) if s != ((L - 1) % spec.window if spec.layer_type == 1 else L - 1)]
        assert torch.equal(kc[b, others], kc0[b, others]) and torch.equal(vc[b, others], vc0[b, others])
    c = compare(np.concatenate(gpu), np.concatenate(ref))
    _assert(c, dtype, "decode")


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_small_every_output(layer_type):
    spec = synthetic.mimo_layer(layer_type)
    # lengths around the 64-key tiles, the 128-slot ring and the 2048-key splits
    lens = [1, 2, 63, 64, 65, 127, 128, 129, 1023, 2047, 2048, 2049, 4097, 5000]
    cap = 5000
    out, inputs, caches = _run_decode(spec, len(lens), cap, lens)
    _check_decode(spec, out, inputs, caches, range(len(lens)), lens)


@pytest.mark.parametrize("window", [16, 64, 100, 128, 192, 256])
def test_decode_sliding_windows(window):
    """Sliding layers with rings of one to four 64-key tiles: up to two tiles
    take the slim kernel form (one stage, 4 CTAs per SM), longer rings the
    2-stage one. Lengths below, at and past the window; every output."""
    spec = synthetic.mimo_layer(1, window=window)
    lens = sorted({1, 2, window - 1, window, window + 1, 2 * window + 3, 700} - {0})
    out, inputs, caches = _run_decode(spec, len(lens), window, lens, seed=window)
    _check_decode(spec, out, inputs, caches, range(len(lens)), lens)


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_stale_slots_hold_nan(layer_type):
    """Cache slots past a sequence's length may hold any bits: with NaN in
    every slot a sequence has not written yet (global: slots >= L; ring:
    slots >= L while L < window), the output equals the one from finite
    caches. Lengths cover the first tiles, which the kernel loads before it
    reads kv_lens."""
    spec = synthetic.mimo_layer(layer_type)
    lens = [1, 2, 63, 64, 65, 100, 127, 128, 129, 191, 192, 300]
    B, cap = len(lens), 512
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, sinks = synthetic.decode_inputs(spec, B, cap, kv_lens, seed=5, layer=0, dtype=BF,
                                                       device="cuda")
    sinks = sinks if layer_type == 1 else None
    kc0, vc0 = kc.clone(), vc.clone()
    for b, L in enumerate(lens):
        kc[b, L:] = float("nan")
        vc[b, L:] = float("nan")
    lay = lib_layer(spec, sinks)
    out = mimo.decode(lay, q, kn, vn, kv_lens.cuda(), kc, vc)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    assert bool(torch.isfinite(out).all())
    G = spec.num_q_heads // spec.num_kv_heads
    gpu, ref = [], []
    for b, L in enumerate(lens):
        for kv, (o, _, _) in enumerate(_oracle_decode(spec, b, L, q, kn, vn, kc0, vc0, sinks)):
            gpu.append(f64(out[b, kv * G:(kv + 1) * G]))
            ref.append(o)
    _assert(compare(np.concatenate(gpu), np.concatenate(ref)), BF, "decode, NaN in unwritten slots")


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_fp32_cuda_core_path(layer_type):
    spec = synthetic.LayerSpec(layer_type, 4, 2 if layer_type else 1, 48, 32, 16, 16,
                               1e4 if layer_type else 1e6, 256, layer_type == 1)
    lens = [1, 3, 16, 17, 40]
    out, inputs, caches = _run_decode(spec, len(lens), 64, lens, dtype=torch.float32)
    _check_decode(spec, out, inputs, caches, range(len(lens)), lens, dtype=torch.float32)


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_cuda_graph_replay(layer_type):
    """After its first call the decode entry point makes no synchronising or
    allocating CUDA call, so a serving loop can capture it in a CUDA graph: a
    replay writes the same output as a direct call, and that output passes
    parity."""
    spec = synthetic.mimo_layer(layer_type)
    lens = [1, 65, 129, 2049, 5000]
    B, cap = len(lens), 5000
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, sinks = synthetic.decode_inputs(spec, B, cap, kv_lens, seed=7, layer=0, dtype=BF,
                                                       device="cuda")
    sinks = sinks if layer_type == 1 else None
    kc0, vc0 = kc.clone(), vc.clone()
    lay = lib_layer(spec, sinks)
    lens_dev = kv_lens.cuda()
    out = torch.empty((B, spec.num_q_heads, spec.v_dim), dtype=BF, device="cuda")
    need = mimo.mimo_attn_decode_workspace_size(lay, mimo.BF16, B, kc.shape[1])
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")

    slots = kc.shape[1]  # the ring of a sliding layer has `window` slots

    def call(stream):
        st = mimo.mimo_attn_decode(lay, mimo.BF16, B, q, kn, vn, lens_dev, kc, vc, slots, out, ws, ws.numel(), stream)
        assert st == mimo.OK

    call(torch.cuda.current_stream())
    torch.cuda.synchronize()
    direct = out.clone()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, direct)
    _check_decode(spec, out, (q, kn, vn, kc0, vc0, sinks), (kc, vc), range(B), lens)


def test_decode_full_size_sampled_batches():
    """Hybrid decode workload (B64, L ~ U[1024, 32768], cache 32768): one
    global and one SWA layer; every head of 6 sampled sequences."""
    lens = synthetic.decode_kv_lens(64, 1024, 32768, seed=0).tolist()
    rng = np.random.default_rng(0)
    batches = sorted(set(rng.integers(0, 64, 4).tolist()) | {int(np.argmax(lens)), int(np.argmin(lens))})
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        out, inputs, caches = _run_decode(spec, 64, 32768, lens)
        _check_decode(spec, out, inputs, caches, batches, lens)


def test_decode_equals_prefill_last_row():
    """Prefill S tokens with caches, then decode token S: the decode output
    equals the oracle's prefill row S over all S+1 tokens."""
    S = 700
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        q, k, v, sinks = synthetic.prefill_inputs(spec, 1, S + 1, seed=9, layer=0, dtype=BF, device="cuda")
        sinks = sinks if lt == 1 else None
        cap = spec.window if lt == 1 else 1024
        kc = torch.zeros((1, cap, spec.num_kv_heads, 192), dtype=BF, device="cuda")
        vc = torch.zeros((1, cap, spec.num_kv_heads, 128), dtype=BF, device="cuda")
        lay = lib_layer(spec, sinks)
        mimo.prefill(lay, q[:, :S].contiguous(), k[:, :S].contiguous(), v[:, :S].contiguous(),
                     k_cache=kc, v_cache=vc)
        lens = torch.tensor([S + 1], dtype=torch.int32, device="cuda")
        out = mimo.decode(lay, q[:, S].contiguous(), k[:, S].contiguous(), v[:, S].contiguous(), lens, kc, vc)
        torch.cuda.synchronize()
        from tests.parity_util import oracle_prefill
        ref = oracle_prefill(spec, q, k, v, sinks, {(0, h): [S] for h in range(64)})
        c = compare(np.concatenate([f64(out[0, h:h + 1]) for h in range(64)]),
                    np.concatenate([ref[(0, h)][1] for h in range(64)]))
        _assert(c, BF, f"decode vs prefill type {lt}")


def test_decode_bad_kv_len_sets_device_error():
    """kv_lens out of range (0, or above a global cache's capacity) is caught
    by the kernel: the device error word gets its bit and that sequence's
    output and cache stay untouched, while the others are computed."""
    spec = synthetic.mimo_layer(0)
    mimo.mimo_attn_get_device_error()
    lens = [0, 100, 5000]
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, _ = synthetic.decode_inputs(spec, 3, 4096, kv_lens, seed=1, layer=0, dtype=BF, device="cuda")
    kc0 = kc.clone()
    out = torch.full((3, 64, 128), 3.0, dtype=BF, device="cuda")
    lay = lib_layer(spec, None)
    mimo.decode(lay, q, kn, vn, kv_lens.cuda(), kc, vc, out=out)
    bits = mimo.mimo_attn_get_device_error()
    assert bits & mimo.DEVERR_KV_LEN
    assert torch.all(out[0] == 3.0) and torch.all(out[2] == 3.0)
    assert torch.equal(kc[0], kc0[0]) and torch.equal(kc[2], kc0[2])
    assert not torch.all(out[1] == 3.0)
    assert mimo.mimo_attn_get_device_error() == 0
