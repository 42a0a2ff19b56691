"""GPU parity of the fp8 (E4M3) KV-cache decode and the cache quantizer
against the fp64 oracle.

Cache inputs are the oracle's E4M3 encoding of N(0,1) bf16 caches: every
bf16 bit pattern is encoded once by oracle.e4m3_encode into a 65536-entry
table, and the caches are that table gathered by the bf16 bits (torch
indexing, no library kernel). The quantizer's codes are a decision taken in
fp32 on the GPU (x / scale rounded to fp32, then nearest E4M3), so the
oracle side takes the same decision on float32 quotients and the codes must
match bit for bit. The new token's key is rotated in fp32 on the GPU and in
fp64 by the oracle, so its codes may differ by one step next to a rounding
boundary; its value codes are bit-exact."""
import math

import numpy as np
import pytest
import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic
import oracle
from tests.parity_util import compare, f64, lib_layer

pytestmark = pytest.mark.gpu

BF = torch.bfloat16
K_SCALE = 1.0 / 16   # cached key = K_SCALE * E4M3 value; N(0,1) keys stay far below 448
V_SCALE = 1.0 / 32


def _bf16_values() -> np.ndarray:
    """Value of every bf16 bit pattern 0..65535 (as float32)."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    return bits.view(np.float32)


def _encode_table(scale: float) -> np.ndarray:
    """E4M3 code of fp32(bf16 value / scale) for every bf16 bit pattern
    (quotients that overflow to infinity saturate like any value above 448);
    NaN patterns, never drawn here, map to code 0."""
    with np.errstate(over="ignore", invalid="ignore"):
        x = _bf16_values() / np.float32(scale)  # float32 quotient, as the GPU forms it
    x = np.where(np.isnan(x), 0.0, x)
    out = np.empty(65536, dtype=np.uint8)
    for i in range(0, 65536, 4096):
        out[i:i + 4096] = oracle.e4m3_encode(x[i:i + 4096].astype(np.float64))
    return out


_TABLES = {}


def _table(scale: float) -> np.ndarray:
    if scale not in _TABLES:
        _TABLES[scale] = _encode_table(scale)
    return _TABLES[scale]


def _encode_on_device(x: torch.Tensor, scale: float) -> torch.Tensor:
    """The oracle's codes of a bf16 device tensor, gathered by bit pattern."""
    lut = torch.from_numpy(_table(scale)).to(x.device)
    idx = x.contiguous().view(torch.int16).to(torch.int32) & 0xFFFF
    return lut[idx.long()]


def _ordinal(codes: np.ndarray) -> np.ndarray:
    """Signed position of each code on the E4M3 number line (+0 and -0 both 0)."""
    c = codes.astype(np.int64)
    return np.where(c & 0x80, -(c & 0x7F), c & 0x7F)


# ---------------------------------------------------------------- quantizer

@pytest.mark.parametrize("scale", [1.0, 1.0 / 16, 0.3, 3.0])
def test_quantize_matches_encoder_bit_exact(scale):
    """Every bf16 bit pattern that is finite (ties, subnormals, saturation
    and both zeros included), plus N(0,1) data of a ragged length."""
    vals = _bf16_values()
    finite = np.isfinite(vals)
    src = torch.from_numpy(np.arange(65536, dtype=np.int32)[finite].astype(np.int16)).view(BF).cuda()
    got = mimo.quantize_fp8(src, scale).cpu().numpy()
    want = _table(scale)[finite]
    assert np.array_equal(got, want), f"{int(np.sum(got != want))} codes differ"
    n = (1 << 20) + 3
    x = synthetic.normal((n,), seed=3, tensor_id=999, dtype=BF, device="cuda")
    got = mimo.quantize_fp8(x, scale)
    assert torch.equal(got, _encode_on_device(x, scale))


def test_quantize_unaligned_and_tiny():
    x = synthetic.normal((4099,), seed=5, tensor_id=998, dtype=BF, device="cuda") * 40
    for off, n in ((1, 1), (3, 2), (7, 4091)):
        src = x[off:off + n]
        assert torch.equal(mimo.quantize_fp8(src, 0.5), _encode_on_device(src, 0.5))


# ------------------------------------------------------------------ decode

def _fp8_inputs(spec, B, cap, lens, seed=0):
    kv_lens = torch.tensor(lens, dtype=torch.int32)
    q, kn, vn, kc, vc, sinks = synthetic.decode_inputs(spec, B, cap, kv_lens, seed=seed, layer=0, dtype=BF,
                                                       device="cuda")
    sinks = sinks if spec.layer_type == 1 else None
    kc8 = torch.empty(kc.shape, dtype=torch.uint8, device="cuda")
    vc8 = torch.empty(vc.shape, dtype=torch.uint8, device="cuda")
    for b in range(B):
        kc8[b] = _encode_on_device(kc[b], K_SCALE)
        vc8[b] = _encode_on_device(vc[b], V_SCALE)
    del kc, vc
    return kv_lens, q, kn, vn, kc8, vc8, sinks


def _check_fp8(spec, out, q, kn, vn, kc0, vc0, kc, vc, sinks, batches, lens):
    G = spec.num_q_heads // spec.num_kv_heads
    vscale = oracle.v_scale(spec.hidden_size, spec.num_q_heads, spec.v_dim)
    gpu, ref = [], []
    for b in batches:
        L = int(lens[b])
        slot = (L - 1) % spec.window if spec.layer_type == 1 else L - 1
        for kv in range(spec.num_kv_heads):
            hs = slice(kv * G, (kv + 1) * G)
            o, kc2, vc2 = oracle.decode_fp8kv(
                f64(q[b, hs]), f64(kn[b, kv]), f64(vn[b, kv]), kc0[b, :, kv].cpu().numpy(),
                vc0[b, :, kv].cpu().numpy(), L, spec.rotary_dim, spec.theta, spec.layer_type, spec.window,
                1 / math.sqrt(spec.qk_dim), None if sinks is None else f64(sinks[hs]), vscale, K_SCALE, V_SCALE)
            gpu.append(f64(out[b, hs]))
            ref.append(o)
            kg = kc[b, slot, kv].cpu().numpy()
            d = np.abs(_ordinal(kg) - _ordinal(kc2[slot]))
            assert d.max() <= 1 and np.mean(d) < 0.05, f"new key codes b={b} kv={kv}: {int(np.sum(d))} steps off"
            assert np.array_equal(vc[b, slot, kv].cpu().numpy(), vc2[slot])
        others = [s for s in range(kc.shape[1]) if s != slot]
        assert torch.equal(kc[b, others], kc0[b, others]) and torch.equal(vc[b, others], vc0[b, others])
    c = compare(np.concatenate(gpu), np.concatenate(ref))
    assert c.max_abs <= 2e-2 and c.mean_abs <= 2e-3, f"fp8 decode: max {c.max_abs:.3e} mean {c.mean_abs:.3e}"


def _run_fp8(spec, B, cap, lens, seed=0):
    kv_lens, q, kn, vn, kc, vc, sinks = _fp8_inputs(spec, B, cap, lens, seed)
    kc0, vc0 = kc.clone(), vc.clone()
    lay = lib_layer(spec, sinks)
    out = mimo.decode_fp8kv(lay, q, kn, vn, kv_lens.cuda(), kc, vc, K_SCALE, V_SCALE)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    return out, (q, kn, vn, kc0, vc0, kc, vc, sinks)


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_fp8_small_every_output(layer_type):
    """Lengths around the 64-key tiles, the 128-slot ring and the 2048-key
    splits; every output of every sequence."""
    spec = synthetic.mimo_layer(layer_type)
    lens = [1, 2, 63, 64, 65, 127, 128, 129, 1023, 2047, 2048, 2049, 4097, 5000]
    out, (q, kn, vn, kc0, vc0, kc, vc, sinks) = _run_fp8(spec, len(lens), 5000, lens)
    _check_fp8(spec, out, q, kn, vn, kc0, vc0, kc, vc, sinks, range(len(lens)), lens)


@pytest.mark.parametrize("window", [16, 64, 100, 128, 192, 256])
def test_decode_fp8_sliding_windows(window):
    """Sliding layers with rings of one to four 64-key tiles: up to two tiles
    take the slim kernel form (4 CTAs per SM), longer rings the 3-stage one.
    Lengths below, at and past the window; every output."""
    spec = synthetic.mimo_layer(1, window=window)
    lens = sorted({1, 2, window - 1, window, window + 1, 2 * window + 3, 700})
    lens = [L for L in lens if L >= 1]
    out, (q, kn, vn, kc0, vc0, kc, vc, sinks) = _run_fp8(spec, len(lens), window, lens, seed=window)
    _check_fp8(spec, out, q, kn, vn, kc0, vc0, kc, vc, sinks, range(len(lens)), lens)


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_fp8_stale_slots_hold_nan(layer_type):
    """E4M3 NaN codes (0x7F, 0xFF) in every slot a sequence has not written
    yet leave the output equal to the one from finite caches."""
    spec = synthetic.mimo_layer(layer_type)
    lens = [1, 2, 63, 64, 65, 100, 127, 128, 129, 191, 192, 300]
    kv_lens, q, kn, vn, kc, vc, sinks = _fp8_inputs(spec, len(lens), 512, lens, seed=6)
    kc0, vc0 = kc.clone(), vc.clone()
    for b, L in enumerate(lens):
        kc[b, L:] = 0x7F
        vc[b, L:] = 0xFF
    lay = lib_layer(spec, sinks)
    out = mimo.decode_fp8kv(lay, q, kn, vn, kv_lens.cuda(), kc, vc, K_SCALE, V_SCALE)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    assert bool(torch.isfinite(out).all())
    G = spec.num_q_heads // spec.num_kv_heads
    vscale = oracle.v_scale(spec.hidden_size, spec.num_q_heads, spec.v_dim)
    gpu, ref = [], []
    for b, L in enumerate(lens):
        for kv in range(spec.num_kv_heads):
            hs = slice(kv * G, (kv + 1) * G)
            o, _, _ = oracle.decode_fp8kv(
                f64(q[b, hs]), f64(kn[b, kv]), f64(vn[b, kv]), kc0[b, :, kv].cpu().numpy(),
                vc0[b, :, kv].cpu().numpy(), L, spec.rotary_dim, spec.theta, spec.layer_type, spec.window,
                1 / math.sqrt(spec.qk_dim), None if sinks is None else f64(sinks[hs]), vscale, K_SCALE, V_SCALE)
            gpu.append(f64(out[b, hs]))
            ref.append(o)
    c = compare(np.concatenate(gpu), np.concatenate(ref))
    assert c.max_abs <= 2e-2 and c.mean_abs <= 2e-3, f"fp8 decode, NaN codes: max {c.max_abs:.3e} mean {c.mean_abs:.3e}"


def test_decode_fp8_full_size_sampled_batches():
    """Decode workload shape (B64, L ~ U[1024, 32768], cache 32768) with fp8
    caches: one global and one SWA layer, every head of 6 sampled sequences."""
    lens = synthetic.decode_kv_lens(64, 1024, 32768, seed=0).tolist()
    rng = np.random.default_rng(1)
    batches = sorted(set(rng.integers(0, 64, 4).tolist()) | {int(np.argmax(lens)), int(np.argmin(lens))})
    for lt in (0, 1):
        spec = synthetic.mimo_layer(lt)
        out, (q, kn, vn, kc0, vc0, kc, vc, sinks) = _run_fp8(spec, 64, 32768, lens)
        _check_fp8(spec, out, q, kn, vn, kc0, vc0, kc, vc, sinks, batches, lens)
        del kc0, vc0, kc, vc
        torch.cuda.empty_cache()


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_fp8_cuda_graph_replay(layer_type):
    """The fp8 entry point captures into a CUDA graph like the bf16 one: a
    replay on fresh caches writes the direct call's output and caches."""
    spec = synthetic.mimo_layer(layer_type)
    lens = [1, 65, 129, 2049, 5000]
    B = len(lens)
    kv_lens, q, kn, vn, kc, vc, sinks = _fp8_inputs(spec, B, 5000, lens, seed=4)
    kc0, vc0 = kc.clone(), vc.clone()
    lay = lib_layer(spec, sinks)
    lens_dev = kv_lens.cuda()
    out = torch.empty((B, spec.num_q_heads, spec.v_dim), dtype=BF, device="cuda")
    need = mimo.mimo_attn_decode_fp8kv_workspace_size(lay, B, kc.shape[1])
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")

    def call():
        st = mimo.mimo_attn_decode_fp8kv(lay, B, q, kn, vn, lens_dev, kc, vc, kc.shape[1], K_SCALE, V_SCALE, out,
                                         ws, ws.numel(), torch.cuda.current_stream())
        assert st == mimo.OK

    call()
    torch.cuda.synchronize()
    direct, kd, vd = out.clone(), kc.clone(), vc.clone()
    out.zero_()
    kc.copy_(kc0)
    vc.copy_(vc0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    kc.copy_(kc0)
    vc.copy_(vc0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, direct) and torch.equal(kc, kd) and torch.equal(vc, vd)
    _check_fp8(spec, out, q, kn, vn, kc0, vc0, kc, vc, sinks, range(B), lens)


def test_decode_fp8_bad_length_sets_error_and_skips():
    """A kv_lens entry above the capacity sets the device error bit; the
    other sequences still pass parity."""
    spec = synthetic.mimo_layer(0)
    lens = [100, 300]
    kv_lens, q, kn, vn, kc, vc, sinks = _fp8_inputs(spec, 2, 256, lens, seed=6)
    kc0, vc0 = kc.clone(), vc.clone()
    bad = torch.tensor([100, 300], dtype=torch.int32, device="cuda")
    lay = lib_layer(spec, None)
    out = torch.zeros((2, spec.num_q_heads, spec.v_dim), dtype=BF, device="cuda")
    mimo.decode_fp8kv(lay, q, kn, vn, bad, kc, vc, K_SCALE, V_SCALE, out=out)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() & mimo.DEVERR_KV_LEN
    assert torch.equal(kc[1], kc0[1]) and torch.equal(vc[1], vc0[1])
    assert torch.all(out[1] == 0)
    _check_fp8(spec, out, q, kn, vn, kc0, vc0, kc, vc, None, [0], lens)


@pytest.mark.parametrize("layer_type", [0, 1])
def test_decode_fp8_small_groups(layer_type):
    """G = 2 (global) and G = 4 with a sink (sliding): query rows beyond G in
    the 16-row mma tile are zero and must not leak into the output."""
    spec = synthetic.LayerSpec(layer_type, 8 if layer_type == 0 else 16, 4, 192, 128, 64, 128,
                               5e6 if layer_type == 0 else 1e4, 1024, layer_type == 1)
    lens = [1, 17, 128, 129, 700]
    out, (q, kn, vn, kc0, vc0, kc, vc, sinks) = _run_fp8(spec, len(lens), 700, lens, seed=8)
    _check_fp8(spec, out, q, kn, vn, kc0, vc0, kc, vc, sinks, range(len(lens)), lens)
