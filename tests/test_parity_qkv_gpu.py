"""GPU parity of the fused QKV projection (tcgen05 GEMM with the RoPE and
cache-write epilogue) against the fp64 oracle.

Inputs: x ~ N(0,1) and w_qkv ~ N(0, 1/hidden) in bf16, so the projections are
near N(0,1) and the bf16 bar of the layer applies (max-abs 2e-2, mean-abs
2e-3: a bf16 rounding of |y| <= 8 is at most 8 * 2^-9 = 1.6e-2; the fp32
accumulation over 4096 exact bf16 products adds ~1e-6)."""
import numpy as np
import pytest
import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic
import oracle
from tests.parity_util import compare, f64, lib_layer

pytestmark = pytest.mark.gpu

BF = torch.bfloat16


def _check(c, what):
    assert c.max_abs <= 2e-2 and c.mean_abs <= 2e-3, f"{what}: max {c.max_abs:.3e} mean {c.mean_abs:.3e} over {c.n}"


def _oracle(spec, x, w, positions, rotary):
    return oracle.qkv_project(f64(x), f64(w), positions, num_q_heads=spec.num_q_heads,
                              num_kv_heads=spec.num_kv_heads, qk_dim=spec.qk_dim, v_dim=spec.v_dim,
                              rotary_dim=rotary, theta=spec.theta)


def _run_and_check(spec, B, S, past, cap, tokens=None, rotary=None, seed=0):
    """Projects B x S tokens after `past` cached positions per sequence, with
    caches, and checks q, k, v and every cache slot against the oracle
    (tokens: the sequence indices to compare, default all)."""
    rotary = spec.rotary_dim if rotary is None else rotary
    x, w = synthetic.projection_inputs(spec, B, S, seed=seed, layer=0, device="cuda")
    lay = lib_layer(spec, None, rotary=rotary)
    Hkv = spec.num_kv_heads
    ring = spec.layer_type == 1
    slots = spec.window if ring else cap
    kc = synthetic.normal((B, slots, Hkv, spec.qk_dim), seed=seed, tensor_id=900, device="cuda")
    vc = synthetic.normal((B, slots, Hkv, spec.v_dim), seed=seed, tensor_id=901, device="cuda")
    kc0, vc0 = kc.clone(), vc.clone()
    past_t = torch.tensor(past, dtype=torch.int32, device="cuda")
    q, k, v = mimo.qkv_project(lay, x, w, past_t, max(past), kc, vc)
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() == 0
    tokens = range(S) if tokens is None else tokens
    gq, rq, gk, rk, gv, rv, gc, rc = [], [], [], [], [], [], [], []
    toks = np.asarray(list(tokens))
    idx = torch.as_tensor(toks, device="cuda")
    for b in range(B):
        pos = past[b] + toks
        oq, ok, ov = _oracle(spec, x[b, idx], w, pos, rotary)
        gq.append(f64(q[b, idx]).ravel())
        rq.append(oq.ravel())
        gk.append(f64(k[b, idx]).ravel())
        rk.append(ok.ravel())
        gv.append(f64(v[b, idx]).ravel())
        rv.append(ov.ravel())
        # cache slots: the compared tokens' slots are predicted (on a ring
        # only the chunk's last `window` tokens are stored); with every token
        # compared, all other slots must be untouched
        owners = {}
        for tk, p in zip(toks, pos):
            if ring and tk < S - spec.window:
                continue
            owners[int(p) % spec.window if ring else int(p)] = (tk, p)
        for sl, (tk, p) in owners.items():
            i = int(np.nonzero(toks == tk)[0][0])
            gc.append(f64(kc[b, sl]).ravel()); rc.append(ok[i].ravel())
            gc.append(f64(vc[b, sl]).ravel()); rc.append(ov[i].ravel())
        if len(toks) == S:
            others = [sl for sl in range(slots) if sl not in owners]
            assert torch.equal(kc[b, others], kc0[b, others]) and torch.equal(vc[b, others], vc0[b, others])
    _check(compare(np.concatenate(gq), np.concatenate(rq)), "q")
    _check(compare(np.concatenate(gk), np.concatenate(rk)), "k")
    _check(compare(np.concatenate(gv), np.concatenate(rv)), "v")
    _check(compare(np.concatenate(gc), np.concatenate(rc)), "caches")


@pytest.mark.parametrize("layer_type", [0, 1])
def test_qkv_project_mimo_layer_every_output(layer_type):
    """MiMo-shaped layer (hidden 4096; 53 / 58 feature tiles of 256), two
    sequences of 300 tokens (a ragged token tile) after 0 and 777 cached
    positions; the ring sees more tokens than it has slots."""
    spec = synthetic.mimo_layer(layer_type)
    _run_and_check(spec, 2, 300, [0, 777], cap=1100)


@pytest.mark.parametrize("rotary", [64, 0])
def test_qkv_project_ragged_feature_tile(rotary):
    """Hq 4, Hkv 2: 1408 features = 5.5 tiles of 256; 130 tokens = one full
    and one 2-row token tile; hidden 256 (4 k-blocks); with and without RoPE."""
    spec = synthetic.LayerSpec(0, 4, 2, 192, 128, 64, 128, 5e6, 256, False)
    _run_and_check(spec, 1, 130, [5], cap=200, rotary=rotary)


def test_qkv_project_full_size_sampled_tokens():
    """Global layer at the stack's prefill size (B4 S32768, cache 32768):
    every output feature of 48 sampled tokens per sequence."""
    spec = synthetic.mimo_layer(0)
    rng = np.random.default_rng(3)
    toks = sorted(set(rng.integers(0, 32768, 44).tolist()) | {0, 127, 128, 32767})
    _run_and_check(spec, 4, 32768, [0, 0, 0, 0], cap=32768, tokens=toks)


@pytest.mark.parametrize("layer_type", [0, 1])
def test_projection_then_attention(layer_type):
    """The projection's rotated outputs through mimo_attn_prefill with
    rotary_dim 0 give the layer: the oracle's attention (with RoPE) over its
    own unrotated projections x W^T."""
    spec = synthetic.mimo_layer(layer_type)
    B, S = 1, 512
    x, w = synthetic.projection_inputs(spec, B, S, seed=5, layer=1, device="cuda")
    sinks = synthetic.normal((spec.num_q_heads,), seed=5, tensor_id=77, dtype=torch.float32, device="cuda") \
        if layer_type == 1 else None
    q, k, v = mimo.qkv_project(lib_layer(spec, None), x, w)
    out = mimo.prefill(lib_layer(spec, sinks, rotary=0), q, k, v)
    torch.cuda.synchronize()
    y = f64(x[0]) @ f64(w).T
    nq, nk = spec.num_q_heads * spec.qk_dim, spec.num_kv_heads * spec.qk_dim
    q0 = y[:, :nq].reshape(B, S, spec.num_q_heads, spec.qk_dim)
    k0 = y[:, nq:nq + nk].reshape(B, S, spec.num_kv_heads, spec.qk_dim)
    v0 = y[:, nq + nk:].reshape(B, S, spec.num_kv_heads, spec.v_dim)
    rows = [0, 1, 127, 128, 129, 300, 511]
    ref = oracle.prefill_layer(q0, k0, v0, layer_type=layer_type, num_kv_heads=spec.num_kv_heads,
                               rotary_dim=spec.rotary_dim, theta=spec.theta, window=spec.window,
                               sinks=None if sinks is None else f64(sinks), hidden_size=spec.hidden_size, rows=rows)
    _check(compare(f64(out[:, rows]).ravel(), ref[:, rows].ravel()), "projection -> attention")


def test_qkv_project_bad_past_sets_error_and_skips():
    spec = synthetic.mimo_layer(0)
    x, w = synthetic.projection_inputs(spec, 2, 64, seed=2, layer=0, device="cuda")
    lay = lib_layer(spec, None)
    past = torch.tensor([3, 50], dtype=torch.int32, device="cuda")  # 50 > max_past_len 10
    q = torch.zeros((2, 64, spec.num_q_heads, spec.qk_dim), dtype=BF, device="cuda")
    need = mimo.mimo_attn_qkv_project_workspace_size(lay, 2, 64, 10)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    st = mimo.mimo_attn_qkv_project(lay, 2, 64, x, w, past, 10, q, None, None, None, None, 0, ws, ws.numel(),
                                    torch.cuda.current_stream())
    assert st == mimo.OK
    torch.cuda.synchronize()
    assert mimo.mimo_attn_get_device_error() & mimo.DEVERR_KV_LEN
    assert torch.all(q[1] == 0)
    oq, _, _ = _oracle(spec, x[0], w, 3 + np.arange(64), spec.rotary_dim)
    _check(compare(f64(q[0]).ravel(), oq.ravel()), "q of the valid sequence")


def test_qkv_project_one_k_block_short_ring():
    """hidden 64 (a single k-block), three sequences of 40 tokens on a
    sliding layer whose 128-slot ring is only partly written."""
    spec = synthetic.LayerSpec(1, 8, 2, 192, 128, 64, 128, 1e4, 64, True)
    _run_and_check(spec, 3, 40, [0, 100, 7], cap=128)
