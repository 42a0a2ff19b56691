"""The units bench.py divides by: visible (query, key) pairs, FLOPs and
algorithmic bytes, checked against brute-force counts on small shapes and
against the closed forms of the benchmark's workloads. No GPU."""
import pytest

import bench
from global_attention_partial_b200 import synthetic


def brute_pairs(layer_type, S, W, past=0):
    n = 0
    for i in range(S):
        for j in range(past + S):
            qi = past + i
            if j <= qi and (layer_type == 0 or qi - j < W):
                n += 1
    return n


@pytest.mark.parametrize("S,W", [(1, 4), (5, 4), (4, 4), (37, 8), (100, 128)])
def test_visible_pairs_brute_force(S, W):
    for lt in (0, 1):
        spec = synthetic.LayerSpec(lt, 4, 2, 48, 32, 16, W, 1e4, 256, lt == 1)
        assert bench.visible_pairs(spec, S) == brute_pairs(lt, S, W)


@pytest.mark.parametrize("S,past", [(1, 0), (7, 3), (20, 50), (64, 200)])
def test_chunk_flops_brute_force(S, past):
    for lt in (0, 1):
        spec = synthetic.LayerSpec(lt, 4, 2, 48, 32, 16, 16, 1e4, 256, lt == 1)
        want = 2 * 4 * brute_pairs(lt, S, 16, past) * 2 * (48 + 32)
        assert bench.chunk_flops(spec, 2, S, past) == want


def test_prefill_flops_of_the_workloads():
    """640 FLOP per visible (query, key) pair per head: the SWA config, the
    global config and the 8-layer stack."""
    swa = synthetic.SWA_PREFILL
    assert bench.prefill_flops(swa.layers[0], swa.batch, swa.seq) == pytest.approx(2.114e10, rel=1e-3)
    ga = synthetic.GLOBAL_PREFILL
    assert bench.prefill_flops(ga.layers[0], ga.batch, ga.seq) == pytest.approx(2.749e12, rel=1e-3)
    st = synthetic.HYBRID_PREFILL
    total = sum(bench.prefill_flops(sp, st.batch, st.seq) for sp in st.layers)
    assert total == pytest.approx(1.800e14, rel=1e-3)


def test_decode_bytes_formula():
    """Cache rows read (visible keys x KV heads x (Dqk + Dv) x element size),
    q read, new k/v read in bf16 and written at the cache's element size,
    O written, sinks read; an fp8 cache halves the cache terms only."""
    spec = synthetic.mimo_layer(1)  # 8 KV heads, window 128, sinks
    lens = [1, 100, 128, 5000]
    vis = [1, 100, 128, 128]
    kv = 8 * (192 + 128)
    base = 4 * 64 * 192 * 2 + 4 * kv * 2 + 4 * 64 * 128 * 2 + 64 * 4
    assert bench.decode_bytes(spec, lens) == sum(vis) * kv * 2 + base + 4 * kv * 2
    assert bench.decode_bytes(spec, lens, 1) == sum(vis) * kv * 1 + base + 4 * kv * 1
    g = synthetic.mimo_layer(0)  # no sink, linear cache: every key is visible
    assert bench.decode_bytes(g, [10]) == 10 * 4 * 320 * 2 + 64 * 192 * 2 + 4 * 320 * 2 * 2 + 64 * 128 * 2


def test_qkv_flops():
    for lt, n in ((0, 64 * 192 + 4 * 320), (1, 64 * 192 + 8 * 320)):
        spec = synthetic.mimo_layer(lt)
        assert bench.qkv_flops(spec, 4, 32768) == 2.0 * 4 * 32768 * n * 4096
