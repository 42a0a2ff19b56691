"""Small fixed cases of single kernels, for profiling them in isolation.

    python -m global_attention_partial_b200.profile_cases decode   # one global decode layer, bf16 then fp8 cache
    python -m global_attention_partial_b200.profile_cases qkv      # one global-layer QKV projection

Each case runs its calls twice untimed (the second pass is the one a
profiler captures: skip the first pass's launches), then times 10 (decode)
or 5 (qkv) more with CUDA events and prints the mean. Inputs are the
synthetic ones of the benchmarks, sized above the 126 MB L2 but a few GB at
most on the device:
  decode  B64, L ~ U[1024, 32768], cache 32768, 4 KV heads (bf16 cache
          2.7 GB, fp8 copy 1.3 GB); scales 1/16 (keys) and 1/32 (values);
  qkv     B1 S16384, hidden 4096, 13568 features (x 128 MB, W 111 MB),
          with the key/value cache write.
"""
from __future__ import annotations

import sys

import torch

import global_attention_partial_b200 as mimo
from global_attention_partial_b200 import synthetic


def _time(fn, reps: int) -> float:
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def decode_case():
    spec = synthetic.mimo_layer(0)
    lens = synthetic.decode_kv_lens(64, 1024, 32768, seed=0)
    q, kn, vn, kc, vc, _ = synthetic.decode_inputs(spec, 64, 32768, lens, seed=0, layer=0, device="cuda")
    lay = mimo.make_layer(0, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim, spec.v_dim, spec.rotary_dim,
                          spec.window, spec.theta, spec.hidden_size, None)
    kc8 = mimo.quantize_fp8(kc, 1 / 16)
    vc8 = mimo.quantize_fp8(vc, 1 / 32)
    ld = lens.cuda()

    def bf16():
        mimo.decode(lay, q, kn, vn, ld, kc, vc)

    def fp8():
        mimo.decode_fp8kv(lay, q, kn, vn, ld, kc8, vc8, 1 / 16, 1 / 32)

    for _ in range(2):
        bf16()
        fp8()
    torch.cuda.synchronize()
    print(f"decode global layer B64: bf16 cache {_time(bf16, 10):.4f} ms, fp8 cache {_time(fp8, 10):.4f} ms")


def qkv_case():
    spec = synthetic.mimo_layer(0)
    B, S = 1, 16384
    x, w = synthetic.projection_inputs(spec, B, S, seed=0, layer=0, device="cuda")
    lay = mimo.make_layer(0, spec.num_q_heads, spec.num_kv_heads, spec.qk_dim, spec.v_dim, spec.rotary_dim,
                          spec.window, spec.theta, spec.hidden_size, None)
    kc = torch.empty((B, S, spec.num_kv_heads, spec.qk_dim), dtype=torch.bfloat16, device="cuda")
    vc = torch.empty((B, S, spec.num_kv_heads, spec.v_dim), dtype=torch.bfloat16, device="cuda")

    def run():
        mimo.qkv_project(lay, x, w, k_cache=kc, v_cache=vc)

    for _ in range(2):
        run()
    torch.cuda.synchronize()
    ms = _time(run, 5)
    n = spec.num_q_heads * spec.qk_dim + spec.num_kv_heads * (spec.qk_dim + spec.v_dim)
    print(f"qkv projection B1 S16384: {ms:.4f} ms, {2.0 * B * S * n * spec.hidden_size / ms / 1e9:.1f} TFLOP/s")


CASES = {"decode": decode_case, "qkv": qkv_case}

if __name__ == "__main__":
    if len(sys.argv) != 2 or sys.argv[1] not in CASES:
        sys.exit(f"usage: python -m global_attention_partial_b200.profile_cases {{{'|'.join(CASES)}}}")
    mimo.load()
    CASES[sys.argv[1]]()
    if mimo.mimo_attn_get_device_error() != 0:
        sys.exit("device error word set")
