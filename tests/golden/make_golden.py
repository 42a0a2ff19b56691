"""Writes tests/golden/oracle_tiny_pair.txt from the fp64 oracle only.

Inputs are closed-form (no RNG) so the fixture is reproducible anywhere:
    q[i, h, d] = sin(0.37 * i + 1.3 * h + 0.11 * d)
    k[i, g, d] = cos(0.23 * i - 0.7 * g + 0.05 * d)
    v[i, g, e] = sin(0.19 * i + 0.9 * g - 0.13 * e)
    sinks[h]   = 0.25 * h - 0.4
The shapes are those of the tiny SWA + global pair (B1 S64 Hq4, Hkv 2 / 1,
qk 48, v 32, rotary 16, window 16, thetas 1e4 / 1e6, hidden 256).
Run: python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

S, HQ, D, DV = 64, 4, 48, 32
LAYERS = [dict(name="swa", layer_type=1, hkv=2, theta=1e4, window=16, sink=True),
          dict(name="global", layer_type=0, hkv=1, theta=1e6, window=0, sink=False)]


def inputs(hkv):
    i = np.arange(S)[:, None, None]
    q = np.sin(0.37 * i + 1.3 * np.arange(HQ)[None, :, None] + 0.11 * np.arange(D)[None, None, :])
    k = np.cos(0.23 * i - 0.7 * np.arange(hkv)[None, :, None] + 0.05 * np.arange(D)[None, None, :])
    v = np.sin(0.19 * i + 0.9 * np.arange(hkv)[None, :, None] - 0.13 * np.arange(DV)[None, None, :])
    sinks = 0.25 * np.arange(HQ) - 0.4
    return q[None], k[None], v[None], sinks


def compute(layer):
    q, k, v, sinks = inputs(layer["hkv"])
    return oracle.prefill_layer(q, k, v, layer_type=layer["layer_type"], num_kv_heads=layer["hkv"],
                                rotary_dim=16, theta=layer["theta"], window=layer["window"],
                                sinks=sinks if layer["sink"] else None, hidden_size=256)[0]


def main():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_pair.txt")
    with open(path, "w") as f:
        f.write("# fp64 oracle output of the tiny SWA + global pair on closed-form inputs;\n")
        f.write("# written by tests/golden/make_golden.py (calls oracle/ only).\n")
        f.write("# columns: layer i h e value\n")
        for layer in LAYERS:
            out = compute(layer)
            for i in range(0, S, 7):
                for h in range(HQ):
                    for e in range(0, DV, 5):
                        f.write(f"{layer['name']} {i} {h} {e} {out[i, h, e]:.17e}\n")


if __name__ == "__main__":
    main()
