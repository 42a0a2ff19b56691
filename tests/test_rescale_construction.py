"""The spike inputs of the rescale parity tests do expose a wrong rescale.

An fp64 emulation of the lazy online softmax runs on the planted inputs
(one global-layer query head, the rows after each jump):

- 128-key tiles;
- a reference maximum that moves only when a tile's maximum exceeds it by
  more than 8 in log2 units.

With the correction factor applied it must equal the oracle. With the
correction dropped (O, the row sum, or both kept at the old scale) it must
miss the bf16 parity bar by a wide margin. Otherwise the GPU test could pass
over a broken rescale. The emulation is test scaffolding: neither the kernels
nor the oracle use it.
"""
import math

import numpy as np
import torch

from global_attention_partial_b200 import synthetic
import oracle
from tests.parity_util import BF16_MAX_ABS, f64
from tests.test_parity_rescale_gpu import BLOCK, PEAK, _plant

THRESHOLD = 8.0


def _lazy_softmax_row(s_log2, vals, correct_o=True, correct_l=True, tile=128):
    """Online softmax of one row over keys in tiles, with the lazy reference."""
    m_ref, l, o = -math.inf, 0.0, np.zeros(vals.shape[1])
    for j0 in range(0, len(s_log2), tile):
        s, vv = s_log2[j0:j0 + tile], vals[j0:j0 + tile]
        mx = float(s.max())
        if mx > m_ref + THRESHOLD or m_ref == -math.inf:
            corr = 0.0 if m_ref == -math.inf else 2.0 ** (m_ref - mx)
            if correct_o:
                o *= corr
            if correct_l:
                l *= corr
            m_ref = mx
        p = 2.0 ** (s - m_ref)
        l += float(p.sum())
        o += p @ vv
    return o / l


def test_a_dropped_correction_breaks_the_bar():
    spec = synthetic.mimo_layer(0)
    S = 4096 + 37
    q, k, v, _ = synthetic.prefill_inputs(spec, 1, S, seed=41, layer=0, dtype=torch.bfloat16)
    _plant(q, k, key_axis=1)
    h, kv = 17, 17 // (spec.num_q_heads // spec.num_kv_heads)
    pos = np.arange(S, dtype=np.float64)
    kr = oracle.rope(f64(k[0, :, kv]), spec.rotary_dim, spec.theta, pos)
    vv = f64(v[0, :, kv])
    rows = [BLOCK[0] + 1, BLOCK[0] + 200, BLOCK[1] + 50, PEAK, PEAK + 300, S - 1]
    qr = oracle.rope(f64(q[0, rows, h]), spec.rotary_dim, spec.theta, pos[rows])
    scale = 1 / math.sqrt(spec.qk_dim)
    exact = oracle.prefill_rows(qr, np.asarray(rows), kr, vv, 0, spec.window, scale, None, 1.0)
    worst = {"right": 0.0, "no_o": 0.0, "no_l": 0.0, "neither": 0.0}
    for n, i in enumerate(rows):
        s = (kr[:i + 1] @ qr[n]) * scale / math.log(2)
        vals = vv[:i + 1]
        variants = {"right": _lazy_softmax_row(s, vals),
                    "no_o": _lazy_softmax_row(s, vals, correct_o=False),
                    "no_l": _lazy_softmax_row(s, vals, correct_l=False),
                    "neither": _lazy_softmax_row(s, vals, correct_o=False, correct_l=False)}
        for name, o in variants.items():
            worst[name] = max(worst[name], float(np.abs(o - exact[n]).max()))
    assert worst["right"] < 1e-9
    for name in ("no_o", "no_l", "neither"):
        assert worst[name] > 10 * BF16_MAX_ABS, (name, worst[name])
