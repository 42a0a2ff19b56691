"""The global-layer kernel's K/V ring protocol, restated on the host.

The kernel (csrc/prefill_ga.cu) streams a CTA's key tiles through a ring of
kRing entries of 16 KB. Key tile j takes entries 5j .. 5j + 2 for its K and
5j + 3, 5j + 4 for its V (mod kRing). Three agents share the ring.

- The TMA producer loads K(0), V(0), K(1), V(1), ... in order. Entry e may
  be refilled once the tile that held entry e - kRing has released that part
  of itself: K after QK_B of that tile, V after PV_B.
- The MMA issuer runs QK_A(0), QK_B(0), then for j = 1 .. n-1: PV_A(j-1)
  (needs P_A(j-1) and V(j-1)), QK_A(j) (K(j)), PV_B(j-1) (P_B(j-1)),
  release V(j-1), QK_B(j), release K(j). Finally PV_A(n-1) and PV_B(n-1).
- Softmax t has P_t(j) once QK_t(j) has run.

The landed and released barriers are two deep: tile j uses barrier j & 1
with parity (j >> 1) & 1. A parity wait is exact only while the barrier is
at most one phase past the waited one, so the model also checks that tile
j + 2 has not reached the same barrier when tile j is waited for. The test
reads kRing and the entries per tile from the kernel source, so changing
either cannot bring in a deadlock or an ambiguous wait unnoticed.
"""
import re
from pathlib import Path

import pytest

SRC = Path(__file__).resolve().parents[1] / "global_attention_partial_b200" / "csrc" / "prefill_ga.cu"


def kernel_constants():
    text = SRC.read_text()
    ring = re.search(r"constexpr int kRing = (\d+);", text)
    per_tile = re.search(r"constexpr int kEntriesPerTile = (\d+);", text)
    assert ring and per_tile, "ring constants not found in prefill_ga.cu"
    return int(ring.group(1)), int(per_tile.group(1))


def issuer_program(n):
    steps = [("wait_K", 0), ("qk", "A", 0), ("qk", "B", 0), ("release_K", 0)]
    for j in range(1, n):
        i = j - 1
        steps += [("wait_P", "A", i), ("wait_V", i), ("pv", "A", i), ("wait_K", j), ("qk", "A", j),
                  ("wait_P", "B", i), ("pv", "B", i), ("release_V", i), ("qk", "B", j), ("release_K", j)]
    steps += [("wait_P", "A", n - 1), ("wait_V", n - 1), ("pv", "A", n - 1),
              ("wait_P", "B", n - 1), ("pv", "B", n - 1), ("release_V", n - 1)]
    return steps


def run(n, ring, per_tile):
    """Returns (completed, ambiguous waits seen)."""
    assert per_tile == 5, "the model's K/V split (3 + 2 entries) follows the kernel"
    loaded_k, loaded_v, rel_k, rel_v = set(), set(), set(), set()
    s_ready, p_ready = set(), set()
    prog = issuer_program(n)
    pc = 0
    prod = 0                       # next producer load: 2 per tile (K then V)
    ambiguous = []

    def free(e):
        if e < ring:
            return True
        jo, part = divmod(e - ring, per_tile)
        done = (rel_k if part < 3 else rel_v)
        # the producer's parity wait on tile jo's release barrier
        if (jo + 2) in done:
            ambiguous.append(("release", jo))
        return jo in done

    progress = True
    while progress:
        progress = False
        while prod < 2 * n:
            j, is_v = divmod(prod, 2)
            first = j * per_tile + (3 if is_v else 0)
            count = 2 if is_v else 3
            if not all(free(first + q) for q in range(count)):
                break
            (loaded_v if is_v else loaded_k).add(j)
            prod += 1
            progress = True
        for t in ("A", "B"):
            for j in range(n):
                if (t, j) in s_ready and (t, j) not in p_ready:
                    p_ready.add((t, j))
                    progress = True
        while pc < len(prog):
            st = prog[pc]
            kind = st[0]
            if kind == "wait_K":
                if (st[1] + 2) in loaded_k:
                    ambiguous.append(("K", st[1]))
                if st[1] not in loaded_k:
                    break
            elif kind == "wait_V":
                if (st[1] + 2) in loaded_v:
                    ambiguous.append(("V", st[1]))
                if st[1] not in loaded_v:
                    break
            elif kind == "wait_P":
                if (st[1], st[2]) not in p_ready:
                    break
            elif kind == "qk":
                s_ready.add((st[1], st[2]))
            elif kind == "release_K":
                rel_k.add(st[1])
            elif kind == "release_V":
                rel_v.add(st[1])
            pc += 1
            progress = True
    return pc == len(prog) and prod == 2 * n, ambiguous


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 8, 17, 64, 255, 256, 300])
def test_every_tile_count_completes_with_exact_waits(n):
    ring, per_tile = kernel_constants()
    done, ambiguous = run(n, ring, per_tile)
    assert done, f"ring of {ring}: {n} key tiles deadlock"
    assert not ambiguous, f"ring of {ring}: parity waits two phases behind: {ambiguous[:3]}"


def test_model_reports_a_ring_smaller_than_one_key_tile():
    """K and V of one tile need 5 entries together: a ring of 4 must stall."""
    assert not run(3, 4, 5)[0]


def test_model_reports_ambiguous_waits_with_a_deeper_ring():
    """With 12 entries the producer can land tile j + 2 on the same two-deep
    barrier before tile j is waited for: the model must flag it (the kernel's
    ring must stay at 10 entries or fewer, or the barriers deepen)."""
    done, ambiguous = run(64, 12, 5)
    assert done and ambiguous
