"""The sliding-window prefill kernel's K/V ring protocol, restated on the host.

The kernel (csrc/prefill_swa.cu) streams each CTA's tiles' 16-key blocks
through a ring of kRing entries. Three agents share it:

- the K/V producer loads the tiles' new blocks in order; an entry's slot can
  be refilled once both MMA issuers have committed the entry it held;
- issuer t serves the tiles n = t, t + 2, ...: before waiting for a tile it
  commits every entry below the tile's span, then waits for the span's
  entries (and for the epilogue of its tile n - 2), and after the tile's PV
  commits every entry below the span of its next tile (or all, after its
  last one).

The workers are taken to progress whenever their inputs are ready; they hold
no ring entries. This model checks that every placement of a CTA's tile range
completes with the kernel's ring size (no agent waits on another forever), and
that it does report the deadlock the protocol had before issuers committed the
entries below a span ahead of waiting for it. The kernel's own bounded waits
turn such a deadlock into the device timeout bit; this test keeps a change of
the ring size or the commit order from reintroducing one.
"""
import re
from pathlib import Path

import pytest

KEY_BLOCK = 16
SRC = Path(__file__).resolve().parents[1] / "global_attention_partial_b200" / "csrc" / "prefill_swa.cu"


def kernel_ring_entries() -> int:
    m = re.search(r"constexpr int kRing = (\d+);", SRC.read_text())
    assert m, "kRing not found in prefill_swa.cu"
    return int(m.group(1))


def tiles(S, P, W, key_off, Hkv, B):
    """(run, first block, last block) of every tile in the kernel's order."""
    num_p = (S + P - 1) // P
    out = []
    for run in range(B * Hkv):
        for pt in range(num_p):
            p0 = pt * P
            k_lo = p0 + key_off - W + 1
            first = k_lo // KEY_BLOCK if k_lo > 0 else 0
            last = (p0 + key_off + P - 1) // KEY_BLOCK
            out.append((run, first, last))
    return out


def ring_cursor(tl):
    """Entry numbers: a run's blocks take consecutive entries in load order."""
    run, last_block, base, nxt = -1, -1, 0, 0
    res = []
    for r, first, last in tl:
        if r != run:
            run, base, first_new = r, nxt - first, first
        else:
            first_new = last_block + 1
        nxt += last - first_new + 1
        last_block = last
        res.append({"e0": base + first, "nb": last - first + 1,
                    "new": list(range(base + first_new, base + last + 1)), "next_entry": nxt})
    return res


def completes(tl, ring, commit_below_before_wait=True) -> bool:
    n = len(tl)
    info = ring_cursor(tl)
    loads = [e for t in info for e in t["new"]]
    committed = (set(), set())
    loaded = set()
    prod = 0
    nxt = [0, 1]          # next tile of each issuer
    freed = [0, 0]        # entries [0, freed) committed by each issuer
    done_tiles = set()    # tiles whose O is ready (their epilogue can run)
    progress = True
    while progress:
        progress = False
        while prod < len(loads):
            prev = loads[prod] - ring
            if prev >= 0 and not (prev in committed[0] and prev in committed[1]):
                break
            loaded.add(loads[prod])
            prod += 1
            progress = True
        for t in (0, 1):
            while nxt[t] < n:
                m = nxt[t]
                e0, nb = info[m]["e0"], info[m]["nb"]
                if commit_below_before_wait:
                    while freed[t] < e0:
                        committed[t].add(freed[t])
                        freed[t] += 1
                if m >= 2 and (m - 2) not in done_tiles:
                    break
                if not all(e in loaded for e in range(e0, e0 + nb)):
                    break
                done_tiles.add(m)
                keep = info[m + 2]["e0"] if m + 2 < n else info[n - 1]["next_entry"]
                while freed[t] < keep:
                    committed[t].add(freed[t])
                    freed[t] += 1
                nxt[t] += 2
                progress = True
    return prod == len(loads) and nxt[0] >= n and nxt[1] >= n


def placements(S, key_off, B=2, Hkv=8, P=16, W=128):
    tl = tiles(S, P, W, key_off, Hkv, B)
    for start in range(len(tl)):
        for length in (1, 2, 3, 5, 8, 17, 40):
            seg = tl[start:start + length]
            if seg:
                yield start, length, seg


# plain prefills (key offset 0) and prefills continuing a cache (the key
# window starts 128 keys before the chunk), lengths around the tile and run
# sizes
CASES = [(100, 0), (160, 0), (300, 0), (256, 128), (600, 128)]


@pytest.mark.parametrize("S,key_off", CASES)
def test_every_cta_placement_completes_with_the_kernel_ring(S, key_off):
    ring = kernel_ring_entries()
    stuck = [(start, length) for start, length, seg in placements(S, key_off) if not completes(seg, ring)]
    assert not stuck, f"ring of {ring}: {len(stuck)} placements deadlock, e.g. {stuck[:3]}"


def test_model_reports_the_deadlock_of_late_commits():
    """Without the commits below a span ahead of the wait, a CTA whose first
    two tiles fall in different runs needs 18 entries: the model must see it
    stall (at the ring size of the kernel when that deadlock was found)."""
    stuck = [1 for _, _, seg in placements(256, 128) if not completes(seg, 12, commit_below_before_wait=False)]
    assert stuck


def test_model_reports_a_ring_smaller_than_one_span():
    """A tile spans up to 9 blocks: a ring of 8 must deadlock somewhere."""
    assert any(not completes(seg, 8) for _, _, seg in placements(160, 0))
