"""The split plan's addressing, checked on the CPU.

The attend kernels split the concatenated (b, h, block) list into equal
contiguous ranges, one per worker (a CTA, or a warp pair of the decode
kernel); a worker that covers part of a (b, h) writes its partial state to
slot worker + b * H + h, and the merge reads slots c + b * H + h for the
workers c_first..c_last its own arithmetic finds for that (b, h).  This test
restates that arithmetic (the block prefix over the lengths, the equal split,
the slot formula) and checks, for random length mixes and worker counts,
that every (b, h) with keys is covered exactly, that the workers writing a
(b, h) are exactly the ones the merge reads, that no two (worker, (b, h))
pairs share a slot, that every slot fits the workspace
(workers + B * H slots), and that the window's slots (after those) overlap
none of them.
"""

import numpy as np
import pytest


def seq_blocks(length, n_cap, bt):
    length = min(max(length, 0), n_cap)
    return (length + bt - 1) // bt


def plan(lengths, H, n_cap, bt, workers):
    pre = np.concatenate([[0], np.cumsum([seq_blocks(int(n), n_cap, bt) for n in lengths])])
    T = H * int(pre[-1])
    P = -(-T // workers) if T else 1
    return pre, T, P


def worker_segments(pre, H, T, P, workers):
    """(worker, b, h, first block, end block) for every piece a worker covers."""
    out = []
    B = len(pre) - 1
    for c in range(workers):
        g0, g1 = c * P, min((c + 1) * P, T)
        g = g0
        while g < g1:
            b = int(np.searchsorted(pre * H, g, side="right")) - 1
            while pre[b + 1] == pre[b]:
                b += 1
            nb = int(pre[b + 1] - pre[b])
            off = g - H * int(pre[b])
            h, j = off // nb, off % nb
            je = min(nb, j + (g1 - g))
            out.append((c, b, h, j, je))
            g += je - j
    return out


@pytest.mark.parametrize("seed", range(12))
def test_slots_are_unique_and_match_the_merge(seed):
    rng = np.random.default_rng(seed)
    B, H = int(rng.integers(1, 9)), int(rng.integers(1, 5))
    n_cap, bt = int(rng.choice([64, 700, 4096])), int(rng.choice([32, 128]))
    lengths = rng.integers(0, n_cap + 1, size=B)
    lengths[rng.random(B) < 0.2] = 0
    workers = int(rng.choice([1, 3, 7, 148, 1184]))
    pre, T, P = plan(lengths, H, n_cap, bt, workers)
    pieces = worker_segments(pre, H, T, P, workers)

    covered = {}
    for c, b, h, j, je in pieces:
        covered.setdefault((b, h), []).append((j, je, c))
    slots = {}
    for (b, h), parts in covered.items():
        parts.sort()
        nb = int(pre[b + 1] - pre[b])
        assert parts[0][0] == 0 and parts[-1][1] == nb
        for (a0, a1, _), (b0, b1, _) in zip(parts, parts[1:]):
            assert a1 == b0                                  # contiguous, no overlap
        # the merge's own arithmetic finds the same workers
        S = H * int(pre[b]) + h * nb
        E = S + nb
        c_first, c_last = S // P, (E - 1) // P
        assert [c for _, _, c in parts] == list(range(c_first, c_last + 1))
        for _, _, c in parts:
            slot = c + b * H + h
            assert slot not in slots, f"slot {slot} of ({b}, {h}) worker {c} already used by {slots[slot]}"
            slots[slot] = ((b, h), c)
    # every (b, h) with keys is covered, and nothing else
    with_keys = {(b, h) for b in range(B) for h in range(H) if seq_blocks(int(lengths[b]), n_cap, bt) > 0}
    assert set(covered) == with_keys
    n_slots = workers + B * H
    assert all(s < n_slots for s in slots)
    window = {n_slots + b * H + h for b in range(B) for h in range(H)}
    assert not window & set(slots)
