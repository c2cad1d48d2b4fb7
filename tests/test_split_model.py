"""Properties of the split-KV work division the tensor-core decode uses, on a plain model of it:

All (query row, page) units are numbered row by row; cluster c of P takes units
[c*U/P, (c+1)*U/P).  The part of row r that cluster c holds writes its partial result to slot
c + r; a row's slots are [c_first + r, c_last + r + 1), and a cluster inside that range that
holds none of the row's units marks its slot empty.  The workspace holds P + rows slots.

The model checks, over many batches: every unit is assigned to exactly one cluster; no two
(row, cluster) parts share a slot; every slot index is below P + rows; each row's slot range
is exactly its parts' slots plus the marked-empty ones; and a cluster's parts are consecutive
rows (skipping rows without pages).  These are the facts the kernel's combine step relies on;
the GPU tests check the kernel itself.
"""
import numpy as np
import pytest


def _split(pages, P):
    U = int(sum(pages))
    start = np.concatenate([[0], np.cumsum(pages)]).astype(np.int64)
    cl = lambda c: c * U // P
    parts = {}  # (row, cluster) -> units
    for c in range(P):
        a, b = cl(c), cl(c + 1)
        for r in range(len(pages)):
            lo, hi = max(a, start[r]), min(b, start[r + 1])
            if lo < hi:
                parts[(r, c)] = (lo, hi)
    return U, start, parts, cl


@pytest.mark.parametrize("seed", range(40))
def test_split_slots_are_injective_and_bounded(seed):
    rng = np.random.default_rng(seed)
    rows = int(rng.integers(1, 300))
    P = int(rng.integers(1, 80))
    # row lengths in pages, including empty rows and a mix of short and long rows
    pages = rng.choice([0, 1, 2, 5, 64, 200, 2048], size=rows, p=[.05, .25, .2, .2, .2, .07, .03])
    U, start, parts, cl = _split(pages, P)

    covered = np.zeros(U, dtype=np.int64)
    for (r, c), (lo, hi) in parts.items():
        covered[lo:hi] += 1
    assert np.all(covered == 1)

    slots = [r + c for (r, c) in parts]
    assert len(set(slots)) == len(slots)
    assert all(0 <= s < P + rows for s in slots)

    for r in range(rows):
        held = sorted(c for (rr, c) in parts if rr == r)
        if pages[r] == 0:
            assert not held
            continue
        first, last = held[0], held[-1]
        # the row's slot range; clusters inside it without units of the row are the empty ones
        empties = [c for c in range(first, last + 1) if (r, c) not in parts]
        for c in empties:  # only clusters with no units at all can sit inside a row's range
            assert cl(c) == cl(c + 1)
        # an empty cluster's slot c + r is not used by any other (row, cluster) part
        for c in empties:
            assert all(rr + cc != c + r for (rr, cc) in parts)

    # the kernel's rule: a cluster without units marks slot c + r empty, r = the row holding unit
    # c*U/P; that slot must never be a real part's (it may lie outside the row's range, where the
    # combine step does not read it)
    real = set(slots)
    for c in range(P):
        u = cl(c)
        if cl(c + 1) == u and u < U:
            r = int(np.searchsorted(start, u, side="right") - 1)
            assert start[r] <= u < start[r + 1]
            assert c + r not in real

    for c in range(P):  # a cluster's parts are consecutive rows, skipping rows without pages
        rws = sorted(r for (r, cc) in parts if cc == c)
        if rws:
            assert rws == [r for r in range(rws[0], rws[-1] + 1) if pages[r] > 0]


def test_more_clusters_than_units_leaves_clusters_empty():
    U, start, parts, cl = _split([1, 1, 1], 10)
    assert sorted(parts) == [(0, 3), (1, 6), (2, 9)]
    assert len({r + c for (r, c) in parts}) == 3
