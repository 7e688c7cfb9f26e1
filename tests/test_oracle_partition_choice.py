"""Pins of the oracle's choice among the candidate partitions of a frame
(DraftAttention2 Sec. 3.3 "Fused quantization and reordering": each region is
a spatially contiguous patch of one frame; App. C.2, cut off after the region
count R_f = ceil(Hv Wv / C)).

The reading the oracle implements: for every band count nb = 1..Hv the rows
are split into balanced bands (taller first) that are walked as a
boustrophedon, column by column inside a band; the walk is cut into R_f
chunks of balanced size; among the candidates whose regions are all
4-connected the smallest total perimeter wins, ties to the smaller nb.

The candidates are enumerated here independently of the oracle (numpy walk,
scipy connected-component labelling, numpy edge count), and the expected
winners and perimeters of the four frame geometries of the workloads are
literal values derived by hand from that enumeration:
16x16 -> nb 2, perimeter 128 (8x8 patches); 30x52 -> nb 4, 866;
60x90 -> nb 8, 2752 (8-row bands); 45x80 -> nb 5, 1898.
Two constructed shapes have a tie between different partitions, which the
smaller band count must win.
"""
import numpy as np
import pytest
from scipy import ndimage

from oracle import oracle as O


def _walk(Hv, Wv, nb):
    base, rem = divmod(Hv, nb)
    cells, r0 = [], 0
    for i in range(nb):
        h = base + (1 if i < rem else 0)
        xs = range(Wv) if i % 2 == 0 else range(Wv - 1, -1, -1)
        for k, x in enumerate(xs):
            ys = range(r0, r0 + h) if k % 2 == 0 else range(r0 + h - 1, r0 - 1, -1)
            cells.extend(y * Wv + x for y in ys)
        r0 += h
    return np.array(cells)


def _candidate(Hv, Wv, nb, C=64):
    n = Hv * Wv
    Rf = -(-n // C)
    sizes = [n // Rf + (1 if j < n % Rf else 0) for j in range(Rf)]
    w = _walk(Hv, Wv, nb)
    reg = np.empty(n, np.int64)
    slot = np.empty(n, np.int64)
    reg[w] = np.repeat(np.arange(Rf), sizes)
    slot[w] = np.concatenate([np.arange(s) for s in sizes])
    g = reg.reshape(Hv, Wv)
    connected = all(ndimage.label(g == j)[1] == 1 for j in range(Rf))
    # sum of the region perimeters: frame border once, every internal cut twice
    perim = 2 * (Hv + Wv) + 2 * int((g[1:] != g[:-1]).sum()) + 2 * int((g[:, 1:] != g[:, :-1]).sum())
    return reg, slot, connected, perim


def _winners(Hv, Wv):
    cands = {nb: _candidate(Hv, Wv, nb) for nb in range(1, Hv + 1)}
    pool = {nb: c for nb, c in cands.items() if c[2]} or cands
    best = min(c[3] for c in pool.values())
    return sorted(nb for nb, c in pool.items() if c[3] == best), best, cands


@pytest.mark.parametrize("Hv,Wv,nb,perim", [(16, 16, 2, 128), (30, 52, 4, 866), (60, 90, 8, 2752),
                                             (45, 80, 5, 1898)])
def test_workload_frames_pick_expected_band_count(Hv, Wv, nb, perim):
    nbs, best, cands = _winners(Hv, Wv)
    assert nbs == [nb] and best == perim
    reg, slot, _ = O.partition(Hv, Wv)
    want_reg, want_slot, connected, p = cands[nb]
    assert connected and p == perim
    assert np.array_equal(reg, want_reg)
    assert np.array_equal(slot, want_slot)


@pytest.mark.parametrize("Hv,Wv,tied", [(10, 14, [1, 2]), (13, 16, [2, 3])])
def test_tie_goes_to_smaller_band_count(Hv, Wv, tied):
    nbs, _, cands = _winners(Hv, Wv)
    assert nbs == tied
    # the tied candidates are different partitions, so the rule decides
    assert not np.array_equal(cands[tied[0]][0], cands[tied[1]][0])
    reg, slot, _ = O.partition(Hv, Wv)
    assert np.array_equal(reg, cands[tied[0]][0])
    assert np.array_equal(slot, cands[tied[0]][1])
