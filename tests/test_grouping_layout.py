"""The decode path's layout of gathered token rows with fixed first tiles, as an
index model on the CPU (no GPU): the layer entry writes the row of assignment
position p of expert e (rank r = p - off[e] in its segment) to
  r < 64:  64 e + r            (the expert's first tile, fixed rows)
  r >= 64: 64 x 64 + p         (further tiles, after the fixed rows)
and the expert kernel reads tile nb of expert e from rows
  nb = 0:  64 e ..             (known before the offsets)
  nb >= 1: 64 x 64 + off[e] + 64 nb ..
Every assignment must land in exactly one tile slot, each tile's rows must be
the ones its expert's assignments were written to, in segment order, and every
row must lie inside the 6T + 64 x 64 rows the workspace holds."""
import numpy as np
import pytest

E, K, NT = 64, 6, 64


def _stable_positions(idx):
    """Offsets and the stable position of every assignment (token-major order
    within each expert's segment)."""
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=E)
    off = np.concatenate([[0], np.cumsum(counts)])
    pos = np.empty(flat.size, dtype=np.int64)
    seen = np.zeros(E, dtype=np.int64)
    for a, e in enumerate(flat):
        pos[a] = off[e] + seen[e]
        seen[e] += 1
    return counts, off, pos


def _entry_row(e, p, off):
    r = p - off[e]
    return e * NT + r if r < NT else E * NT + p


def _tile_rows(e, nb, counts, off):
    n = max(0, min(NT, counts[e] - nb * NT))
    first = e * NT if nb == 0 else E * NT + off[e] + nb * NT
    return first, n


@pytest.mark.parametrize("T,skew", [(64, False), (128, False), (296, False), (128, True), (295, True)])
def test_fixed_first_tiles_cover_every_assignment_once(T, skew):
    g = np.random.default_rng(T + 7 * skew)
    if skew:  # most assignments on the first experts: several tiles per expert
        p = 1.0 / np.arange(1, E + 1) ** 2
        p /= p.sum()
        idx = np.stack([g.choice(E, K, replace=False, p=p) for _ in range(T)])
    else:
        idx = np.stack([g.choice(E, K, replace=False) for _ in range(T)])
    counts, off, pos = _stable_positions(idx)
    N = T * K
    rows_total = N + E * NT
    written = {}
    flat = idx.reshape(-1)
    for a in range(N):
        row = _entry_row(flat[a], pos[a], off)
        assert 0 <= row < rows_total
        assert row not in written, "two assignments on one gathered row"
        written[row] = a
    read = {}
    for e in range(E):
        n_tiles = max(1, -(-counts[e] // NT))
        for nb in range(n_tiles):
            first, n = _tile_rows(e, nb, counts, off)
            for j in range(n):
                row = first + j
                assert 0 <= row < rows_total
                assert row in written, f"expert {e} tile {nb} reads row {row} that no assignment wrote"
                a = written[row]
                assert flat[a] == e and pos[a] == off[e] + nb * NT + j, "tile rows out of segment order"
                read[row] = (e, nb, j)
    assert set(read) == set(written), "an assignment no tile reads"
    if skew and T >= 128:
        assert (counts > NT).any()  # the further-tile rows are exercised
