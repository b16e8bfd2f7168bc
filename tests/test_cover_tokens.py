"""The token selection the Beam-shape GPU parity tests use: from a routing alone it must pick
tokens whose slots fall on every m-tile of every expert (the CUDA path orders each expert's
rows by ascending token id and cuts them into m-tiles of a fixed row count).  Checked here
against a plain enumeration of rows and m-tiles on random and skewed routings."""
import numpy as np
import pytest

from tests import gpu_helpers as H


class _Wl:
    def __init__(self, E):
        self.E = E


class _Case:
    def __init__(self, idx, E):
        self.idx = idx
        self.wl = _Wl(E)


def _routing(T, E, k, rng, skew=0.0):
    p = np.ones(E)
    if skew:
        p = 1.0 / (1.0 + np.arange(E)) ** skew
    p = p / p.sum()
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        idx[t] = np.sort(rng.choice(E, size=k, replace=False, p=p))
    return idx


def _tiles(idx, E, tile_rows):
    """{(e, m): [tokens of m-tile m of expert e, in row order]} by plain enumeration."""
    tiles = {}
    for e in range(E):
        rows = [t for t in range(idx.shape[0]) if e in idx[t]]
        for r, t in enumerate(rows):
            tiles.setdefault((e, r // tile_rows), []).append(t)
    return tiles


@pytest.mark.parametrize("T,E,k,tr,skew", [(300, 16, 4, 8, 0.0), (500, 32, 8, 16, 1.0),
                                           (1000, 8, 2, 128, 0.0), (7, 16, 4, 128, 0.0)])
def test_every_tile_has_its_first_and_last_row_selected(T, E, k, tr, skew):
    rng = np.random.default_rng(T + E)
    idx = _routing(T, E, k, rng, skew)
    picks = set(H.cover_tokens(_Case(idx, E), tile_rows=tr, tile_ends=True))
    for (e, m), toks in _tiles(idx, E, tr).items():
        assert toks[0] in picks and toks[-1] in picks, (e, m)


@pytest.mark.parametrize("T,E,k,tr,skew", [(300, 16, 4, 8, 0.0), (800, 32, 8, 16, 1.5)])
def test_every_tile_has_a_selected_row_and_each_expert_its_ends(T, E, k, tr, skew):
    rng = np.random.default_rng(T * E)
    idx = _routing(T, E, k, rng, skew)
    picks = set(H.cover_tokens(_Case(idx, E), tile_rows=tr, tile_ends=False))
    tiles = _tiles(idx, E, tr)
    for (e, m), toks in tiles.items():
        assert picks.intersection(toks), (e, m)
    for e in range(E):
        rows = [t for t in range(T) if e in idx[t]]
        if rows:
            assert rows[0] in picks and rows[-1] in picks, e
    # far fewer tokens than one per m-tile: each chosen token covers several
    assert len(picks) < len(tiles)
