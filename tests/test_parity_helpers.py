"""Host logic of the GPU parity checks (no GPU): the work-unit cover that
picks which tokens of a full-size case are compared with the oracle."""
import numpy as np
import pytest

from tests._parity import tile_cover


def units_brute_force(idx, E, tile, shared):
    """Every work unit as the set of tokens it holds: bucket e lists the
    (t, k) picks of e in (t, k) order and is cut into pieces of `tile`; the
    shared bucket holds tokens 0..T-1 in pieces of `tile`."""
    T, K = idx.shape
    units = []
    for e in range(E):
        toks = [t for t in range(T) for k in range(K) if idx[t, k] == e]
        for m in range(0, len(toks), tile):
            units.append(set(toks[m:m + tile]))
    if shared:
        for m in range(0, T, tile):
            units.append(set(range(m, min(T, m + tile))))
    return units


@pytest.mark.parametrize("T,E,K,tile,shared,skew", [(300, 16, 2, 32, True, 1.2), (700, 8, 3, 128, True, 0.0),
                                                     (90, 40, 8, 16, False, 2.0), (1, 4, 2, 16, True, 0.0)])
def test_cover_hits_every_unit(T, E, K, tile, shared, skew):
    rng = np.random.default_rng(T + E)
    p = 1.0 / np.arange(1, E + 1) ** skew
    p /= p.sum()
    idx = np.array([rng.choice(E, K, replace=False, p=p) for _ in range(T)], np.int32)
    cover = set(tile_cover(idx, E, tile, shared).tolist())
    for u in units_brute_force(idx, E, tile, shared):
        assert u & cover, "a work unit has no checked token"
    # every bucket spanning several units has its last token checked
    for e in range(E):
        toks = [t for t in range(T) for k in range(K) if idx[t, k] == e]
        if len(toks) > tile:
            assert toks[-1] in cover
    assert T - 1 in cover
