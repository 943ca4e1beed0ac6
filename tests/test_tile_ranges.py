"""The tile-range arithmetic of the prefill and backward kernels, restated and checked by
brute force over many shapes (CPU only). The kernels walk only the tiles their rows can
see; a formula that dropped a tile holding a visible (query, key) pair would lose terms of
the sums, so every visible pair must fall in a walked tile.

Restated from the kernels' index arithmetic (same names):
  forward / dQ CTA of queries q0 .. q0 + BM - 1:  off = Nk - N,
      khi = causal ? min(q0 + BM - 1 + off, Nk - 1) : Nk - 1,
      klo = (causal && W > 0) ? max(0, q0 + off - W + 1) : 0,
      key tiles klo // BN .. khi // BN
  dK/dV CTA of keys k0 .. k0 + KT - 1:
      i_lo = causal ? max(0, k0 - off) : 0,
      i_hi = (causal && W > 0) ? min(N - 1, k0 + KT - 1 - off + W - 1) : N - 1,
      query tiles i_lo // QT .. i_hi // QT (none when i_hi < i_lo)
"""
import itertools

import numpy as np


def visible(N, Nk, causal, W):
    pos = np.arange(N)[:, None] + (Nk - N)
    j = np.arange(Nk)[None, :]
    m = np.ones((N, Nk), dtype=bool)
    if causal:
        m &= j <= pos
        if W > 0:
            m &= j > pos - W
    return m


def key_tiles(q0, BM, BN, N, Nk, causal, W):
    off = Nk - N
    khi = min(q0 + BM - 1 + off, Nk - 1) if causal else Nk - 1
    klo = max(0, q0 + off - W + 1) if (causal and W > 0) else 0
    if khi < klo:
        return range(0)
    return range(klo // BN, khi // BN + 1)


def query_tiles(k0, KT, QT, N, Nk, causal, W):
    off = Nk - N
    i_lo = max(0, k0 - off) if causal else 0
    i_hi = min(N - 1, k0 + KT - 1 - off + W - 1) if (causal and W > 0) else N - 1
    if i_hi < i_lo:
        return range(0)
    return range(i_lo // QT, i_hi // QT + 1)


SHAPES = [(N, Nk) for N in (1, 5, 63, 64, 65, 130, 257) for Nk in (N, N + 1, N + 70, 2 * N + 129)]


def test_query_side_tiles_cover_every_visible_pair():
    """Forward kernels (V1: 128 queries x 64 keys; V2: 128 x 128) and the dQ kernel (64 x 128)."""
    for (N, Nk), causal, W, (BM, BN) in itertools.product(SHAPES, (True, False), (0, 1, 7, 64, 200),
                                                         ((128, 64), (128, 128), (64, 128))):
        if W and not causal:
            continue
        vis = visible(N, Nk, causal, W)
        for q0 in range(0, N, BM):
            tiles = key_tiles(q0, BM, BN, N, Nk, causal, W)
            rows = vis[q0:q0 + BM]
            cols = np.nonzero(rows.any(axis=0))[0]
            for j in cols:
                assert j // BN in tiles, (N, Nk, causal, W, BM, BN, q0, j)


def test_key_side_tiles_cover_every_visible_pair():
    """The dK/dV kernel (128 keys x 64 queries)."""
    for (N, Nk), causal, W in itertools.product(SHAPES, (True, False), (0, 1, 7, 64, 200)):
        if W and not causal:
            continue
        vis = visible(N, Nk, causal, W)
        for k0 in range(0, Nk, 128):
            tiles = query_tiles(k0, 128, 64, N, Nk, causal, W)
            rows = np.nonzero(vis[:, k0:k0 + 128].any(axis=1))[0]
            for i in rows:
                assert i // 64 in tiles, (N, Nk, causal, W, k0, i)
            # and no walked tile lies wholly past the sequence
            for t in tiles:
                assert t * 64 < N


def test_every_row_sees_a_key():
    """The kernels rely on every query row having at least one visible key (its state is
    set by the first visible tile)."""
    for (N, Nk), causal, W in itertools.product(SHAPES, (True, False), (0, 1, 7)):
        if W and not causal:
            continue
        assert visible(N, Nk, causal, W).any(axis=1).all()


def v2_cta_tile(idx, n_qt, units, group, B, causal, QBAND=32):
    """The V2 prefill's CTA order, restated: bands of QBAND query tiles (heaviest first
    when causal), then (batch entry, KV head) groups, then the band's tiles, then the pairs
    of a tile. Returns (query tile, pair, batch entry)."""
    ppg = group // 2
    n_kvh = units // ppg
    per_band = QBAND * ppg * n_kvh * B
    band = idx // per_band
    r_b = idx - band * per_band
    band_len = min(QBAND, n_qt - QBAND * band)
    grp = r_b // (band_len * ppg)
    r_g = r_b - grp * (band_len * ppg)
    qt_i = QBAND * band + r_g // ppg
    return (n_qt - 1 - qt_i if causal else qt_i), (grp % n_kvh) * ppg + r_g % ppg, grp // n_kvh


def test_v2_cta_order_covers_every_tile_once():
    """The grid has n_qt * units * B CTAs; the order must hand out each (query tile, pair,
    batch entry) exactly once, bands of partial length included, and keep the pairs of a
    CTA's KV head together."""
    for n_qt, Hq, Hkv, B in ((512, 64, 8, 1), (128, 64, 8, 1), (3, 16, 2, 2), (1, 8, 4, 3),
                             (33, 4, 2, 1), (65, 32, 2, 2), (7, 64, 2, 1), (64, 8, 1, 2)):
        units, group = Hq // 2, Hq // Hkv
        for causal in (True, False):
            got = [v2_cta_tile(i, n_qt, units, group, B, causal) for i in range(n_qt * units * B)]
            assert len(set(got)) == len(got) == n_qt * units * B
            assert all(0 <= t < n_qt and 0 <= u < units and 0 <= b < B for t, u, b in got)
            if causal:  # the last CTAs take the lightest band
                assert max(t for t, _, _ in got[-units * B:]) < 32
