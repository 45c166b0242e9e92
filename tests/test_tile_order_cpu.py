"""The integer GEMM's tile order visits every output tile exactly once.

The persistent GEMM (csrc/qs_gemm.cuh, ``Problem::tile_origin``) gives each
CTA pair the linear tile indices t = pair, pair + pairs, ... < num_tiles and
maps t to a tile origin.  Two orders exist: n-fastest (band = 0) and, for the
8-bit x 8-bit form, bands of ``band`` N-tiles with M advancing inside a band
and a narrower last band when the band width does not divide the N-tile
count.  This restates that map and checks, over a range of grid shapes, that
it is a bijection from [0, num_tiles) onto the m_tiles x n_tiles grid, and
that the union of every pair's share is the whole grid for several pair
counts.  No GPU is involved.
"""

import itertools

import pytest

BAND_N = 18  # kBandN of the 8x8 instantiation (tiles of 256 x 256)


def tile_origin(t, m_tiles, n_tiles, band):
    """(m, n) tile coordinates of linear index t (the kernel's map, in tiles)."""
    if band > 0:
        per_band = band * m_tiles
        g, r = divmod(t, per_band)
        gn = min(band, n_tiles - g * band)
        return r // gn, g * band + r % gn
    return t // n_tiles, t % n_tiles


# 18 and 9: the integer GEMM's bands of 256- and 512-column tiles; 36 and 18
# are also the SD4 GEMM's bands of 192- and 384-column tiles (its tile_origin
# is the same map with the band given per form)
@pytest.mark.parametrize("band", [0, BAND_N, 9, 36, 1])
def test_tile_order_is_a_bijection(band):
    for m_tiles, n_tiles in itertools.product(range(1, 40), range(1, 80)):
        seen = set()
        for t in range(m_tiles * n_tiles):
            m, n = tile_origin(t, m_tiles, n_tiles, band)
            assert 0 <= m < m_tiles and 0 <= n < n_tiles, (m_tiles, n_tiles, t)
            seen.add((m, n))
        assert len(seen) == m_tiles * n_tiles, (m_tiles, n_tiles)


def test_tile_order_at_large_grids():
    # the Wan FFN W8A8 grid (128 x 54 tiles) and the chain's shapes, plus
    # grids with a narrow last band (20 N-tiles = 18 + 2, 37 = 2 x 18 + 1)
    for m_tiles, n_tiles in [(128, 54), (128, 60), (128, 20), (2, 20), (2, 37), (129, 79),
                             (32, 36)]:
        seen = {tile_origin(t, m_tiles, n_tiles, BAND_N) for t in range(m_tiles * n_tiles)}
        assert len(seen) == m_tiles * n_tiles


@pytest.mark.parametrize("pairs", [1, 7, 74])
def test_every_pair_share_covers_the_grid_once(pairs):
    for m_tiles, n_tiles in [(16, 20), (2, 20), (16, 10), (128, 54), (128, 27), (3, 1)]:
        num = m_tiles * n_tiles
        count = {}
        for pair in range(pairs):
            for t in range(pair, num, pairs):
                key = tile_origin(t, m_tiles, n_tiles, BAND_N)
                count[key] = count.get(key, 0) + 1
        assert len(count) == num and set(count.values()) == {1}


def test_banded_order_keeps_a_band_of_columns_together():
    # inside a band, consecutive indices stay within the band's N-tiles while
    # M advances: the property that keeps the band's weight slice in L2
    m_tiles, n_tiles = 16, 40
    per_band = BAND_N * m_tiles
    for t in range(m_tiles * n_tiles):
        g = t // per_band
        _, n = tile_origin(t, m_tiles, n_tiles, BAND_N)
        assert g * BAND_N <= n < min((g + 1) * BAND_N, n_tiles)
