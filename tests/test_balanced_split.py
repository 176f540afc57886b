"""Host-side check of the persistent pass's work split: with C = min(grid,
U) working CTAs, CTA c owns global tiles [c U / C, (c+1) U / C) (never
empty), the CTA holding tile t is ((t+1) C - 1) // U, and the pieces of one
(sequence, kv head) segment fit in min(grid, capacity tiles) workspace
slots.  (Same integer formulas as the kernel and the merge.)"""
import numpy as np


def start(c, U, C):
    return c * U // C


def cta_of(t, U, C):
    return ((t + 1) * C - 1) // U


def test_cta_of_tile_inverts_the_ranges():
    rng = np.random.default_rng(0)
    for _ in range(300):
        U = int(rng.integers(1, 5000))
        C = min(int(rng.integers(1, 300)), U)
        for t in rng.integers(0, U, 50):
            c = cta_of(int(t), U, C)
            assert 0 <= c < C
            assert start(c, U, C) <= t < start(c + 1, U, C)


def test_segment_pieces_fit_their_slots():
    rng = np.random.default_rng(1)
    for _ in range(200):
        grid = int(rng.integers(1, 200))
        tiles = [int(x) for x in rng.integers(0, 40, int(rng.integers(1, 30)))]
        U = sum(tiles)
        if U == 0:
            continue
        C = min(grid, U)
        assert all(start(c + 1, U, C) > start(c, U, C) for c in range(C))
        first = 0
        for n in tiles:
            if n:
                pieces = cta_of(first + n - 1, U, C) - cta_of(first, U, C) + 1
                assert 1 <= pieces <= min(grid, n)  # x2 partials per piece in the workspace
            first += n
