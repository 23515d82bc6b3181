"""A model of how the one-token decode kernel partitions its work, checked on the
CPU for many shapes:

* rows per CTA: an even split over two CTAs per SM, rounded up to the fewest
  rows whose bf16 scales fill whole 16-byte units;
* each warp's contiguous range, copied with one bulk copy per pair (and per
  gate/up area with a gated output);
* each lane group's walk over its rows, stepping the (pair, column) pair RPI
  rows at a time (several pairs at once when a pair has fewer rows than RPI).

Invariants: every output element is computed exactly once; each bulk copy of
weight rows stays inside its expert's rows and inside the CTA's shared-memory
area; when scale rows are bulk-copied, every source and destination offset and
every size is a multiple of 16 bytes (what the copy instruction requires); the
lane walk's (pair, column) always matches the row it reads.
"""

import math

import pytest


def rows_unit(G):
    u = 8
    while u > 1 and (u // 2) * G % 8 == 0:
        u //= 2
    return u


def rows_per_cta(total, G, sms=148):
    ctas = 2 * sms
    rb = -(-total // ctas)
    u = rows_unit(G)
    return -(-rb // u) * u


def check_partition(R, n, G, lpr, glu, sms=148):
    nn = n // 2 if glu else n
    areas = 2 if glu else 1
    total = R * nn
    rb = rows_per_cta(total, G, sms)
    ctas = -(-total // rb)
    s_bulk = nn % rows_unit(G) == 0
    rpi = 32 // lpr
    seen = [0] * total
    ids = [(7 * p + 3) % 11 for p in range(R)]  # any expert per pair
    for cta in range(ctas):
        g0 = cta * rb
        nrows = min(rb, total - g0)
        p_first, p_last = g0 // nn, (g0 + nrows - 1) // nn
        assert p_last - p_first < 64
        if s_bulk:
            for p in range(p_first, p_last + 1):
                lo = g0 - p * nn if p == p_first else 0
                hi = g0 + nrows - p * nn if p == p_last else nn
                for h in range(areas):
                    dst = (h * rb + p * nn + lo - g0) * G * 2
                    src = ((ids[p] * n + h * nn + lo) * G) * 2
                    size = (hi - lo) * G * 2
                    assert dst % 16 == 0 and src % 16 == 0 and size % 16 == 0, (R, n, G, cta, p, h)
        rpw = -(-nrows // 8)
        for warp in range(8):
            a = min(warp * rpw, nrows)
            b = min(a + rpw, nrows)
            r = a
            while r < b:  # the warp's bulk copies of weight rows
                g = g0 + r
                p, c0 = divmod(g, nn)
                cnt = min(b - r, nn - c0)
                for h in range(areas):
                    first_row = ids[p] * n + h * nn + c0
                    assert ids[p] * n <= first_row and first_row + cnt <= ids[p] * n + n
                    assert 0 <= h * rb + r and h * rb + r + cnt <= areas * rb
                r += cnt
            for gi in range(rpi):  # each lane group's walk
                g = g0 + a + gi
                p, c = divmod(g, nn)
                r = a + gi
                while r < b + gi:
                    if r < b:
                        assert (p, c) == divmod(g0 + r, nn), (R, n, lpr, cta, warp, gi, r)
                        seen[g0 + r] += 1
                    c += rpi
                    while c >= nn:
                        c -= nn
                        p += 1
                    r += rpi
    assert all(v == 1 for v in seen), (R, n, G, lpr, glu)
    return rb, ctas, s_bulk


@pytest.mark.parametrize("glu", [False, True])
@pytest.mark.parametrize("lpr", [4, 8, 16, 32])
def test_partition_many_shapes(lpr, glu):
    for R in (1, 2, 3, 5, 8, 13, 32, 64):
        for n in (1, 2, 3, 4, 5, 6, 10, 13, 14, 38, 96, 200, 704, 1408, 2816):
            if glu and n % 2:
                continue  # a gated output needs gate and up halves
            for G in (1, 2, 3, 4, 11, 16, 22, 44, 88):
                check_partition(R, n, G, lpr, glu)


def test_decode_shapes():
    # gate/up: 8 pairs x 1408 rows, 44 groups: 40 rows per CTA, 282 CTAs, bulk-copied scales
    assert check_partition(8, 1408, 44, 32, False) == (40, 282, True)
    # the same weights as a gated output: 704 outputs per pair, 20 per CTA, the same 282 CTAs
    assert check_partition(8, 1408, 44, 32, True) == (20, 282, True)
    # down: 8 x 2816 rows, 11 groups (odd): rows per CTA a multiple of 8
    assert check_partition(8, 2816, 11, 8, False) == (80, 282, True)


def test_rows_unit_fills_16_bytes():
    for G in range(1, 200):
        u = rows_unit(G)
        assert u * G * 2 % 16 == 0
        assert u == 1 or (u // 2) * G * 2 % 16 != 0  # and it is the fewest such rows
        assert math.gcd(u, 8) == u
