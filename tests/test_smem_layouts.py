"""Host-side check of the shared-memory layouts of the compact 64x64 forward
kernel (gspn_compact64.cu): every warp-wide access pattern it issues must be
free of bank conflicts, i.e. take the minimum number of wavefronts for its
byte count, and the Hacc layout must be a bijection per row.

The address expressions below restate the kernel's; B200 shared memory has
32 banks of 4 bytes, and a warp access of 4/8/16-byte elements is served in
1/2/4 phases of 32/16/8 lanes.
"""
import itertools

import pytest

S, LPL, BOX = 64, 16, 2048


def hacc_off(r, u):
    return r * 256 + ((u ^ ((r >> 2) & 15) ^ ((u >> 4) & 1)) << 3)


def wavefronts(addrs, width):
    """Wavefronts a warp access needs: addrs[lane] = byte address."""
    lanes_per_phase = {4: 32, 8: 16, 16: 8}[width]
    total = 0
    for ph in range(0, 32, lanes_per_phase):
        banks = {}
        for a in addrs[ph:ph + lanes_per_phase]:
            for wd in range(width // 4):
                word = a // 4 + wd
                banks.setdefault(word % 32, set()).add(word)
        total += max(len(v) for v in banks.values())
    return total


def optimal(width):
    return 32 * width // 128


def lanes():
    return [(l >> 4, l & 15) for l in range(32)]


def test_hacc_is_a_bijection_per_row():
    for r in range(S):
        units = sorted((hacc_off(r, u) - r * 256) >> 3 for u in range(32))
        assert units == list(range(32))


@pytest.mark.parametrize("p,u", itertools.product(range(4), range(32)))
def test_row_pass_hacc_stores(p, u):
    # lane (g, t) stores the unit u of row 4t+p of its channel plane g
    addrs = [g * 16384 + hacc_off(4 * t + p, u) for g, t in lanes()]
    assert wavefronts(addrs, 8) == optimal(8)


@pytest.mark.parametrize("s,m", itertools.product(range(S), range(2)))
def test_column_pass_hacc_loads(s, m):
    # lane (g, t) reads units 2t, 2t+1 (columns 4t..4t+3) of row s
    addrs = [g * 16384 + hacc_off(s, 2 * t + m) for g, t in lanes()]
    assert wavefronts(addrs, 8) == optimal(8)


@pytest.mark.parametrize("box,p", itertools.product(range(4), range(4)))
def test_row_pass_stage_reads(box, p):
    # column chunks: four 512-byte slices (rows 4*r_hi + p), [plane][r_hi][16 B]
    addrs = [box * BOX + p * 512 + g * 256 + t * 16 for g, t in lanes()]
    assert wavefronts(addrs, 16) == optimal(16)


@pytest.mark.parametrize("box,e", itertools.product(range(4), range(8)))
def test_column_pass_stage_reads(box, e):
    # row chunks: [plane][8 rows][128 B]; lane (g, t) reads columns 4t..4t+3
    addrs = [box * BOX + g * 1024 + e * 128 + t * 8 for g, t in lanes()]
    assert wavefronts(addrs, 8) == optimal(8)


def test_row_pass_slices_hold_lane_rows():
    # the element-stride-4 boxes put row 4*r_hi + r_lo of plane g at
    # slice r_lo, offset g*256 + r_hi*16: lane t's rows 4t..4t+3 are its 4 slices
    seen = set()
    for g, r_lo, r_hi in itertools.product(range(2), range(4), range(16)):
        off = r_lo * 512 + g * 256 + r_hi * 16
        assert off not in seen
        seen.add(off)
    assert len(seen) == 2 * 64 and max(seen) + 16 == BOX
