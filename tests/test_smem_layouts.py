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

S, LPL, BOX = 64, 32, 1024


def hacc_off(r, u):
    return r * 256 + ((u ^ ((r >> 1) & 15)) << 3)


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


def test_hacc_is_a_bijection_per_row():
    for r in range(S):
        units = sorted((hacc_off(r, u) - r * 256) >> 3 for u in range(32))
        assert units == list(range(32))


@pytest.mark.parametrize("p,u", list(itertools.product(range(2), range(32))))
def test_row_pass_hacc_stores(p, u):
    # lane t stores the unit u of row 2t+p
    addrs = [hacc_off(2 * t + p, u) for t in range(32)]
    assert wavefronts(addrs, 8) == optimal(8)


@pytest.mark.parametrize("s", range(S))
def test_column_pass_hacc_loads(s):
    # lane t reads unit t (columns 2t, 2t+1) of row s
    addrs = [hacc_off(s, t) for t in range(32)]
    assert wavefronts(addrs, 8) == optimal(8)


@pytest.mark.parametrize("box,p", list(itertools.product(range(4), range(2))))
def test_row_pass_stage_reads(box, p):
    # column chunk: two boxes of every other row (element stride 2); row
    # 2*r_hi + r_lo sits at r_lo*512 + r_hi*16; lane t reads rows 2t, 2t+1
    addrs = [box * BOX + p * 512 + t * 16 for t in range(32)]
    assert wavefronts(addrs, 16) == optimal(16)


def test_column_chunk_slices_cover_the_box():
    offs = sorted(r_lo * 512 + r_hi * 16 for r_lo in range(2) for r_hi in range(32))
    assert offs == [16 * i for i in range(64)]


@pytest.mark.parametrize("box,e", list(itertools.product(range(4), range(8))))
def test_column_pass_stage_reads(box, e):
    # row chunk box: [8 rows][128 B]; lane t reads columns 2t, 2t+1
    addrs = [box * BOX + e * 128 + t * 4 for t in range(32)]
    assert wavefronts(addrs, 4) == optimal(4)

