"""Host-side check of the shared-memory layouts of the compact 64x64 forward
kernel (gspn_compact64.cu): every warp-wide access pattern it issues must be
free of bank conflicts, i.e. take the minimum number of wavefronts for its
byte count, and the row sums the row pass stores must be read back by the
column pass at the same addresses.

The Hacc (row-sum plane) addresses are taken from the kernel's source: the
definitions of its offset variables are extracted and evaluated, so a change
to the kernel's layout is checked as it stands (or fails to parse here).
B200 shared memory has 32 banks of 4 bytes, and a warp access of
4/8/16-byte elements is served in 1/2/4 phases of 32/16/8 lanes.
"""
import itertools
import os
import re

import pytest

KERNEL = os.path.join(os.path.dirname(__file__), "..", "linear_spatial_propagation_b200", "csrc", "gspn_compact64.cu")

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



# ---- the kernel's own Hacc address expressions ----------------------------------------

def _kernel_src():
    return open(KERNEL).read()


def _section(src, start, end):
    a = src.index(start)
    return src[a:src.index(end, a)]


def _expr(section, name):
    """The C expression of `const uint32_t name = ...;` (or of a pointer
    `name = haccp + ...;`) in this part of the kernel, as Python."""
    m = re.search(r"const uint32_t " + name + r" = ([^;]+);", section)
    if m is None:
        m = re.search(r"unsigned char\* const " + name + r" = haccp \+ ([^;]+);", section)
    assert m is not None, f"{name} not found in the kernel source"
    e = m.group(1).replace("(uint32_t)", "")
    e = re.sub(r"(\d+)u\b", r"\1", e)
    return e.replace("S", "64")


def _ev(expr, **v):
    return eval(expr, {"__builtins__": {}}, v)


def _kernel_hacc():
    src = _kernel_src()
    prelude = _section(src, "unsigned char* const hrow", "auto row_half")
    row = _section(src, "auto row_half", "auto col_half")
    col = _section(src, "auto col_half", "bool ok = true;")
    # the access forms these offsets are used in
    assert "sts64f(hrow + p * 256 + oA," in row and "sts64f(hrow + p * 256 + oB," in row
    assert "lds64f(hA + e * 256 + oA)" in col and "lds64f(hB - e * 256 + oB)" in col
    return {"hrow": _expr(prelude, "hrow"), "tk8": _expr(prelude, "tk8"), "t8": _expr(prelude, "t8"),
            "q8": _expr(row, "q8"), "row_oA": _expr(row, "oA"), "row_oB": _expr(row, "oB"),
            "hA": _expr(col, "hA"), "hB": _expr(col, "hB"), "k8": _expr(col, "k8"),
            "col_oA": _expr(col, "oA"), "col_oB": _expr(col, "oB")}


def _row_pass_stores(k):
    """{(row, unit): (address, (p, q, e, direction))} of the row pass's
    completed row sums: steps s = 8q + e of its second half (q = 4..7), odd e;
    left->right stores unit s/2 of rows 2t + p, right->left unit 31 - s/2."""
    st = {}
    for q in range(4, 8):
        for e in range(1, 8, 2):
            for t in range(32):
                tk8 = _ev(k["tk8"], t=t)
                q8 = _ev(k["q8"], q=q)
                oA = _ev(k["row_oA"], q8=q8, e=e, tk8=tk8)
                oB = _ev(k["row_oB"], oA=oA)
                for p in range(2):
                    base = _ev(k["hrow"], t=t) + p * 256
                    s_ = 8 * q + e
                    for key, addr in (((2 * t + p, s_ >> 1), base + oA), ((2 * t + p, 31 - (s_ >> 1)), base + oB)):
                        assert key not in st, f"row sum {key} stored twice"
                        st[key] = (addr, (p, q, e))
    return st


def _col_pass_loads(k):
    """{(row, unit): address} of the column pass's first half (q = 0..3): lane t
    reads unit t of row 8q + e (top->bottom) and of row 63 - 8q - e."""
    ld = {}
    for q in range(4):
        k8 = _ev(k["k8"], q=q)
        for e in range(8):
            for t in range(32):
                t8 = _ev(k["t8"], t=t)
                oA = _ev(k["col_oA"], k8=k8, e=e, t8=t8)
                oB = _ev(k["col_oB"], oA=oA)
                ld[(8 * q + e, t)] = _ev(k["hA"], q=q) + e * 256 + oA
                ld[(63 - 8 * q - e, t)] = _ev(k["hB"], q=q) - e * 256 + oB
    return ld


def test_kernel_row_sums_are_read_back_where_they_were_stored():
    k = _kernel_hacc()
    st, ld = _row_pass_stores(k), _col_pass_loads(k)
    assert sorted(st) == sorted(ld) == [(r, u) for r in range(64) for u in range(32)]
    for key, addr in ld.items():
        assert st[key][0] == addr, f"row sum {key}: stored at {st[key][0]}, loaded from {addr}"
    assert sorted(a for a, _ in st.values()) == [8 * i for i in range(64 * 32)]  # the plane, each unit once


def test_kernel_hacc_accesses_are_conflict_free():
    k = _kernel_hacc()
    st = _row_pass_stores(k)
    # one warp store: all 32 lanes, one (p, q, e, direction)
    by_access = {}
    for (r, u), (addr, (p, q, e)) in st.items():
        t = r >> 1
        dirn = u == ((8 * q + e) >> 1)
        by_access.setdefault((p, q, e, dirn), [None] * 32)[t] = addr
    assert len(by_access) == 2 * 4 * 4 * 2
    for addrs in by_access.values():
        assert None not in addrs and wavefronts(addrs, 8) == optimal(8)
    ld = _col_pass_loads(k)
    for r in range(64):
        assert wavefronts([ld[(r, t)] for t in range(32)], 8) == optimal(8)
