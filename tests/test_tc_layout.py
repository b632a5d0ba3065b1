"""The packed symmetric state layout of the tensor-core path (tc_layout.cuh).

The header is compiled for the host with g++ and its tables are checked
against what the builder, the scan and the readout rely on:
  - the 2176 rows hold every pair (i, j), i <= j, exactly once (2080 rows) and
    96 padding rows with i > j; row_index inverts row_ij on the pairs;
  - builder items 0-3 (tiles 4c..4c+3): a lane has the same j in all 4 tiles;
  - readout: each 32-bit word (rows 2p, 2p+1) is (i, j), (i, j+1) with j even
    or (i, j), (i+1, j) with i even; off-diagonal 16-row groups share one i.
The layout of KATA-Mg with two factors (coordinates 0-31 and 32-63) must
hold every pair inside one factor exactly once, no pair across the factors,
and keep the same builder and readout properties (items of tiles 0-3 and
4-7, and tile 8).
"""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kernelized_linear_attention_fwd_b200", "csrc")


@pytest.fixture(scope="module")
def tables(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("layout") / "layout_dump")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", CSRC,
                           os.path.join(ROOT, "tests", "csrc", "layout_dump.cpp"), "-o", exe])
    tabs = {1: ({}, {}), 2: ({}, {})}
    for line in subprocess.check_output([exe], text=True).splitlines():
        tag, a, b, c = line.split()
        rows, pairs = tabs[int(tag[1])]
        if tag[0] == "R":
            rows[int(a)] = (int(b), int(c))
        else:
            pairs[(int(a), int(b))] = int(c)
    return tabs


@pytest.fixture(scope="module")
def table(tables):
    return tables[1]


def test_rows_cover_every_pair_once(table):
    rows, pairs = table
    assert len(rows) == 17 * 128
    valid = {r: ij for r, ij in rows.items() if ij[0] <= ij[1]}
    assert len(valid) == 64 * 65 // 2
    assert len(set(valid.values())) == len(valid)
    assert all(0 <= i < 64 and 0 <= j < 64 for i, j in rows.values())
    assert len(pairs) == 2080
    for (i, j), r in pairs.items():
        assert rows[r] == (i, j)


def test_builder_lane_keeps_its_column(table):
    rows, _ = table
    for c in range(4):
        for lane in range(128):
            assert len({rows[128 * (4 * c + m) + lane][1] for m in range(4)}) == 1


def test_readout_words_are_single_products(table):
    rows, _ = table
    for r0 in range(0, 17 * 128, 2):
        (i0, j0), (i1, j1) = rows[r0], rows[r0 + 1]
        same_i = i0 == i1 and j1 == j0 + 1 and j0 % 2 == 0
        same_j = j0 == j1 and i1 == i0 + 1 and i0 % 2 == 0
        assert same_i or same_j, (r0, rows[r0], rows[r0 + 1])
    for k in range(96):  # off-diagonal groups of 16 rows share one i
        assert len({rows[16 * k + x][0] for x in range(16)}) == 1


def test_two_factor_layout(tables):
    rows, pairs = tables[2]
    assert len(rows) == 9 * 128
    valid = {r: ij for r, ij in rows.items() if ij[0] <= ij[1]}
    want = {(i, j) for i in range(64) for j in range(i, 64) if i // 32 == j // 32}
    assert len(want) == 2 * 32 * 33 // 2 == 1056
    assert set(valid.values()) == want and len(valid) == len(want)
    assert set(pairs) == want
    for (i, j), r in pairs.items():
        assert rows[r] == (i, j)
    # builder items: tiles 0-3 and 4-7 keep one column per lane
    for c in range(2):
        for lane in range(128):
            assert len({rows[128 * (4 * c + m) + lane][1] for m in range(4)}) == 1
    # readout words are single bf16x2 products
    for r0 in range(0, 9 * 128, 2):
        (i0, j0), (i1, j1) = rows[r0], rows[r0 + 1]
        same_i = i0 == i1 and j1 == j0 + 1 and j0 % 2 == 0
        same_j = j0 == j1 and i1 == i0 + 1 and i0 % 2 == 0
        assert same_i or same_j, (r0, rows[r0], rows[r0 + 1])
    # tiles 4-8 are tiles 12-16 of the single-factor layout
    rows1, _ = tables[1]
    for r in range(4 * 128, 9 * 128):
        assert rows[r] == rows1[r + 8 * 128]
