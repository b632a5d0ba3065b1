"""The packed symmetric state layout of the tensor-core path (tc_layout.cuh).

The header is compiled for the host with g++ and its tables are checked
against what the builder, the scan and the readout rely on:
  - the 2176 rows hold every pair (i, j), i <= j, exactly once (2080 rows) and
    96 padding rows with i > j; row_index inverts row_ij on the pairs;
  - builder items 0-3 (tiles 4c..4c+3): a lane has the same j in all 4 tiles;
  - readout: each 32-bit word (rows 2p, 2p+1) is (i, j), (i, j+1) with j even
    or (i, j), (i+1, j) with i even; off-diagonal 16-row groups share one i.
"""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kernelized_linear_attention_fwd_b200", "csrc")


@pytest.fixture(scope="module")
def table(tmp_path_factory):
    exe = str(tmp_path_factory.mktemp("layout") / "layout_dump")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", CSRC,
                           os.path.join(ROOT, "tests", "csrc", "layout_dump.cpp"), "-o", exe])
    rows, pairs = {}, {}
    for line in subprocess.check_output([exe], text=True).splitlines():
        tag, a, b, c = line.split()
        if tag == "R":
            rows[int(a)] = (int(b), int(c))
        else:
            pairs[(int(a), int(b))] = int(c)
    return rows, pairs


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
