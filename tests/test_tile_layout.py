"""The library's private row-tile layout, checked on the CPU.

A small host program is compiled with nvcc against the library's own internal
header and calls its host-and-device position functions (the ones the CUDA-core
path reads codes with).  For every (tile row, column) of a tile it prints where
the code's bits sit.  The test checks that the placement is a bijection onto
the tile's code area: every code bit of every position lands on its own bit,
inside the area, and together they cover it exactly.  A lane's piece must also
hold exactly the codes of that lane's mma.m16n8k16 A fragments (rows g and
g + 8, columns 2c, 2c + 1, 2c + 8, 2c + 9 of each 16-wide slice).
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantized_expert_ffn_token_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")

K = 192   # three 64-wide k groups

PROGRAM = r"""
#include <cstdio>
#include "moe_internal.cuh"
using namespace qeffn;
int main() {
    const int K = %d;
    // Q4B32: one 4-bit field per position
    for (int r = 0; r < 16; ++r)
        for (int k = 0; k < K; ++k) {
            int byte, sh;
            q4_code_pos(r, k, &byte, &sh);
            printf("q4 %%d %%d %%d\n", r, k, byte * 8 + sh);
        }
    // Q3B32: three single bits per position
    for (int r = 0; r < 16; ++r)
        for (int k = 0; k < K; ++k) {
            int byte[3], bit[3];
            q3_code_pos(r, k, byte, bit);
            printf("q3 %%d %%d %%d %%d %%d\n", r, k, byte[0] * 8 + bit[0], byte[1] * 8 + bit[1], byte[2] * 8 + bit[2]);
        }
    // Q2B32: one 2-bit field per position
    for (int r = 0; r < 16; ++r)
        for (int k = 0; k < K; ++k) {
            int byte, sh;
            q2_code_pos(r, k, &byte, &sh);
            printf("q2 %%d %%d %%d\n", r, k, byte * 8 + sh);
        }
    MatLayout l4 = make_layout(MOE_Q4B32, 16, K), l3 = make_layout(MOE_Q3B32, 16, K);
    MatLayout l2 = make_layout(MOE_Q2B32, 16, K);
    printf("bytes %%d %%d %%d %%d %%d %%d\n", l4.code_bytes, l4.kg_bytes, l3.code_bytes, l3.kg_bytes,
           l2.code_bytes, l2.kg_bytes);
    return 0;
}
""" % K


@pytest.fixture(scope="module")
def positions(tmp_path_factory):
    nvcc = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("layout")
    src, exe = d / "layout.cu", d / "layout"
    src.write_text(PROGRAM)
    subprocess.check_call([nvcc, "-std=c++17", "-I", INCLUDE, "-I", CSRC, "-o", str(exe), str(src)])
    out = subprocess.check_output([str(exe)], text=True).split("\n")
    rows = {"q4": {}, "q3": {}, "q2": {}}
    sizes = None
    for line in out:
        p = line.split()
        if not p:
            continue
        if p[0] == "bytes":
            sizes = tuple(int(v) for v in p[1:])
        else:
            rows[p[0]][(int(p[1]), int(p[2]))] = [int(v) for v in p[3:]]
    return rows, sizes


def _bits(fmt, pos):
    """All code bits (absolute bit index in the code area) of one position."""
    if fmt == "q4":
        return [pos[0] + b for b in range(4)]
    if fmt == "q2":
        return [pos[0], pos[0] + 1]
    return pos


@pytest.mark.parametrize("fmt, width, kg_bytes", [("q4", 4, 512), ("q3", 3, 384), ("q2", 2, 256)])
def test_codes_fill_the_code_area_exactly_once(positions, fmt, width, kg_bytes):
    rows, sizes = positions
    code_bytes = {"q4": sizes[0], "q3": sizes[2], "q2": sizes[4]}[fmt]
    assert {"q4": sizes[1], "q3": sizes[3], "q2": sizes[5]}[fmt] == kg_bytes
    assert code_bytes == (K // 64) * kg_bytes == 16 * K * width // 8
    seen = set()
    for (r, k), pos in rows[fmt].items():
        for b in _bits(fmt, pos):
            assert 0 <= b < 8 * code_bytes
            assert b not in seen, f"{fmt}: bit {b} used twice (row {r}, k {k})"
            seen.add(b)
    assert len(seen) == 8 * code_bytes


@pytest.mark.parametrize("fmt, piece", [("q4", 16), ("q3", 12), ("q2", 8)])
def test_each_lane_piece_holds_its_fragment_codes(positions, fmt, piece):
    rows, _ = positions
    kg_bytes = 32 * piece
    for (r, k), pos in rows[fmt].items():
        g, c = r % 8, (k % 8) // 2
        lane = 4 * g + c
        start = 8 * ((k // 64) * kg_bytes + lane * piece)
        for b in _bits(fmt, pos):
            assert start <= b < start + 8 * piece, f"{fmt}: row {r}, k {k} outside lane {lane}'s piece"


def test_q2_fields_of_a_block_share_one_multiplier(positions):
    """Q2B32: within a lane's word, the fields of the first 32-block of a k group
    sit at bit offsets 0, 2, 8, 10 of a half (multipliers 1 and 4 once OR-ed into
    an fp16 mantissa, taking the word and the word shifted right by 8) and those
    of the second block at 4, 6, 12, 14 (multipliers 16 and 64); rows g use the
    lower multiplier of each pair and rows g + 8 the higher one."""
    rows, _ = positions
    for (r, k), pos in rows["q2"].items():
        off = pos[0] % 16                       # bit offset inside the 16-bit half
        first_block = (k % 64) < 32
        assert off in ((0, 2, 8, 10) if first_block else (4, 6, 12, 14))
        low_multiplier = (off % 8) in (0, 4)    # fields 0, 4 of a byte-half: x1 or x16
        assert low_multiplier == (r < 8)
