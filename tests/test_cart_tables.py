"""Pins of the library's Cartesian coupling tables (generated at build time by
csrc/gen_tables.cpp; used by the Cartesian edge convolution and the Cartesian node-local
product) against the oracle's Cartesian coupling (oracle/cartesian.py: index contractions,
the Levi-Civita symbol for odd paths, STF projection of full 3^l tensors), mapped into the
library's independent STF components by the tests' own expansion and entry picks
("FlashCart 如何让等变原子间势更快更准?", section "FlashCart 用笛卡尔内核替代球谐耦合").
Every path of L <= 3, entry by entry; no GPU needed."""
import os
import re

import numpy as np
import pytest

from cart_layout import coupling_table
from cg_tensor_products_b200 import build as etp_build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "cg_tensor_products_b200", "csrc", "generated", "etp_tables.h")


@pytest.fixture(scope="module")
def tables():
    if not os.path.exists(HEADER):
        etp_build.generate_tables()
    txt = open(HEADER).read()
    body = txt.split("constexpr CgNz kCart[kCartTotal] = {", 1)[1].split("};", 1)[0]
    entries = [(int(a), int(b), int(c), float(v)) for a, b, c, v in
               re.findall(r"\{(-?\d+), (-?\d+), (-?\d+), ([-+0-9.eE]+)\}", body)]

    def grid(name):
        g = txt.split(f"constexpr int {name}[4][4][4] = {{", 1)[1].split("};", 1)[0]
        return np.array([int(v) for v in re.findall(r"-?\d+", g)]).reshape(4, 4, 4)

    total = int(re.search(r"constexpr int kCartTotal = (\d+);", txt).group(1))
    assert len(entries) == total
    return entries, grid("kCartOff"), grid("kCartCnt")


PATHS = [(a, b, c) for a in range(4) for b in range(4) for c in range(4) if abs(a - b) <= c <= a + b]


@pytest.mark.parametrize("path", PATHS)
def test_compiled_cartesian_table_matches_oracle(tables, path):
    entries, off, cnt = tables
    l1, l2, l3 = path
    got = np.zeros((2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1))
    for m1, m2, m3, v in entries[off[path]: off[path] + cnt[path]]:
        got[m1, m2, m3] += v
    ref = coupling_table(l1, l2, l3)
    assert np.max(np.abs(got - ref)) < 1e-12 * max(1.0, np.max(np.abs(ref)))
    assert cnt[path] == np.count_nonzero(np.abs(ref) > 1e-12)     # zeros omitted, nothing else


def test_off_triangle_paths_are_empty(tables):
    _, _, cnt = tables
    for a in range(4):
        for b in range(4):
            for c in range(4):
                if not abs(a - b) <= c <= a + b:
                    assert cnt[a, b, c] == 0
