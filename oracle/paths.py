"""Irreps strings and tensor-product path enumeration for the oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Source passage: "FlashCart 如何让等变原子间势更快更准?", section "生成内核在高阶下胜过
球谐基线" — the edge convolution couples node features with the edge's
spherical harmonics over all allowed paths. The pages fix no path rule, so:
  * an irreps string lists each l once, ascending: "0+1+2", the range "0..3",
    or with parity letters "0e+1o+2e";
  * a path (l1, l2, l3) takes l1 from the input irreps, l2 = 0..sh_lmax, l3 from
    the output irreps, and exists iff |l1 - l2| <= l3 <= l1 + l2 (SO(3));
  * when parity letters are given, additionally p1 * (-1)^l2 == p3 (O(3));
  * paths are ordered lexicographically by (l1, l2, l3);
  * several paths into the same l3 are summed into one l3 block of C channels;
  * the feature layout is [node][l block ascending, m = -l..l][channel].
"""
from __future__ import annotations

import re


def parse_irreps(s: str):
    """Return a list of (l, parity) with parity in {+1, -1, None}."""
    s = s.replace(" ", "")
    m = re.fullmatch(r"(\d+)\.\.(\d+)", s)
    if m:
        lo, hi = int(m.group(1)), int(m.group(2))
        if lo > hi:
            raise ValueError(s)
        return [(l, None) for l in range(lo, hi + 1)]
    out = []
    for tok in s.split("+"):
        m = re.fullmatch(r"(\d+)([eo]?)", tok)
        if not m:
            raise ValueError(f"bad irreps token {tok!r}")
        par = {"": None, "e": 1, "o": -1}[m.group(2)]
        out.append((int(m.group(1)), par))
    ls = [l for l, _ in out]
    if ls != sorted(set(ls)):
        raise ValueError("irreps must list each l once, ascending")
    pars = {p is None for _, p in out}
    if len(pars) != 1:
        raise ValueError("either every irrep has a parity letter or none has")
    return out


def block_offsets(irreps):
    """{l: first component index of the l block}, and the total component count."""
    off, pos = {}, 0
    for l, _ in irreps:
        off[l] = pos
        pos += 2 * l + 1
    return off, pos


def enumerate_paths(irreps_in: str, sh_lmax: int, irreps_out: str):
    """Paths as a list of (l1, l2, l3), lexicographic."""
    ins, outs = parse_irreps(irreps_in), parse_irreps(irreps_out)
    use_parity = ins[0][1] is not None
    if use_parity != (outs[0][1] is not None):
        raise ValueError("input and output must both carry parity letters or neither")
    paths = []
    for l1, p1 in ins:
        for l2 in range(sh_lmax + 1):
            for l3, p3 in outs:
                if not (abs(l1 - l2) <= l3 <= l1 + l2):
                    continue
                if use_parity and p1 * (-1) ** l2 != p3:
                    continue
                paths.append((l1, l2, l3))
    return paths
