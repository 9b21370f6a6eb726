"""Work-unit order of the backward kernels (host check).

``unit_of`` in csrc/fa_internal.h maps a CTA index onto (tile rank, head):
heads in groups of kHeadGroup, tile-major within a group.  This test reads
kHeadGroup from the header, restates the mapping and checks that it is a
bijection onto every (tile rank, head) pair, and that within each group the
heaviest tile rank (0) comes first, for full and partial head groups.
"""
import os
import re

import pytest

HDR = os.path.join(os.path.dirname(__file__), "..", "exact_attention_112_b200", "csrc", "fa_internal.h")


def _group():
    src = open(HDR).read()
    body = src[src.index("void unit_of("):]
    return int(re.search(r"kHeadGroup = (\d+);", body).group(1))


def unit_of(idx, n_heads, n_tiles, g):
    per_group = g * n_tiles
    grp = idx // per_group
    r = idx - grp * per_group
    g0 = grp * g
    gsz = min(g, n_heads - g0)
    return r // gsz, g0 + r % gsz


@pytest.mark.parametrize("n_heads,n_tiles", [(1, 1), (2, 3), (8, 64), (9, 3), (17, 33), (64, 32), (512, 4)])
def test_bijection_and_order(n_heads, n_tiles):
    g = _group()
    seq = [unit_of(i, n_heads, n_tiles, g) for i in range(n_heads * n_tiles)]
    assert sorted(seq) == [(t, h) for t in range(n_tiles) for h in range(n_heads)]
    # inside a group the tile ranks never decrease (heaviest first)
    for grp_start in range(0, n_heads, g):
        ranks = [t for (t, h) in seq if grp_start <= h < grp_start + g]
        assert ranks == sorted(ranks)
