"""bench.py's work accounting on CPU: kept-tile FLOPs and the FLOPs the
attention kernel executes when it walks the union of two query tiles' block
lists, both against brute force over the oracle's block lists."""
import os
import sys

import numpy as np
import pytest

import oracle
import svg_workloads as W

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def lists(wl):
    kinds = np.array([0 if c == "S" else 1 for c in wl.planted], np.uint8)
    return oracle.block_list(oracle.shape_of(wl), oracle.params_of(wl), kinds)


@pytest.mark.parametrize("key", ["tiny-f4-8x8", "cogvideox-f13-30x45", "wan2.1-1.3b-f21-30x52"])
def test_kept_and_executed_flops_equal_brute_force(key):
    wl = W.WORKLOADS[key]
    rp, col, _ = lists(wl)
    kept = executed = 0.0
    nqb, npair = wl.nqb, (wl.nqb + 1) // 2
    for bh in range(wl.B * wl.H):
        for p in range(npair):
            union = set()
            for qb in (2 * p, 2 * p + 1):
                if qb >= nqb:
                    continue
                t = bh * nqb + qb
                rows = min(wl.bq, wl.L - qb * wl.bq)
                for kb in col[rp[t]:rp[t + 1]]:
                    kept += 4.0 * wl.d * rows * min(wl.bk, wl.L - int(kb) * wl.bk)
                    union.add(int(kb))
                if wl.bq != 128:
                    executed += 4.0 * wl.d * wl.bq * wl.bk * (rp[t + 1] - rp[t])
            if wl.bq == 128:
                executed += len(union) * 2 * 4.0 * wl.d * wl.bq * wl.bk
    assert bench.kept_tile_flops(rp, col, wl) == pytest.approx(kept, rel=1e-12)
    assert bench.executed_tile_flops(rp, col, wl) == pytest.approx(executed, rel=1e-12)
    assert executed >= kept
