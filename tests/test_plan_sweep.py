"""Host-side planner invariants over a sweep of problem shapes (no GPU): the
waves of every tier cover all wave items exactly, the per-call workspace
holds the waves each stream owns, the launch count follows the tier's
structure, and the filter chunks hold whole channel pairs where the filter
grids pack two channels.  (The planner is the library's own; the pages fix
none of this, so the checks are of internal consistency.)"""
import itertools

import numpy as np
import pytest

from dimensional_long_convolution_b200 import hyena_nd as H

SHAPES = [(n,) for n in (8, 64, 256, 512, 4096, 1 << 16, 1 << 19, 1 << 21)] + \
         [(a, b) for a, b in itertools.product((8, 32, 64, 128, 256), (8, 64, 256))] + \
         [(a, b, c) for a, b, c in itertools.product((8, 64, 128), (16, 128), (8, 64, 256))]
BC = [(1, 1), (1, 7), (2, 64), (3, 5), (8, 256)]


def _items(info, dims, B, C):
    return B * ((C + 1) // 2) if info["tier"] == "long_1d" else B * C


@pytest.mark.parametrize("dims", SHAPES)
@pytest.mark.parametrize("B,C", BC)
def test_plan_invariants(dims, B, C):
    p = H.problem(dims, B, C, H.BF16)
    info = H.plan_info(p)
    tier = info["tier"]
    if tier in ("rows_1d", "fused_2d"):
        assert info["wave"] == 0 and info["waves"] == 1 and info["launches"] == 1 and info["streams"] == 1
        assert H.workspace_bytes_for(p, H.CALL_CONV) == 256
    else:
        items, wave, waves = _items(info, dims, B, C), info["wave"], info["waves"]
        assert wave >= 1 and waves * wave >= items > (waves - 1) * wave
        assert 1 <= info["streams"] <= 3 and info["streams"] <= waves
        per_item = (8 * 2 * dims[0]) if tier == "long_1d" else 8 * int(np.prod(dims))
        need = info["streams"] * wave * per_item
        assert H.workspace_bytes_for(p, H.CALL_CONV) >= 256 + need
        per_wave = (2 * info["split_levels"] - 1) if tier == "long_1d" else 3
        assert info["launches"] == waves * per_wave
        if tier != "long_1d":
            # waves hold whole channels' samples once a wave reaches B
            assert wave % B == 0 or wave < B
    # the filter chunk: at least one channel, at most C; whole pairs where
    # the grids pack two channels (2D, 3D, long 1D)
    fc = info["filter_chunk"]
    assert 1 <= fc <= C
    paired = len(dims) >= 2 or dims[0] > 256
    if paired and fc < C:
        assert fc % 2 == 0
    # every call's workspace is within the total, which is the largest
    sizes = [H.workspace_bytes_for(p, c) for c in (H.CALL_CONV, H.CALL_FILTER, H.CALL_KERNEL_GRAD)]
    assert H.workspace_bytes(p) == max(sizes)
