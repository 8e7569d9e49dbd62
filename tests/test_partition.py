"""Host-side check of the fused product's work split (no GPU).

The fused GEMV splits the (16-row tile, 128-column superblock) units of a
matrix evenly over the warps (w owns [w*U/W, (w+1)*U/W), W <= U); a tile covered by several warps is combined
from per-warp partial slots (slot index tile + warp) by the last warp to
arrive, which expects exactly owner(first unit) .. owner(last unit) to
contribute.  This test restates that arithmetic (plan + owner formula) and
checks, over many sizes, that: every unit is owned by exactly one warp, every
warp named as a contributor really owns units of the tile, slot indices are
unique and inside the workspace, and the plan never hands a warp an empty
range.
"""
import itertools


def plan(units, sm_count, warps_per_cta=16):
    ctas = min(sm_count, max(1, -(-units // warps_per_cta)))
    return min(units, ctas * warps_per_cta)


def owner(x, units, warps):
    """Largest w with floor(w * units / warps) <= x."""
    return ((x + 1) * warps - 1) // units


def check(n, k, sm_count):
    tiles = -(-n // 16)
    nsb = (k // 32 + 3) // 4
    units = tiles * nsb
    warps = plan(units, sm_count)
    assert warps <= sm_count * 16
    ranges = [(gw * units // warps, (gw + 1) * units // warps) for gw in range(warps)]
    assert all(lo < hi for lo, hi in ranges)  # no empty warp
    assert ranges[0][0] == 0 and ranges[-1][1] == units
    assert all(ranges[i][1] == ranges[i + 1][0] for i in range(warps - 1))
    for x in range(units):
        lo, hi = ranges[owner(x, units, warps)]
        assert lo <= x < hi
    slots = set()
    for r in range(tiles):
        first, last = owner(r * nsb, units, warps), owner((r + 1) * nsb - 1, units, warps)
        touching = [gw for gw, (lo, hi) in enumerate(ranges) if lo < (r + 1) * nsb and hi > r * nsb]
        assert touching == list(range(first, last + 1))
        whole = [gw for gw in touching if ranges[gw][0] <= r * nsb and (r + 1) * nsb <= ranges[gw][1]]
        if len(touching) > 1:
            assert not whole
            for gw in touching:
                slot = r + gw
                assert slot not in slots and slot < tiles + warps
                slots.add(slot)
        else:
            assert whole == touching


def test_partition_invariants():
    ns = [1, 15, 16, 17, 33, 100, 1024, 4096, 14336]
    ks = [32, 96, 128, 160, 1056, 4096, 8192, 14336]
    for n, k, sms in itertools.product(ns, ks, (1, 7, 148)):
        if (-(-n // 16)) * ((k // 32 + 3) // 4) > 200_000:
            continue
        check(n, k, sms)
