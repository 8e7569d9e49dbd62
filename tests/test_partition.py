"""Host-side check of the fused product's work split (no GPU).

The fused GEMV lists the (16-row tile, 128-column superblock) units of all
matrices of a call one after another and splits them evenly over the warps
(w owns [w*U/W, (w+1)*U/W), W <= U).  A tile covered by several warps is
combined from per-warp partial slots (slot index tile + warp) by the tile's
first warp, which expects exactly owner(first unit) + 1 .. owner(last unit)
to contribute.  This test restates that arithmetic (plan + owner formula)
and checks, over many sizes and over a batch of matrices, that: every unit
is owned by exactly one warp, every warp named as a contributor really owns
units of the tile, slot indices are unique and inside the workspace, and the
plan never hands a warp an empty range.
"""
import itertools


def warps_per_cta(m):
    """12 warps for the one- to four-row kernels and for 17..32 rows, else 16."""
    nt = (min(max(m, 1), 32) + 7) // 8
    return 12 if m <= 4 or nt >= 3 else 16


def plan(units, sm_count, m=1):
    wpc = warps_per_cta(m)
    ctas = min(sm_count, max(1, -(-units // wpc)))
    return min(units, ctas * wpc), ctas * wpc


def owner(x, units, warps):
    """Largest w with floor(w * units / warps) <= x."""
    return ((x + 1) * warps - 1) // units


def check(shapes, sm_count, m=1):
    """shapes: the (n, k) of the matrices of one call."""
    tiles = [-(-n // 16) for n, _ in shapes]
    nsbs = [(k // 32 + 3) // 4 for _, k in shapes]
    units = sum(t * s for t, s in zip(tiles, nsbs))
    warps, launched = plan(units, sm_count, m)
    assert warps <= launched <= sm_count * 16
    ranges = [(gw * units // warps, (gw + 1) * units // warps) for gw in range(warps)]
    assert all(lo < hi for lo, hi in ranges)  # no empty warp
    assert ranges[0][0] == 0 and ranges[-1][1] == units
    assert all(ranges[i][1] == ranges[i + 1][0] for i in range(warps - 1))
    for x in range(units):
        lo, hi = ranges[owner(x, units, warps)]
        assert lo <= x < hi
    slots, ub, tb = set(), 0, 0
    for nt, nsb in zip(tiles, nsbs):
        for r in range(nt):
            lo_u, hi_u = ub + r * nsb, ub + (r + 1) * nsb
            first, last = owner(lo_u, units, warps), owner(hi_u - 1, units, warps)
            touching = [gw for gw, (lo, hi) in enumerate(ranges) if lo < hi_u and hi > lo_u]
            assert touching == list(range(first, last + 1))
            whole = [gw for gw in touching if ranges[gw][0] <= lo_u and hi_u <= ranges[gw][1]]
            if len(touching) > 1:
                assert not whole
                for gw in touching:
                    slot = tb + r + gw
                    assert slot not in slots and slot < sum(tiles) + warps
                    slots.add(slot)
            else:
                assert whole == touching
        ub += nt * nsb
        tb += nt


def test_partition_invariants():
    ns = [1, 15, 16, 17, 33, 100, 1024, 4096, 14336]
    ks = [32, 96, 128, 160, 1056, 4096, 8192, 14336]
    for n, k, sms in itertools.product(ns, ks, (1, 7, 148)):
        if (-(-n // 16)) * ((k // 32 + 3) // 4) > 200_000:
            continue
        for m in (1, 8, 32):
            check([(n, k)], sms, m)


def test_partition_of_a_batched_layer():
    """The seven matrices of a Llama-3-8B-shaped layer in one call, at the
    row counts of the decode and skinny paths."""
    layer = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096),
             (4096, 14336)]
    for m in (1, 2, 4, 8, 16, 32):
        check(layer, 148, m)
    check([(100, 4096), (17, 1056), (4096, 160)], 148, 1)  # ragged tiles and a short last problem
