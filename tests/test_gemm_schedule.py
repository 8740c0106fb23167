"""The GEMM kernels' work schedule (data-parallel, hybrid stream-K, stream-K, and the grouped
int8 kernel's remainder stream-K), enumerated on the host by the functions the kernels run
(h3b_gemm_schedule), against the properties the kernels rely on: every (tile, K slice) is computed exactly once; each tile is finished by
the unit holding its last K slice, which adds the partials of exactly the lower units that
computed the rest; a unit parks at most one partial, as its first item, so its slot and
flag are written once and every wait points at work done before anything else.  No GPU."""
import collections
import random

import pytest

from video_diffusion_transformer_03_b200 import h3b

# (tiles, k_blocks, units): the block GEMMs at 1,600 and 832 tokens on 74 CTA pairs, the
# 768x1344 workload, then edge cases (fewer tiles than units, one K slice, one unit)
SHAPES = [(252, 48, 74), (84, 48, 74), (336, 48, 74), (84, 192, 74), (48, 48, 74),
          (48, 192, 74), (144, 48, 74), (192, 48, 74), (540, 48, 74), (1620, 48, 74),
          (32, 128, 74), (10, 8, 74), (1, 1, 1), (1, 7, 3), (5, 1, 4), (148, 8, 74),
          (149, 3, 74), (147, 200, 148)]


def _random_shapes(n, seed=3):
    rng = random.Random(seed)
    return [(rng.randint(1, 400), rng.randint(1, 200), rng.randint(1, 80)) for _ in range(n)]


def hybrid_tile0(tiles, units):
    return max(0, tiles // units - 1) * units


def remainder_tile0(tiles, units):
    return tiles // units * units


def split_iters(tiles, kb, units, mode):
    tile0 = (hybrid_tile0(tiles, units) if mode == h3b.SCHED_HYBRID_STREAM_K else
             remainder_tile0(tiles, units) if mode == h3b.SCHED_REMAINDER_STREAM_K else 0)
    return (tiles - tile0) * kb


def runs_split(tiles, kb, units, mode):
    """Whether the GEMM calls split this shape in this mode (else they run it
    data-parallel): a unit with an empty range would never publish the flag its tile's
    owner waits for, so the pair kernels want 4 K slices per unit, the grouped kernel one
    group per unit and a partial wave past whole ones."""
    if mode == h3b.SCHED_REMAINDER_STREAM_K:
        return tiles > units and split_iters(tiles, kb, units, mode) >= units
    return split_iters(tiles, kb, units, mode) >= 4 * units


def check_schedule(tiles, kb, units, mode):
    per_unit = [h3b.gemm_schedule(tiles, kb, units, mode, u) for u in range(units)]
    cover = [[0] * kb for _ in range(tiles)]
    by_tile = collections.defaultdict(list)
    for u, items in enumerate(per_unit):
        parks = [i for i, it in enumerate(items) if it[3] == -1]
        assert parks in ([], [0]), (u, items)          # one partial at most, first
        for t, k0, k1, merge in items:
            assert 0 <= t < tiles and 0 <= k0 < k1 <= kb, (u, items)
            for k in range(k0, k1):
                cover[t][k] += 1
            if merge == -1:
                assert k1 < kb
            else:
                assert k1 == kb and 0 <= merge <= u
            by_tile[t].append((u, k0, k1, merge))
    assert all(c == 1 for row in cover for c in row)
    for t, parts in by_tile.items():
        owner = [p for p in parts if p[2] == kb]
        assert len(owner) == 1, (t, parts)
        ou, ok0, _, merge = owner[0]
        others = sorted(parts, key=lambda p: p[0])
        others.remove(owner[0])
        # the partials come from units merge .. ou-1, one each, in K order
        assert [p[0] for p in others] == list(range(merge, ou)), (t, parts)
        k = 0
        for p in others:
            assert p[1] == k and p[3] == -1
            k = p[2]
        assert k == ok0
    return per_unit


# (tiles, groups, units): the grouped int8 FC2 at 1,600 and 2,048 tokens (256 x 128 tiles,
# 1024-column groups, 74 pairs) and edge cases of the remainder form
GROUPED_SHAPES = [(168, 12, 74), (192, 8, 74), (75, 12, 74), (149, 1, 74), (148, 12, 74),
                  (80, 3, 74), (7, 5, 3)]


@pytest.mark.parametrize("tiles,kb,units", SHAPES + GROUPED_SHAPES + _random_shapes(300))
@pytest.mark.parametrize("mode", [h3b.SCHED_DATA_PARALLEL, h3b.SCHED_HYBRID_STREAM_K,
                                  h3b.SCHED_STREAM_K, h3b.SCHED_REMAINDER_STREAM_K],
                         ids=["dp", "hybrid", "sk", "remainder"])
def test_schedule_properties(tiles, kb, units, mode):
    if mode != h3b.SCHED_DATA_PARALLEL and not runs_split(tiles, kb, units, mode):
        with pytest.raises(h3b.H3BError):
            h3b.gemm_schedule(tiles, kb, units, mode, 0)
        return
    per_unit = check_schedule(tiles, kb, units, mode)
    if mode == h3b.SCHED_DATA_PARALLEL:
        for u, items in enumerate(per_unit):
            assert items == [(t, 0, kb, u) for t in range(u, tiles, units)]


@pytest.mark.parametrize("tiles,kb,units", SHAPES + _random_shapes(100, seed=5))
def test_hybrid_splits_only_the_last_one_to_two_waves(tiles, kb, units):
    tile0 = hybrid_tile0(tiles, units)
    sk_iters = (tiles - tile0) * kb
    if sk_iters < 4 * units:
        pytest.skip("run data-parallel by the GEMM calls")
    per_unit = h3b.gemm_schedule
    for u in range(units):
        items = per_unit(tiles, kb, units, h3b.SCHED_HYBRID_STREAM_K, u)
        split = [it for it in items if it[0] >= tile0]
        whole = [it for it in items if it[0] < tile0]
        # split phase first, then this unit's data-parallel tiles u, u + units, ...
        assert items == split + whole
        assert whole == [(t, 0, kb, u) for t in range(u, tile0, units)]
        # an equal share of the split iterations (the kernels' integer cut)
        share = sum(k1 - k0 for _, k0, k1, _ in split)
        assert share == sk_iters * (u + 1) // units - sk_iters * u // units
    if tiles >= units:
        assert units <= tiles - tile0 < 2 * units


@pytest.mark.parametrize("tiles,kb,units", GROUPED_SHAPES + _random_shapes(100, seed=7))
def test_remainder_splits_only_the_partial_wave(tiles, kb, units):
    if not runs_split(tiles, kb, units, h3b.SCHED_REMAINDER_STREAM_K):
        pytest.skip("run data-parallel by the grouped GEMM")
    tile0 = remainder_tile0(tiles, units)
    sk_iters = (tiles - tile0) * kb
    for u in range(units):
        items = h3b.gemm_schedule(tiles, kb, units, h3b.SCHED_REMAINDER_STREAM_K, u)
        split = [it for it in items if it[0] >= tile0]
        whole = [it for it in items if it[0] < tile0]
        # the split items first, then every whole wave data-parallel
        assert items == split + whole
        assert whole == [(t, 0, kb, u) for t in range(u, tile0, units)]
        share = sum(k1 - k0 for _, k0, k1, _ in split)
        assert share == sk_iters * (u + 1) // units - sk_iters * u // units
        assert share >= 1                      # every unit publishes what its owner awaits
    assert 0 < tiles - tile0 < units


def test_block_shapes_examples():
    # QKV at 1,600 tokens (252 tiles, 48 K slices, 74 pairs), pair 0: parks the first 19
    # slices of tile 149, finishes tile 148 alone, then data-parallel tiles 0 and 74
    assert h3b.gemm_schedule(252, 48, 74, h3b.SCHED_HYBRID_STREAM_K, 0) == [
        (149, 0, 19, -1), (148, 0, 48, 0), (0, 0, 48, 0), (74, 0, 48, 0)]
    # out-projection at 1,600 tokens (84 tiles): pair 5 parks 38 slices of tile 6, then
    # finishes tile 5 from slice 32 after adding pair 4's partial
    assert h3b.gemm_schedule(84, 48, 74, h3b.SCHED_HYBRID_STREAM_K, 5) == [
        (6, 0, 38, -1), (5, 32, 48, 4)]
    # grouped int8 FC2 at 1,600 tokens (168 tiles of 12 groups, 74 pairs): pair 0 parks
    # groups 0-2 of tile 148, then runs tiles 0 and 74 whole; pair 73 finishes tile 167
    # from group 8 after adding the sums of pairs 70-72
    assert h3b.gemm_schedule(168, 12, 74, h3b.SCHED_REMAINDER_STREAM_K, 0) == [
        (148, 0, 3, -1), (0, 0, 12, 0), (74, 0, 12, 0)]
    assert h3b.gemm_schedule(168, 12, 74, h3b.SCHED_REMAINDER_STREAM_K, 73) == [
        (167, 8, 12, 70), (73, 0, 12, 73), (147, 0, 12, 73)]


def test_schedule_rejects_bad_arguments():
    for args in [(0, 8, 4, 0, 0), (8, 0, 4, 0, 0), (8, 8, 0, 0, 0), (8, 8, 4, 4, 0),
                 (8, 8, 4, 0, 4), (8, 8, 4, 0, -1), (8, 8, 4, 3, 0)]:
        with pytest.raises(h3b.H3BError):
            h3b.gemm_schedule(*args)
