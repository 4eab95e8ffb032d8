"""The GEMM kernels' work schedule with the last wave split along K, checked on
the host (the same code the kernels run, through mx_debug_split_units): every
K stage of every tile is computed exactly once; whole tiles keep the plain
order; a split tile's pieces come from consecutive workers, the last of them
finishes the tile and knows the first; each worker leaves at most one partial
sum (so one slot per worker suffices) and runs it before its finishing piece;
the split is balanced and planned only when it pays."""
import itertools

import pytest

from fp8_quantization_block_b200 import mx

WHOLE, PARTIAL, FINISH = mx.KUNIT_WHOLE, mx.KUNIT_PARTIAL, mx.KUNIT_FINISH


def schedule(tiles, workers, kt, mode):
    n, _ = mx.split_units(tiles, workers, kt, mode, 0)
    return n, [mx.split_units(tiles, workers, kt, mode, c)[1] for c in range(n)]


def check_schedule(tiles, workers, kt, mode):
    n, units = schedule(tiles, workers, kt, mode)
    covered = {}
    split = any(u[3] != WHOLE for us in units for u in us)
    rem = tiles % workers
    for c, us in enumerate(units):
        kinds = [u[3] for u in us]
        # whole tiles first, in the plain order c, c + n, ...
        nw = kinds.count(WHOLE) if not split else sum(1 for u in us if u[3] == WHOLE and u[0] < tiles - rem)
        for i in range(nw):
            assert us[i][:4] == (c + i * n, 0, kt, WHOLE)
        pieces = us[nw:]
        assert len(pieces) <= 2
        assert kinds.count(PARTIAL) <= 1
        if PARTIAL in kinds and FINISH in kinds:
            assert kinds.index(PARTIAL) < kinds.index(FINISH)   # the partial sum comes first
        if FINISH in kinds:
            assert kinds[-1] == FINISH                            # the finishing piece comes last
        for tile, kb, ke, kind, first in us:
            assert 0 <= tile < tiles and 0 <= kb < ke <= kt
            assert kb % 2 == 0 and (ke % 2 == 0 or ke == kt)      # whole two-stage scale groups
            assert (kind == WHOLE) == (kb == 0 and ke == kt)
            if kind == PARTIAL:
                assert ke < kt
            if kind == FINISH:
                assert 0 <= first < c
            for k in range(kb, ke):
                assert (tile, k) not in covered, (tile, k)
                covered[(tile, k)] = (c, kind, first)
    assert len(covered) == tiles * kt                             # every stage of every tile, once
    # a split tile: pieces on consecutive workers first .. last; the last
    # finishes it, the others are partial sums
    for t in range(tiles):
        owners = sorted({covered[(t, k)][0] for k in range(kt)})
        if len(owners) == 1:
            assert covered[(t, 0)][1] == WHOLE
            continue
        assert owners == list(range(owners[0], owners[-1] + 1))
        fin = covered[(t, kt - 1)]
        assert fin[0] == owners[-1] and fin[1] == FINISH and fin[2] == owners[0]
        for c in owners[:-1]:
            kinds = {covered[(t, k)][1] for k in range(kt) if covered[(t, k)][0] == c}
            assert kinds == {PARTIAL}
        # k order follows the worker order
        ks = [covered[(t, k)][0] for k in range(kt)]
        assert ks == sorted(ks)
    return n, units, split


CASES = list(itertools.product([1, 5, 73, 74, 100, 148, 192, 216, 300, 1000],
                               [1, 2, 7, 74, 148], [1, 2, 3, 4, 5, 8, 24, 31, 32, 64], [0, 1, 2]))


@pytest.mark.parametrize("tiles,workers,kt,mode", CASES)
def test_schedule_covers_every_stage_once(tiles, workers, kt, mode):
    check_schedule(tiles, workers, kt, mode)


def test_plan_rules():
    # never: plain tiles on min(T, P) workers
    for t, p, k in [(192, 74, 24), (112, 148, 32), (5, 148, 64)]:
        n, units, split = check_schedule(t, p, k, mx.MX_K_SPLIT_NEVER)
        assert not split and n == min(t, p)
    # a full last wave: nothing to split
    assert not check_schedule(148, 74, 24, mx.MX_K_SPLIT_ALWAYS)[2]
    # auto splits only GEMMs with at most half as many tiles as workers
    assert not check_schedule(192, 74, 24, mx.MX_K_SPLIT_AUTO)[2]     # the DiT GEMM's pair tiles
    assert not check_schedule(112, 148, 32, mx.MX_K_SPLIT_AUTO)[2]    # 28672-wide skinny GEMM
    assert check_schedule(32, 148, 112, mx.MX_K_SPLIT_AUTO)[2]        # 8192-wide, K = 28672
    assert check_schedule(192, 74, 24, mx.MX_K_SPLIT_ALWAYS)[2]
    # at most 8 workers share a tile: one tile of 256 stages on 8 of 148 workers
    n, units, split = check_schedule(1, 148, 256, mx.MX_K_SPLIT_AUTO)
    assert split and n == 8
    # auto wants 16 stages or more per worker: 64 stages over 8 workers is too little
    assert not check_schedule(1, 148, 64, mx.MX_K_SPLIT_AUTO)[2]
    assert check_schedule(1, 148, 64, mx.MX_K_SPLIT_ALWAYS)[2]
    assert not check_schedule(40, 148, 32, mx.MX_K_SPLIT_AUTO)[2]      # 40 x 10240 x 8192 NVFP4
    # fewer groups than workers: no split (no worker may be left without K)
    assert not check_schedule(5, 148, 4, mx.MX_K_SPLIT_ALWAYS)[2]
    # the single-kernel grid limit: more workers than slots never split
    assert not check_schedule(300, 149, 64, mx.MX_K_SPLIT_ALWAYS)[2]


@pytest.mark.parametrize("tiles,kt", [(1, 256), (4, 128), (32, 112), (40, 64), (70, 200)])
def test_auto_split_bounds_the_workers_of_a_tile(tiles, kt):
    """With at most 8 workers per tile, ranges hold at least m = floor(S / P)
    groups, so a tile of ng groups is shared by at most (ng - 2) // m + 2
    workers: nine or ten for these shapes."""
    n, units = schedule(tiles, 148, kt, mx.MX_K_SPLIT_AUTO)
    assert n == min(148, 8 * tiles)
    ng = (kt + 1) // 2
    m = tiles * ng // n
    owners = {}
    for c, us in enumerate(units):
        for tile, kb, ke, kind, first in us:
            owners.setdefault(tile, set()).add(c)
    assert max(len(v) for v in owners.values()) <= (ng - 2) // m + 2 <= 10


@pytest.mark.parametrize("tiles,workers,kt", [(192, 74, 24), (112, 148, 32), (112, 148, 64), (44, 74, 24),
                                              (250, 148, 13)])
def test_split_is_balanced(tiles, workers, kt):
    """The workers' K stages differ by at most one scale group (two stages)
    plus a ragged last stage, against a whole tile without the split."""
    n, units, split = check_schedule(tiles, workers, kt, mx.MX_K_SPLIT_ALWAYS)
    assert split and n == workers
    work = [sum(ke - kb for _, kb, ke, _, _ in us) for us in units]
    assert max(work) - min(work) <= 3
    assert max(work) < (tiles // workers + 1) * kt


def test_dit_shape_plan():
    """256 x 256 pair tiles of the DiT GEMM (4096 x 3072, K = 3072 MXFP8:
    24 stages) on 74 pairs with the tail split forced: two whole waves, then
    44 tiles' 528 groups over the 74 pairs (7 or 8 groups each)."""
    n, units, split = check_schedule(192, 74, 24, mx.MX_K_SPLIT_ALWAYS)
    assert split and n == 74
    for c, us in enumerate(units):
        assert [u[0] for u in us[:2]] == [c, c + 74]
        assert sum(ke - kb for _, kb, ke, _, _ in us[2:]) in (14, 16)


def test_workspace_sizes():
    for fmt, M, K in [(0, 4096, 3072), (3, 16, 8192), (2, 1, 8192), (0, 128, 256), (3, 4608, 3072)]:
        base = mx.mx_fused_workspace_bytes(fmt, M, K)
        split = mx.mx_fused_split_workspace_bytes(fmt, M, K)
        quads = min(4, (M + 31) // 32)
        assert base % 256 == 0 and split % 256 == 0
        assert split - base == 148 * 8 * quads * 4096
        # the header holds the band counters and 148 slot counters
        codes = mx.mx_codes_bytes(fmt, M, K)
        scales = mx.mx_scales_bytes(fmt, M, K)
        header = (64 + 4 * ((M + 127) // 128) + 4 * 148 + 255) // 256 * 256
        assert base == header + (codes + 255) // 256 * 256 + (scales + 255) // 256 * 256
    assert mx.mx_fused_split_workspace_bytes(99, 16, 256) == 0
    assert mx.mx_fused_split_workspace_bytes(0, -1, 256) == 0


def test_debug_key_values():
    assert mx.mx_debug_set(mx.MX_DEBUG_K_SPLIT, 3) == mx.MX_ERR_INVALID_ARG
    for v in (mx.MX_K_SPLIT_ALWAYS, mx.MX_K_SPLIT_NEVER, mx.MX_K_SPLIT_AUTO):
        assert mx.mx_debug_set(mx.MX_DEBUG_K_SPLIT, v) == mx.MX_OK
    assert mx.split_units(10, 4, 8, 0, 99)[1] == []
    with pytest.raises(mx.MxError):
        mx.split_units(10, 0, 8, 0, 0)
