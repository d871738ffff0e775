"""Host-side GEMM planning (no GPU): the plan query of the C ABI, and the
stream-K work split of decode tiles checked by enumeration.

The stream-K model below restates the kernel's rules (CTA c runs the flattened
iterations [c*L/G, (c+1)*L/G); a unit that does not cover its whole tile
writes slot 2c if it is the CTA's first unit, else 2c+1; the fix-up block of
boundary c sums, for the tile that boundary falls in, the slots of CTA c-1 and
of every CTA starting inside the tile) and checks on many shapes that every
(tile, k-block) is computed exactly once and that every split tile is summed
exactly once, from exactly the slots its contributors wrote."""
import ctypes

import pytest

from w8a8_int8_quantized_norm_b200 import sq

SMS = 148  # what the planner assumes when no device is visible


@pytest.fixture(scope="module")
def L():
    return sq.lib()


def _plan(M, N, K, path=0, split=0):
    return sq.gemm_plan(M, N, K, path, split)


def test_plan_kinds_and_workspace_agree_with_the_size_query(L):
    p = _plan(1, 28672, 8192)
    assert (p.kernel, p.stream_k, p.split_k, p.tile_m, p.tile_n) == (2, 1, 1, 128, 16)
    assert p.ctas == SMS and p.launches == 2
    assert p.workspace_bytes == 2 * SMS * 128 * 1 * 4
    # 8 x 48 tiles of 256 x 256 and 8 x 55 of 256 x 224 fill 74 SM pairs in 6
    # rounds, 8 x 64 of 256 x 192 in 7; a K step costs about 480 + 0.625 TN
    # cycles, so 224 wins
    p = _plan(2048, 12288, 4096)
    assert (p.kernel, p.tile_m, p.tile_n, p.launches, p.workspace_bytes) == (1, 256, 224, 1, 0)
    # one round at every width: the narrowest step wins
    assert _plan(1024, 3000, 272).tile_n == 192
    # 59 / 67 / 79 tiles: one round at 256 and 224, two at 192
    assert _plan(200, 15000, 64).tile_n == 224
    # 296 tiles of 256 are 4 full rounds, 344 of 224 take 5: 256 wins
    assert _plan(2048, 9472, 128).tile_n == 256
    p = _plan(16384, 57344, 8192)
    assert (p.kernel, p.tile_m, p.tile_n) == (1, 256, 256)
    p = _plan(2048, 12288, 4096, path=3)
    assert (p.kernel, p.tile_m, p.tile_n, p.ctas) == (0, 128, 256, SMS)
    p = _plan(16, 1024, 8192, split=4)
    assert (p.kernel, p.stream_k, p.split_k, p.workspace_bytes) == (2, 0, 4, 4 * 16 * 1024 * 4)
    # one whole tile per SM: no tile is shared, no fix-up, no workspace
    p = _plan(4, 128 * SMS, 128)
    assert (p.stream_k, p.launches, p.workspace_bytes) == (1, 1, 0)
    for M, N, K, split in [(1, 28672, 8192, 0), (16, 1024, 8192, 0), (128, 57344, 8192, 0),
                           (16, 1024, 8192, 4), (64, 10240, 8192, 0)]:
        assert _plan(M, N, K, 0, split).workspace_bytes == sq.gemm_workspace_size(M, N, K, split)


def test_plan_rejects_bad_arguments(L):
    info = sq.GemmPlanInfo()
    assert L.sq_w8a8_gemm_plan(1, 1, 0, 0, 0, ctypes.byref(info)) == 1
    assert L.sq_w8a8_gemm_plan(1, 1, 16, 4, 0, ctypes.byref(info)) == 1
    assert L.sq_w8a8_gemm_plan(1, 1, 16, 0, 0, None) == 1
    assert L.sq_w8a8_gemm_plan(300, 64, 64, 1, 2, ctypes.byref(info)) == 2


def _streamk_model(tiles, kbt, G):
    L_ = tiles * kbt
    start = [c * L_ // G for c in range(G + 1)]
    computed = {}
    slots = {}  # slot -> (tile, kb0, kb1)
    finals = set()
    for c in range(G):
        it, end, first = start[c], start[c + 1], True
        while it < end:
            tile, kb0 = divmod(it, kbt)
            kb1 = min(kbt, kb0 + (end - it))
            for kb in range(kb0, kb1):
                assert (tile, kb) not in computed
                computed[(tile, kb)] = c
            it += kb1 - kb0
            if kb0 == 0 and kb1 == kbt:
                finals.add(tile)
            else:
                slot = 2 * c + (0 if first else 1)
                assert slot not in slots
                slots[slot] = (tile, kb0, kb1)
            first = False
    assert len(computed) == L_
    summed = {}
    for c in range(1, G):
        b = start[c]
        if b % kbt == 0:
            continue
        tile = b // kbt
        t0, t1 = tile * kbt, tile * kbt + kbt
        if start[c - 1] > t0:
            continue
        used = []
        for cc in range(c - 1, G):
            if start[cc] >= t1:
                break
            used.append(2 * cc if start[cc] // kbt == tile else 2 * cc + 1)
        assert tile not in summed
        summed[tile] = used
    # every split tile summed once, from exactly its slots, covering its K range once
    split_tiles = {t for (t, _, _) in slots.values()}
    assert set(summed) == split_tiles and not (split_tiles & finals)
    assert split_tiles | finals == set(range(tiles))
    for tile, used in summed.items():
        assert sorted(used) == sorted(s for s, (t, _, _) in slots.items() if t == tile)
        ranges = sorted(slots[s][1:] for s in used)
        assert ranges[0][0] == 0 and ranges[-1][1] == kbt
        assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    return bool(slots)


@pytest.mark.parametrize("tiles,kbt,G", [(224, 64, 148), (448, 64, 148), (8, 64, 148),
                                         (80, 64, 148), (148, 1, 148), (1, 3, 3), (3, 1, 3),
                                         (296, 2, 148), (7, 13, 148), (1000, 5, 148),
                                         (2, 300, 148), (64, 229, 148)])
def test_streamk_partition_and_fixup_cover_every_iteration_once(tiles, kbt, G):
    G = min(G, tiles * kbt)
    has_slots = _streamk_model(tiles, kbt, G)
    # the planner's workspace decision matches: slots exist iff a boundary is inside a tile
    assert has_slots == any((c * tiles * kbt // G) % kbt for c in range(1, G))
