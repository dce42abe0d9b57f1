"""Host-side checks of the persistent schedule (no GPU needed).

The kernel's work list comes from the same scheduler code that
fle_plan_units runs on the host.  For every workload below, over all CTAs of
the plan: each tile's k-blocks are computed exactly once; a tile computed
whole has one unit; a shared (stream-K) tile's contributors are exactly the
CTAs first..last that the finishing CTA will read, in k order, each with the
workspace slot the finishing CTA expects; no CTA holds more than two shared
tiles; and the k-blocks are balanced across CTAs.
"""
import math
from collections import defaultdict

import pytest
from hypothesis import given, settings, strategies as st

import reduction_epilogue_b200 as fle
from reduction_epilogue_b200 import build as fle_build

WORKLOADS = [
    (128, 1024, 1024, "scale_hardtanh_gelu"),
    (2048, 8192, 8192, "scale_hardtanh_gelu"),
    (1024, 8192, 8192, "avgpool_gelu_scale_rowmax"),
    (128, 32768, 32768, "swish_scale"),
    (16, 8192, 8192, "scale_hardtanh_gelu"),
    (64, 8192, 8192, "scale_hardtanh_gelu"),
    (256, 8192, 8192, "scale_hardtanh_gelu"),
    (1024, 8192, 8192, "scale_hardtanh_gelu"),
    (4096, 8192, 8192, "scale_hardtanh_gelu"),
    (7, 36, 33, "swish_scale"),
    (300, 132, 1000, "none"),
    (129, 4100, 777, "none"),
    (33, 20000, 3000, "scale_hardtanh_gelu"),
]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fle_build.build()
    fle.load()


def collect(M, K, N, desc, sms):
    grid, _ = fle.plan_units(M, K, N, desc, sms, 0)
    per_cta = [fle.plan_units(M, K, N, desc, sms, c)[1] for c in range(grid)]
    return grid, per_cta


@pytest.mark.parametrize("sms", [148, 132, 7])
@pytest.mark.parametrize("precision", ["tf32", "3xtf32"])
@pytest.mark.parametrize("M,K,N,problem", WORKLOADS)
def test_schedule_covers_every_kblock_once(M, K, N, problem, precision, sms):
    check_schedule(M, K, N, problem, precision, sms)


@settings(max_examples=200, deadline=None, derandomize=True)
@given(M=st.integers(1, 6000), K4=st.integers(1, 4000), N=st.integers(1, 50000),
       problem=st.sampled_from(["scale_hardtanh_gelu", "swish_scale", "avgpool_gelu_scale_rowmax", "none"]),
       precision=st.sampled_from(["tf32", "3xtf32"]), sms=st.sampled_from([148, 132, 16, 7]))
def test_schedule_random_shapes(M, K4, N, problem, precision, sms):
    # the same invariants on shapes drawn at random (K a multiple of 4, as
    # the ABI requires)
    if problem == "avgpool_gelu_scale_rowmax":
        N = max(N, 16)
    check_schedule(M, 4 * K4, N, problem, precision, sms)


def check_schedule(M, K, N, problem, precision, sms):
    desc = fle.desc_for(problem, precision)
    grid, per_cta = collect(M, K, N, desc, sms)
    assert 1 <= grid <= sms
    # k-blocks are 32 wide
    num_kb = max(int(r[4]) for rows in per_cta for r in rows)
    assert num_kb == math.ceil(K / 32)
    cover = defaultdict(list)  # tile -> [(kb0, kb1, cta, row)]
    for c, rows in enumerate(per_cta):
        partial_slots = []
        for r in rows:
            t, ta, tb, kb0, kb1, partial, slot, first, last, slot_rule, b0, bw = (int(v) for v in r)
            assert 0 <= kb0 < kb1 <= num_kb
            cover[t].append((kb0, kb1, c, (ta, tb, b0, bw), partial, slot, first, last, slot_rule))
            if partial:
                partial_slots.append(slot)
                assert slot == slot_rule
        assert len(partial_slots) <= 2 and len(set(partial_slots)) == len(partial_slots)

    tiles = sorted(cover)
    assert tiles == list(range(len(tiles)))
    tas = {e[3][0] for v in cover.values() for e in v}
    tbs = {e[3][1] for v in cover.values() for e in v}
    if tbs == {-1}:
        check_mixed_widths(M, N, cover, per_cta)
    else:
        assert len(tas) * len(tbs) == len(tiles)
        # a uniform grid: tile tb starts at B row tb * width
        widths = {e[3][3] for v in cover.values() for e in v}
        assert len(widths) == 1
        assert all(e[3][2] == e[3][1] * e[3][3] for v in cover.values() for e in v)
    # the tiles span exactly the operand rows (A side holds M, or N in the
    # swapped order, in tiles of 128 rows, or 256 rows on CTA pairs)
    a_rows = {math.ceil(M / 128), math.ceil(N / 128), math.ceil(M / 256), math.ceil(N / 256)}
    assert len(tas) in a_rows

    for t, units in cover.items():
        units.sort()
        # exact cover of [0, num_kb)
        pos = 0
        for kb0, kb1, *_ in units:
            assert kb0 == pos
            pos = kb1
        assert pos == num_kb
        assert len({u[3] for u in units}) == 1  # one (ta, tb) per tile
        if len(units) == 1:
            assert units[0][4] == 0  # whole tile, not shared
        else:
            ctas = [u[2] for u in units]
            assert all(u[4] == 1 for u in units)
            first, last = units[0][6], units[0][7]
            assert all((u[6], u[7]) == (first, last) for u in units)
            assert ctas == list(range(first, last + 1))  # CTA order = k order

    # balance: stream-K spreads the remainder evenly
    load = [sum(int(r[4]) - int(r[3]) for r in rows) for rows in per_cta]
    assert sum(load) == len(tiles) * num_kb
    assert max(load) - min(load) <= num_kb


def check_mixed_widths(M, N, cover, per_cta):
    # A plan of mixed tile widths (the 512-wide pair kernel): every 256-row
    # panel of the output is cut into 512-wide tiles from column 0, then
    # 384-wide ones, which together cover [0, N) once (the last may reach
    # past N); at most one tile of each width per pair, all tiles whole.
    assert M > 128
    grid = len(per_cta)
    panels = defaultdict(list)
    for t, units in cover.items():
        assert len(units) == 1 and units[0][4] == 0
        ta, tb, b0, bw = units[0][3]
        panels[ta].append((b0, bw))
    assert sorted(panels) == list(range(math.ceil(M / 256)))
    for ta, tl in panels.items():
        tl.sort()
        pos = 0
        for b0, bw in tl:
            assert b0 == pos and bw in (512, 384)
            pos += bw
        assert pos >= N and tl[-1][0] < N
        ws = [bw for _, bw in tl]
        assert ws == sorted(ws, reverse=True)  # 512-wide first
    n512 = sum(1 for tl in panels.values() for _, bw in tl if bw == 512)
    n384 = sum(1 for tl in panels.values() for _, bw in tl if bw == 384)
    assert n512 <= grid and n384 <= grid
    for rows in per_cta:
        ws = [int(r[11]) for r in rows]
        assert ws.count(512) <= 1 and ws.count(384) <= 1
        if len(ws) == 2:
            assert ws == [512, 384]  # the wide tile first


def test_headline_shape_plans():
    # 2048x8192x8192 in TF32 runs 256-row tiles on CTA pairs, of mixed
    # widths: 128 tiles 512 wide (two 256-wide MMAs sharing each x tile)
    # would be two waves on the 74 pairs of 148 SMs, the second of 54; the
    # plan runs one wave of 74 tiles 512 wide and one of 73 tiles 384 wide
    # (a 256-wide and a 128-wide MMA), each pair at most one of each.  In
    # 3xTF32 (no wide tiles) it runs 256x256 tiles: 3.46 waves, three of whole
    # tiles and the 34 tiles of the last wave split in two k-aligned halves
    # on 68 pairs.
    desc = fle.desc_for("scale_hardtanh_gelu", "tf32")
    grid, per_cta = collect(2048, 8192, 8192, desc, 148)
    assert grid == 74 and _tiles(per_cta) == 74 + 73
    units = [r for rows in per_cta for r in rows]
    assert all(int(r[5]) == 0 for r in units)
    assert sum(1 for r in units if int(r[11]) == 512) == 74
    assert sum(1 for r in units if int(r[11]) == 384) == 73
    # columns per pair: 512 + 384 on 73 pairs, 512 on one
    cols = sorted(sum(int(r[11]) for r in rows) for rows in per_cta)
    assert cols == [512] + [896] * 73
    check_schedule(2048, 8192, 8192, "scale_hardtanh_gelu", "tf32", 148)
    grid3, per3 = collect(2048, 8192, 8192, fle.desc_for("scale_hardtanh_gelu", "3xtf32"), 148)
    assert grid3 == 74 and _tiles(per3) == 256
    load = [sum(int(r[4]) - int(r[3]) for r in rows) for rows in per3]
    assert sum(load) == 256 * 256 and max(load) - min(load) == 128
    halves = [r for rows in per3 for r in rows if r[5]]
    assert len(halves) == 68
    assert {(int(r[3]), int(r[4])) for r in halves} == {(0, 128), (128, 256)}


def test_k_aligned_split_needs_one_partial_slot():
    # 4096x8192x8192 in TF32: 256 wide tiles = 3 waves + 34 tiles split in two
    # k-aligned halves; every CTA holds at most one shared tile, in slot 0, so
    # the workspace holds one 128x512 partial per stream-K CTA.
    desc = fle.desc_for("scale_hardtanh_gelu", "tf32")
    grid, per = collect(4096, 8192, 8192, desc, 148)
    assert grid == 74 and _tiles(per) == 256
    shared = [[r for r in rows if int(r[5])] for rows in per]
    assert sum(len(x) for x in shared) == 68
    assert all(len(x) <= 1 and all(int(r[6]) == 0 for r in x) for x in shared)


def test_weight_streamed_once_shapes_split_each_tile():
    # M = 16 (swapped): 64 weight tiles of 128 rows on 148 SMs; each tile is
    # split into two k-aligned halves on 128 CTAs, every CTA streaming the
    # same 128 k-blocks of one tile.
    desc = fle.desc_for("scale_hardtanh_gelu", "tf32")
    grid, per_cta = collect(16, 8192, 8192, desc, 148)
    assert grid == 128
    units = [r for rows in per_cta for r in rows]
    assert len(units) == 128
    assert {(int(r[3]), int(r[4])) for r in units} == {(0, 128), (128, 256)}


def test_skinny_weight_stream_runs_whole_tiles_on_pairs():
    # 128 x 32768 x 32768 in TF32: 128 weight tiles of 256 rows on the 74
    # CTA pairs, each tile streamed whole by one pair (measured faster than
    # splitting the stream along K); 3xTF32 keeps one-CTA tiles of 128 rows.
    desc = fle.desc_for("swish_scale", "tf32")
    grid, per_cta = collect(128, 32768, 32768, desc, 148)
    assert grid == 74
    units = [r for rows in per_cta for r in rows]
    assert len(units) == 128 and all(int(r[5]) == 0 for r in units)  # whole tiles, no partials
    assert {(int(r[3]), int(r[4])) for r in units} == {(0, 1024)}
    grid3, per3 = collect(128, 32768, 32768, fle.desc_for("swish_scale", "3xtf32"), 148)
    assert grid3 == 148


def test_workspace_matches_the_plan():
    # two fp32 partial tiles per CTA plus one counter per shared tile
    desc = fle.desc_for("swish_scale", "tf32")
    lib = fle.load()
    import ctypes
    n = ctypes.c_int(0)
    g = ctypes.c_int(0)
    assert lib.fle_plan_units(128, 32768, 32768, ctypes.byref(desc), 148, 0, None, 0,
                              ctypes.byref(n), ctypes.byref(g)) == 0
    assert g.value == 74  # CTA pairs, whole tiles: no workspace


def _tiles(per):
    return 1 + max(int(r[0]) for rows in per for r in rows)


def test_pair_tile_width_fills_the_waves():
    # Direct pair plans take 224-wide tiles instead of 256 when that fills the
    # waves on 74 pairs better, and 512-wide tiles (TF32) when those are
    # enough cheaper per column.  1024 x 8192 x 8192 in TF32: 4 x 16 = 64
    # tiles of 512, one wave (224 wide: 148 tiles, two full waves; 256 wide:
    # 128 tiles, the second wave 54 of 74 pairs).  In 3xTF32 (no wide tiles)
    # the 256-wide plan spreads its uneven wave over all pairs, which costs
    # about as much as 224, and it keeps 256.  256 x 8192 x 8192 is 37 tiles
    # of 224 split in two on all 74 pairs (256 wide: 32 tiles on 64 pairs).
    d = fle.desc_for("avgpool_gelu_scale_rowmax", "tf32")
    grid, per = collect(1024, 8192, 8192, d, 148)
    assert grid == 64 and _tiles(per) == 64 and all(int(r[5]) == 0 for rows in per for r in rows)
    d = fle.desc_for("avgpool_gelu_scale_rowmax", "3xtf32")
    grid, per = collect(1024, 8192, 8192, d, 148)
    assert grid == 74 and _tiles(per) == 128
    d = fle.desc_for("scale_hardtanh_gelu", "tf32")
    grid, per = collect(256, 8192, 8192, d, 148)
    assert grid == 74 and _tiles(per) == 37
    assert all(len(rows) == 1 and int(rows[0][5]) == 1 for rows in per)
    # 2048 x 8192 x 8192: 512 wide, cut into mixed widths (see the headline test)
    grid, per = collect(2048, 8192, 8192, d, 148)
    assert {int(r[11]) for rows in per for r in rows} == {512, 384}


def test_mixed_widths_only_where_they_shorten_the_plan():
    # The mixed cut is taken for 512-wide plans of more than one wave that
    # it shortens: not for 4096 x 8192 x 8192 (3.5 waves: three whole and
    # one split in two), 1024 x 8192 x 8192 (one wave) or 2304 x 2048 x 8192
    # (144 tiles, no cut fits); yes for 3584 x 128 x 4096 (112 tiles of 512:
    # 74 of 512 and 52 of 384), 4096 x 128 x 3584 (16 panels) and the ragged
    # 2000 x 260 x 7000.
    d = fle.desc_for("none", "tf32")
    for M, K, N in [(4096, 8192, 8192), (1024, 8192, 8192), (2304, 2048, 8192)]:
        _, per = collect(M, K, N, d, 148)
        assert all(int(r[2]) >= 0 for rows in per for r in rows), (M, K, N)
    for M, K, N, wide, narrow in [(3584, 128, 4096, 74, 52), (4096, 128, 3584, 74, 54), (2000, 260, 7000, 74, 52)]:
        grid, per = collect(M, K, N, d, 148)
        ws = [int(r[11]) for rows in per for r in rows]
        assert ws.count(512) == wide and (narrow is None or ws.count(384) == narrow), (M, K, N)
        check_schedule(M, K, N, "none", "tf32", 148)


def test_uneven_last_wave_spreads_only_in_3xtf32():
    # 512 x 8192 x 14336 on 74 pairs.  TF32 runs whole tiles only (2 x 28 =
    # 56 tiles of 512, one wave; CTAs sharing a weight slab keep reading it
    # together from L2).  3xTF32 (112 tiles of 256 = 74 + 38; the 38 of the
    # last wave cannot be split evenly, 74 // 38 = 1) spreads the last wave's
    # k-blocks over all 74 pairs.
    tf = fle.desc_for("avgpool_gelu_scale_rowmax", "tf32")
    grid, per = collect(512, 8192, 14336, tf, 148)
    assert grid == 56 and _tiles(per) == 56 and all(int(r[5]) == 0 for rows in per for r in rows)
    x3 = fle.desc_for("avgpool_gelu_scale_rowmax", "3xtf32")
    grid, per = collect(512, 8192, 14336, x3, 148)
    load = [sum(int(r[4]) - int(r[3]) for r in rows) for rows in per]
    assert grid == 74 and _tiles(per) == 112
    assert sum(load) == 112 * 256 and max(load) - min(load) <= 1


def test_swapped_3xtf32_spreads_its_uneven_last_wave():
    # 128 x 32768 x 32768 in 3xTF32 runs the one-CTA swapped kernel: 256 weight
    # tiles of 128 rows on 148 CTAs, one full wave and 108 tiles that cannot be
    # split evenly (148 // 108 = 1).  Their k-blocks are spread over all 148
    # CTAs, so every CTA does one whole tile and 747 or 748 k-blocks more.
    d = fle.desc_for("swish_scale", "3xtf32")
    grid, per = collect(128, 32768, 32768, d, 148)
    load = [sum(int(r[4]) - int(r[3]) for r in rows) for rows in per]
    assert grid == 148 and _tiles(per) == 256
    assert sum(load) == 256 * 1024 and max(load) - min(load) <= 1
