"""Host-side work schedule of vkv_chunk_attn (CPU only, through the C ABI).

The schedule is host logic: units of one or two 128-row query tiles balanced
over the SMs, and, when a workspace is given, units cut along the key axis
into pieces whose partial results the kernel combines.  These tests read the
schedule the library would launch (vkv_debug_schedule, no device needed) and
check that it is a valid cover of the work:

* every (sequence, query tile) appears exactly once as a whole unit, or as
  the pieces of exactly one unit whose key-step ranges tile [0, steps)
  without gap or overlap;
* a unit has at most 8 pieces, each with its own workspace slot, slots of one
  unit consecutive, all slots distinct and below n_slots;
* a CTA's piece entries are the ones its unit list meets, in order;
* on the benchmarked shapes the split schedule is within a few per cent of
  the cost model's perfect balance, and clearly better than whole units.
"""
import ctypes

import numpy as np
import pytest

from kv_cache_attention_chunk_b200 import build, vkv

PIECE = 1 << 12
TWO = 1 << 13
C1 = 0.9  # single-tile cost relative to a pair over the same keys (the library's default)
KX_RATE = 0.65  # the selecting kernel's one-tile unit: cost per key step relative to a pair (the library's default)


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    vkv.lib()


def _seg_args(B, H, Lq, Lkv, branches, d=128):
    a = vkv.vkv_attn_args()
    a.mode = vkv.MODE_SEGMENTS
    a.B, a.H, a.Lq, a.Lkv, a.d = B, H, Lq, Lkv, d
    a.scale = 1.0 / np.sqrt(d)
    a.n_branches = len(branches)
    keep = []
    for i, br in enumerate(branches):
        arr = (vkv.vkv_segment * max(1, len(br)))(*[vkv.vkv_segment(s, n) for s, n in br])
        keep.append(arr)
        a.segs[i] = ctypes.cast(arr, ctypes.POINTER(vkv.vkv_segment))
        a.n_segs[i] = len(br)
    a._keep = keep
    steps = sum((n + 127) // 128 for br in branches for _, n in br if n > 0)
    return a, [steps] * (B * H)


def _ragged_args(Lq, lens, d=128):
    a = vkv.vkv_attn_args()
    a.mode = vkv.MODE_RAGGED
    H = len(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    a.B, a.H, a.Lq, a.Lkv, a.d = 1, H, Lq, int(cu[-1]), d
    a.scale = 1.0 / np.sqrt(d)
    a._cu = cu
    a.cu_seqlens_host = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    return a, [(n + 127) // 128 for n in lens]


def _check_cover(sch, n_seq, T, steps, n_sm, kx=False):
    cb, cp, units, pieces = sch["cta_begin"], sch["cta_piece0"], sch["units"], sch["pieces"]
    assert len(cb) <= n_sm + 1 and cb[0] == 0 and cb[-1] == len(units)
    assert np.all(np.diff(cb) >= 0)
    seen = {}
    slots = set()
    load = np.zeros(len(cb) - 1)
    for c in range(len(cb) - 1):
        k = cp[c]
        for code in units[cb[c]:cb[c + 1]]:
            code = int(code)
            s, tile0, two = code >> 14, code & 0xFFF, bool(code & TWO)
            tiles = (tile0, tile0 + 1) if two else (tile0,)
            assert tile0 + len(tiles) <= T and s < n_seq
            rate = 1.0 if two else C1
            S = steps(s, two) if callable(steps) else steps[s]
            if code & PIECE:
                x, y = (int(v) for v in pieces[k])
                k += 1
                j0, j1 = x & 0xFFFF, x >> 16
                slot0, idx, n = y & 0xFFFF, (y >> 16) & 0xFF, y >> 24
                assert 2 <= n <= 8 and idx < n and 0 <= j0 < j1 <= S
                assert slot0 + idx < sch["n_slots"] and (slot0 + idx) not in slots
                slots.add(slot0 + idx)
                seen.setdefault((s, tiles), []).append((j0, j1, slot0, idx, n, S))
                load[c] += rate * (j1 - j0 + 4.0)
            else:
                assert (s, tiles) not in seen
                seen[(s, tiles)] = "whole"
                # a whole one-tile unit of the selecting kernel splits its key steps
                # over the two softmax warpgroups
                load[c] += (KX_RATE * S + 2.0) if (kx and not two) else rate * (S + 2.0)
        assert k == cp[c + 1]
    # every query tile of every sequence exactly once
    covered = {}
    for (s, tiles), v in seen.items():
        for t in tiles:
            assert (s, t) not in covered
            covered[(s, t)] = True
        if v != "whole":
            v = sorted(v)
            assert len({p[2] for p in v}) == 1 and sorted(p[3] for p in v) == list(range(v[0][4]))
            assert len(v) == v[0][4]
            assert v[0][0] == 0 and v[-1][1] == v[0][5]
            for a, b in zip(v, v[1:]):
                assert a[1] == b[0]
    assert len(covered) == n_seq * T
    assert len(slots) == sch["n_slots"]
    return load


WAN14B = (1, 40, 4680, 37440, [[(0, 1560), (32760, 4680)], [(1560, 31200)]])
WAN13B = (1, 12, 4680, 37440, [[(0, 1560), (32760, 4680)], [(1560, 31200)]])
PYRAMID = [21840] * 4 + [53040, 39000, 31200, 26520] + [15600] * 4


def _read_spread(sch, steps):
    """Per sequence: the spread, in key steps of the cost model, of the times at which
    its units (and pieces) would read key step 0 -- start time minus first step --
    when every CTA starts at 0 and runs its list in order.  0 means every unit of
    the sequence streams the same K/V tiles at the same time (one DRAM read,
    shared through L2)."""
    cb, cp, units, pieces = sch["cta_begin"], sch["cta_piece0"], sch["units"], sch["pieces"]
    t0 = {}
    for c in range(len(cb) - 1):
        t, k = 0.0, cp[c]
        for code in units[cb[c]:cb[c + 1]]:
            code = int(code)
            s, two = code >> 14, bool(code & TWO)
            rate = 1.0 if two else C1
            if code & PIECE:
                x = int(pieces[k][0])
                k += 1
                j0, j1 = x & 0xFFFF, x >> 16
                t0.setdefault(s, []).append(t - j0 * rate)
                t += rate * (j1 - j0 + 4.0)
            else:
                t0.setdefault(s, []).append(t)
                t += rate * (steps[s] + 2.0)
    return np.array([max(v) - min(v) for _, v in sorted(t0.items())])


@pytest.mark.parametrize("shape", [WAN14B, WAN13B], ids=["wan14b", "wan13b"])
def test_dense_split_schedule_covers_balances_and_groups_heads(shape):
    """Dense dual-branch shapes: the split schedule covers the work, is within 3.5 % of
    the cost model's perfect balance and well below whole units (Wan-14B: 37 query
    tiles per head leave 5.8 pair-costs on the busiest SM against 5.1 on average;
    Wan-1.3B: one pair and one lone tile per SM).  Its units are dealt out head by
    head, so the units of most heads (each head's odd last tile included) stream its
    K/V at the same time; only a head cut by a wave boundary is spread over two
    waves."""
    B, H, Lq, Lkv, br = shape
    a, steps = _seg_args(B, H, Lq, Lkv, br)
    T = (Lq + 127) // 128
    whole = vkv.attn_schedule(a, 148, False)
    assert len(whole["pieces"]) == 0 and whole["n_slots"] == 0
    lw = _check_cover(whole, B * H, T, steps, 148)
    sp = vkv.attn_schedule(a, 148, True)
    ls = _check_cover(sp, B * H, T, steps, 148)
    assert sp["n_slots"] > 0
    ideal = (B * H) * ((T // 2) + C1 * (T & 1)) * (steps[0] + 2.0) / 148
    assert ls.max() <= 1.035 * ideal
    assert ls.max() <= 0.9 * lw.max()
    unit = steps[0] + 2.0
    spread = _read_spread(sp, steps)
    assert np.median(spread) <= 0.05 * unit
    assert spread.max() <= 1.2 * unit
    assert (spread > 0.75 * unit).sum() <= max(3, H // 5)


def test_ragged_split_schedule_covers_and_balances():
    a, steps = _ragged_args(4680, PYRAMID)
    T = 37
    whole = vkv.attn_schedule(a, 148, False)
    lw = _check_cover(whole, 12, T, steps, 148)
    sp = vkv.attn_schedule(a, 148, True)
    ls = _check_cover(sp, 12, T, steps, 148)
    ideal = sum((T // 2 + C1) * (s + 2.0) for s in steps) / 148
    assert ls.max() <= 1.06 * ideal
    assert ls.max() <= 0.85 * lw.max()


@pytest.mark.parametrize("n_sm", [1, 3, 16, 148])
@pytest.mark.parametrize("Lq,lens", [(130, [300, 5000, 70]), (1000, [64 * 128, 1, 0, 3000]), (77, [40000])])
def test_small_ragged_schedules_cover(n_sm, Lq, lens):
    a, steps = _ragged_args(Lq, lens)
    T = (Lq + 127) // 128
    for split in (False, True):
        _check_cover(vkv.attn_schedule(a, n_sm, split), len(lens), T, steps, n_sm)


@pytest.mark.parametrize("n_sm", [2, 7, 148, 160])
def test_small_segment_schedules_cover(n_sm):
    a, steps = _seg_args(2, 3, 700, 9000, [[(0, 100), (5000, 2000)], [(100, 4900)]])
    for split in (False, True):
        _check_cover(vkv.attn_schedule(a, n_sm, split), 6, 6, steps, n_sm)


def test_sparse_and_unsized_ragged_never_split():
    a, _ = _ragged_args(4680, PYRAMID)
    a.cu_seqlens_host = None
    assert len(vkv.attn_schedule(a, 148, True)["pieces"]) == 0
    assert vkv.vkv_chunk_attn_workspace_size(a) == 0


def test_workspace_size_needs_no_device_but_a_device_count():
    # without a device the size query cannot know the SM count and reports 0
    a, _ = _seg_args(*WAN14B)
    import torch
    if not torch.cuda.is_available():
        assert vkv.vkv_chunk_attn_workspace_size(a) == 0


@pytest.mark.parametrize("topk,grouped", [(72, True), (144, True), (144, False)])
def test_block_sparse_split_schedule_covers_and_balances(topk, grouped):
    """Block-sparse pieces are cut in the schedule's estimated key steps of a unit
    (persistent blocks plus the expected union of its query blocks' selections,
    two blocks per step) and scaled on the device to the real count."""
    a = vkv.vkv_attn_args()
    a.mode = vkv.MODE_BLOCK_SPARSE
    a.B, a.H, a.Lq, a.Lkv, a.d = 1, 12, 4608, 36 * 1536, 128
    a.scale, a.block, a.n_persist, a.topk = 0.088, 64, 32, topk
    a.window_blk0, a.n_win_blk = 30 * 1536 // 64, 144
    a.qblk_order = 1 if grouped else None  # only NULL or not matters to the schedule
    u4 = min(144, (1.5 if grouped else 4.0) * topk)
    u2 = min(144, (1.25 if grouped else 2.0) * topk)
    S2, S1 = int(np.ceil((32 + u4) / 2)), int(np.ceil((32 + u2) / 2))
    steps = lambda s, two: S2 if two else S1  # noqa: E731
    whole = vkv.attn_schedule(a, 148, False)
    lw = _check_cover(whole, 12, 36, steps, 148)
    sp = vkv.attn_schedule(a, 148, True)
    assert len(sp["pieces"]) > 0
    ls = _check_cover(sp, 12, 36, steps, 148)
    ideal = 216 * (S2 + 2.0) / 148
    assert ls.max() <= 0.88 * lw.max() and ls.max() <= 1.15 * ideal


@pytest.mark.parametrize("topk,grouped", [(9, True), (9, False), (36, True), (144, True)])
def test_selecting_kernel_balances_with_alternating_one_tile_units(topk, grouped):
    """With the selection in the kernel (window block means given) units stay
    whole.  216 two-tile units on 148 SMs would leave some SMs with two and others
    with one; a one-tile unit there splits its key steps over the two softmax
    warpgroups and costs about 0.65 of its steps, so the schedule mixes pairs and
    such units and the busiest SM carries well under two pairs."""
    a = vkv.vkv_attn_args()
    a.mode = vkv.MODE_BLOCK_SPARSE
    a.B, a.H, a.Lq, a.Lkv, a.d = 1, 12, 4608, 36 * 1536, 128
    a.scale, a.block, a.n_persist, a.topk = 0.088, 64, 32, topk
    a.window_blk0, a.n_win_blk = 30 * 1536 // 64, 144
    a.qblk_order = 1 if grouped else None  # only NULL or not matters to the schedule
    a.kbar = 16                            # likewise: the kernel selects for itself
    u4 = min(144, (1.5 if grouped else 4.0) * topk)
    u2 = min(144, (1.25 if grouped else 2.0) * topk)
    S2, S1 = int(np.ceil((32 + u4) / 2)), int(np.ceil((32 + u2) / 2))
    steps = lambda s, two: S2 if two else S1  # noqa: E731
    for split in (False, True):
        sch = vkv.attn_schedule(a, 148, split)
        assert len(sch["pieces"]) == 0
        assert np.any((sch["units"] & TWO) == 0), "expected one-tile units"
        load = _check_cover(sch, 12, 36, steps, 148, kx=True)
        assert load.max() <= 0.85 * 2 * (S2 + 2.0)


@pytest.mark.parametrize("topk", [9, 18, 36])
def test_short_block_sparse_units_are_not_split(topk):
    """Units of fewer than 48 estimated key steps stay whole (their real key counts
    vary with the selections, and a piece's fixed cost weighs too much on them)."""
    a = vkv.vkv_attn_args()
    a.mode = vkv.MODE_BLOCK_SPARSE
    a.B, a.H, a.Lq, a.Lkv, a.d = 1, 12, 4608, 36 * 1536, 128
    a.scale, a.block, a.n_persist, a.topk = 0.088, 64, 32, topk
    a.window_blk0, a.n_win_blk = 30 * 1536 // 64, 144
    a.qblk_order = 1
    assert len(vkv.attn_schedule(a, 148, True)["pieces"]) == 0
