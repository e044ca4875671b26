"""Pins of the head-aware compaction oracle (CPU only).

What fixes each part: the per-head lengths and frame counts that the pages'
config-4 readings state, hand-worked merge roundings, the FULL policy reducing
to a plain reshape of the dense cache, and the bf16 rounding of the merge
against an independent library conversion.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import compaction as C

FT, HIST, CUR, RECENT = 1560, 60, 3, 2
PYRAMID = [(C.ANCHOR, 8)] * 4 + [(C.WAVE, p) for p in (2, 3, 4, 5)] + [(C.VEIL, 8)] * 4


def test_config4_per_head_lengths():
    lens = [len(C.head_frames(p, x, HIST, CUR, RECENT)) * FT for p, x in PYRAMID]
    assert lens == [21840] * 4 + [53040, 39000, 31200, 26520] + [15600] * 4
    assert sum(lens) == 299520


def test_wave_frame_counts():
    # middle frames only: drop the sink, the 2 recent and the 3 current frames
    counts = [len(C.head_frames(C.WAVE, P, HIST, CUR, RECENT)) - 6 for P in (2, 3, 4, 5)]
    assert counts == [28, 19, 14, 11]
    for P in (2, 3, 4, 5):
        mid = C.head_frames(C.WAVE, P, HIST, CUR, RECENT)[1:-5]
        assert all((HIST - f) % P == 0 and 1 <= f <= 57 for f in mid)


def test_anchor_frames_evenly_spaced_both_ends():
    assert C.head_frames(C.ANCHOR, 8, HIST, CUR, RECENT) == [0, 1, 9, 17, 25, 33, 41, 49, 57, 58, 59, 60, 61, 62]
    assert C.head_frames(C.ANCHOR, 1, 10, 0, 2) == [0, 1, 8, 9]
    # 3 frames over [1, 6]: positions 1, 3.5, 6 -> 1, 3, 6
    assert C.head_frames(C.ANCHOR, 3, 9, 1, 2) == [0, 1, 3, 6, 7, 8, 9]


def test_veil_pairs_precede_recent_frames():
    assert C.head_frames(C.VEIL, 8, HIST, CUR, RECENT) == [0, (50, 51), (52, 53), (54, 55), (56, 57), 58, 59,
                                                            60, 61, 62]
    assert C.head_frames(C.VEIL, 0, HIST, CUR, RECENT) == [0, 58, 59, 60, 61, 62]


def test_bad_rules_rejected():
    with pytest.raises(ValueError):
        C.head_frames(C.VEIL, 3, HIST, CUR, RECENT)
    with pytest.raises(ValueError):
        C.head_frames(C.ANCHOR, 58, HIST, CUR, RECENT)
    with pytest.raises(ValueError):
        C.head_frames(C.WAVE, 0, HIST, CUR, RECENT)


def _bits(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _vals(b):
    return torch.from_numpy(b.view(np.int16).copy()).view(torch.bfloat16).float().numpy()


def test_merge_hand_cases():
    # (a, b, bf16 mean): exact means, and halfway cases that round to the even mantissa
    cases = [
        (1.0, 1.0078125, 1.0),          # 1 + 2^-8: halfway between 1 (even) and 1 + 2^-7 (odd)
        (1.0078125, 1.015625, 1.015625),  # 1 + 1.5*2^-7: halfway, the even neighbour is 1 + 2^-6
        (1.0078125, 1.0234375, 1.015625),  # exact
        (-2.0, 3.0, 0.5),
        (0.0, -0.0, 0.0),
    ]
    a = _bits([c[0] for c in cases])
    b = _bits([c[1] for c in cases])
    got = _vals(C.merge_frames(a, b))
    assert np.array_equal(got, np.array([c[2] for c in cases], dtype=np.float32))


def test_merge_matches_library_rounding():
    rng = np.random.default_rng(5)
    a = _bits(rng.standard_normal(4096).astype(np.float32) * 3)
    b = _bits(rng.standard_normal(4096).astype(np.float32) * 3)
    ref = ((torch.from_numpy(_vals(a)) + torch.from_numpy(_vals(b))) * 0.5).to(torch.bfloat16)
    got = torch.from_numpy(C.merge_frames(a, b).view(np.int16).copy()).view(torch.bfloat16)
    assert torch.equal(got, ref)


def test_full_policy_is_the_dense_cache_per_head():
    rng = np.random.default_rng(6)
    B, H, d, ft, hist, cur = 2, 3, 8, 5, 6, 2
    k = rng.integers(0, 1 << 15, size=(B, (hist + cur) * ft, H, d), dtype=np.uint16)
    v = rng.integers(0, 1 << 15, size=(B, (hist + cur) * ft, H, d), dtype=np.uint16)
    kf, vf, cu, _ = oracle.compact_cache(k, v, [(C.FULL, 0)] * H, ft, hist, cur, 2)
    assert np.array_equal(kf, np.concatenate([k[b, :, h] for b in range(B) for h in range(H)], 0))
    assert np.array_equal(vf, np.concatenate([v[b, :, h] for b in range(B) for h in range(H)], 0))
    assert cu.tolist() == [i * (hist + cur) * ft for i in range(B * H + 1)]


def test_compacted_rows_come_from_the_listed_frames():
    rng = np.random.default_rng(7)
    B, H, d, ft, hist, cur = 1, 4, 4, 3, 12, 1
    rules = [(C.ANCHOR, 3), (C.WAVE, 3), (C.VEIL, 4), (C.FULL, 0)]
    k = rng.integers(0, 1 << 14, size=(B, (hist + cur) * ft, H, d), dtype=np.uint16)
    kf, _, cu, frames = oracle.compact_cache(k, k, rules, ft, hist, cur, 2)
    for h in range(H):
        rows = kf[cu[h]:cu[h + 1]]
        for i, f in enumerate(frames[h]):
            blk = rows[i * ft:(i + 1) * ft]
            if isinstance(f, tuple):
                want = C.merge_frames(k[0, f[0] * ft:(f[0] + 1) * ft, h], k[0, f[1] * ft:(f[1] + 1) * ft, h])
            else:
                want = k[0, f * ft:(f + 1) * ft, h]
            assert np.array_equal(blk, want)


def _round_toward_zero(x32):
    return (np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_planted_rounding_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(C, "bf16_bits_round", _round_toward_zero)
    with pytest.raises(AssertionError):
        test_merge_hand_cases()
