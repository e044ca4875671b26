"""Pins of the persistent-memory management oracle (CPU only).

Keys built so that every block's representative is a known multiple of the
mean query direction give closed-form scores; on them the expected persistent
set is written out by hand.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import memory as M


def _case(x_blocks, d=8, Lq=100, seed=0):
    """Blocks of 64 constant key rows x_c * e0 (+ zero-mean noise in the other dims);
    queries whose mean is e0.  Score of block c = x_c exactly."""
    rng = np.random.default_rng(seed)
    nblk = len(x_blocks)
    k = np.zeros((1, nblk * 64, 1, d))
    for c, x in enumerate(x_blocks):
        k[0, c * 64:(c + 1) * 64, 0, 0] = x
        noise = rng.integers(-4, 5, size=(32, d - 1)).astype(np.float64)
        k[0, c * 64:c * 64 + 32, 0, 1:] = noise
        k[0, c * 64 + 32:(c + 1) * 64, 0, 1:] = -noise  # zero mean over the block
    q = np.zeros((1, Lq, 1, d))
    q[0, :, 0, 0] = 1.0
    noise = rng.integers(-4, 5, size=(Lq // 2, d - 1)).astype(np.float64)
    q[0, :Lq // 2, 0, 1:] = noise
    q[0, Lq // 2:2 * (Lq // 2), 0, 1:] = -noise
    return torch.from_numpy(q), torch.from_numpy(k)


def test_scores_are_the_planted_values():
    xs = [3.0, -1.0, 0.5, 2.0, 7.0, -2.0, 4.0]
    q, k = _case(xs)
    ids, sc = oracle.persist_update(q, k, np.array([[0, 1, 2]]), 3, 4)
    assert np.allclose(sc[0], [3.0, -1.0, 0.5, 2.0, 7.0, -2.0, 4.0])
    # candidates 0..6 with scores above: top 3 = blocks 4 (7), 6 (4), 0 (3)
    assert ids.tolist() == [[0, 4, 6]]


def test_no_evicted_blocks_keeps_the_set():
    q, k = _case([1.0, 5.0, -3.0, 2.0])
    ids, _ = oracle.persist_update(q, k, np.array([[3, 1, 0]]), 2, 0)
    assert ids.tolist() == [[0, 1, 3]]


def test_equal_scores_keep_the_lower_block_id():
    q, k = _case([1.0, 2.0, 2.0, 2.0, 0.0])
    ids, _ = oracle.persist_update(q, k, np.array([[0, 3]]), 1, 2)  # candidates 0, 3, 1, 2
    assert ids.tolist() == [[1, 2]]


def test_shifting_every_key_leaves_the_choice_unchanged():
    q, k = _case([0.3, -0.7, 1.1, 0.2, 0.9, -0.1], Lq=64)
    ids0, sc0 = oracle.persist_update(q, k, np.array([[0, 1, 5]]), 2, 3)
    w = np.linspace(-2, 2, 8)
    ids1, sc1 = oracle.persist_update(q, k + torch.from_numpy(w), np.array([[0, 1, 5]]), 2, 3)
    assert np.array_equal(ids0, ids1)
    qbar = oracle.to64(q)[0, :, 0].mean(0)
    assert np.allclose(sc1 - sc0, qbar @ w)


_orig = M.persist_update


def test_query_representative_weights_every_row():
    # 70 query rows: 64 of (1, 0) and 6 of (0, 4).  The row mean (64/70, 24/70) prefers
    # block 0 (keys (1, 0)); the unweighted mean of the two block means, (0.5, 2),
    # would prefer block 1 (keys (0, 1)).
    d = 2
    q = np.zeros((1, 70, 1, d))
    q[0, :64, 0] = [1.0, 0.0]
    q[0, 64:, 0] = [0.0, 4.0]
    k = np.zeros((1, 128, 1, d))
    k[0, :64, 0] = [1.0, 0.0]  # block 0: score = mean q . e0 = 64/70
    k[0, 64:, 0] = [0.0, 1.0]  # block 1: score = 24/70
    ids, sc = oracle.persist_update(torch.from_numpy(q), torch.from_numpy(k), np.array([[1]]), 0, 1)
    assert np.allclose(sc[0], [24 / 70, 64 / 70])
    assert ids.tolist() == [[0]]


def _wrong_tie(q, k, persist_idx, evict_blk0, n_evict, block=64):
    ids, sc = _orig(q, k, persist_idx, evict_blk0, n_evict, block)
    # keeps the higher block id on ties
    out = []
    for s in range(ids.shape[0]):
        cands = [int(c) for c in persist_idx[s]] + list(range(evict_blk0, evict_blk0 + n_evict))
        best = sorted(range(len(cands)), key=lambda i: (-sc[s][i], -cands[i]))[:ids.shape[1]]
        out.append(sorted(cands[i] for i in best))
    return np.array(out, dtype=np.int32), sc


def test_planted_tie_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "persist_update", _wrong_tie)
    with pytest.raises(AssertionError):
        test_equal_scores_keep_the_lower_block_id()


def _unweighted_block_means(q, k, persist_idx, evict_blk0, n_evict, block=64):
    q64 = oracle.to64(q)
    nq = -(-q64.shape[1] // block)
    bm = np.stack([q64[:, j * block:(j + 1) * block].mean(1) for j in range(nq)], 1).mean(1)
    q2 = np.repeat(bm[:, None], q64.shape[1], axis=1)
    return _orig(torch.from_numpy(q2), k, persist_idx, evict_blk0, n_evict, block)


def test_planted_weighting_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(oracle, "persist_update", _unweighted_block_means)
    with pytest.raises(AssertionError):
        test_query_representative_weights_every_row()
