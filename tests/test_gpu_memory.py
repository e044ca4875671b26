"""GPU parity of the persistent-memory update against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_attention_chunk_b200 import workloads as W
from parity_util import to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def vk():
    from kv_cache_attention_chunk_b200 import vkv
    vkv.lib()
    return vkv


def _planted(d, Lq, seed, x_blocks):
    """Block c's keys are x_c * u plus zero-mean noise; the queries' mean is u: score_c = x_c
    (up to fp32 rounding), far apart, so the choice is unique."""
    rng = np.random.default_rng(seed)
    H, nblk = 2, len(x_blocks)
    u = np.zeros(d)
    u[0] = 1.0
    k = np.zeros((1, nblk * 64, H, d), dtype=np.float32)
    for h in range(H):
        for c, x in enumerate(x_blocks):
            n = rng.integers(-3, 4, size=(32, d)).astype(np.float32) * 0.25
            n[:, 0] = 0.0
            k[0, c * 64:c * 64 + 32, h] = x * u + n
            k[0, c * 64 + 32:(c + 1) * 64, h] = x * u - n
    q = rng.integers(-3, 4, size=(1, Lq, H, d)).astype(np.float32) * 0.25
    q[0, :, :, 0] = 1.0
    q[0, :, :, 1:] -= q[0, :, :, 1:].mean(axis=0, keepdims=True).round(2)
    return (torch.from_numpy(q).to(torch.bfloat16), torch.from_numpy(k).to(torch.bfloat16))


@pytest.mark.parametrize("d,Lq", [(128, 256), (64, 200)])
def test_persist_update_planted_exact(d, Lq):
    xs = [float(x) for x in np.random.default_rng(3).permutation(40)[:24] - 12.5]
    q, k = _planted(d, Lq, 5, xs)
    persist = np.array([[0, 2, 4, 6, 8, 10, 12, 14]] * 2, dtype=np.int32)
    ids, sc = vk().persist_update(q.to(DEV), k.to(DEV), torch.from_numpy(persist).to(DEV), 16, 8, scores=True)
    torch.cuda.synchronize()
    ref_ids, ref_sc = oracle.persist_update(q, k, persist, 16, 8)
    assert np.abs(to_np(sc) - ref_sc).max() < 2e-3
    assert np.array_equal(ids.cpu().numpy(), ref_ids)


def test_persist_update_no_evicted_blocks_sorts_the_set():
    c = W.cfg_sparse()
    pers = np.ascontiguousarray(c.persist_idx[:, ::-1])  # descending input
    ids, _ = vk().persist_update(c.q.to(DEV), c.k.to(DEV), torch.from_numpy(pers).to(DEV), 0, 0)
    torch.cuda.synchronize()
    assert np.array_equal(ids.cpu().numpy(), np.sort(pers, axis=1))


@pytest.mark.parametrize("n_evict", [24, 100])
def test_persist_update_full_sparse_config(n_evict):
    # config-3 shape: 32 persistent blocks per head; the oldest window frame (24 blocks)
    # leaves, or 100 blocks (132 candidates: every warp of the cluster pools several)
    c = W.cfg_sparse()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ids, sc = vk().persist_update(c.q.to(DEV), c.k.to(DEV), torch.from_numpy(c.persist_idx).to(DEV),
                                  c.window_blk0, n_evict, scores=True, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref_ids, ref_sc = oracle.persist_update(c.q, c.k, c.persist_idx, c.window_blk0, n_evict)
    assert np.abs(to_np(sc) - ref_sc).max() < 1e-3
    got = ids.cpu().numpy()
    C = c.persist_idx.shape[1]
    for s in range(got.shape[0]):
        cands = list(c.persist_idx[s]) + list(range(c.window_blk0, c.window_blk0 + n_evict))
        score = dict(zip(cands, ref_sc[s]))
        assert len(set(got[s])) == C and list(got[s]) == sorted(got[s])
        kept = set(int(x) for x in got[s])
        dropped = [x for x in cands if x not in kept]
        # a valid top-C under the fp64 scores, up to fp32 rounding of near-ties
        assert min(score[x] for x in kept) >= max(score[x] for x in dropped) - 1e-4
        order = sorted(cands, key=lambda x: (-score[x], x))
        gap = score[order[C - 1]] - score[order[C]]
        if gap > 1e-4:
            assert kept == set(order[:C])


def test_persist_update_bad_id_sets_error_word():
    c = W.cfg_sparse()
    pers = c.persist_idx.copy()
    pers[3, 5] = c.window_blk0 + 2  # inside the evicted range
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    ids, _ = vk().persist_update(c.q.to(DEV), c.k.to(DEV), torch.from_numpy(pers).to(DEV), c.window_blk0, 24,
                                 err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == vk().DEVERR_BAD_INDEX
