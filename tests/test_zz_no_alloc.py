"""vkv_block_select_noalloc: block selection for callers that cannot allocate.

Some callers cannot allocate device memory at the moment they call the
library (a serving loop whose memory is fully planned at start-up and that
hands the library no allocator, or a host program that only has this C
interface).  The no-alloc variant keeps the pooled block vectors in a fixed
scratch array inside the library instead of a caller workspace.  These tests
call it through the C ABI and check it against the workspace entry point,
twice in a row (the array is shared by every call and keeps the previous
call's contents), and check that requests larger than the array are refused.

This file is collected last on purpose, so that a run which stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from kv_cache_attention_chunk_b200 import build, vkv, workloads as W


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    vkv.lib()


def _args(B, H, Lq, Lkv, window_blk0, n_win_blk, topk, q_ptr, k_ptr, q_strides, k_strides, out_idx, out_scores):
    a = vkv.vkv_select_args()
    a.B, a.H, a.d, a.block = B, H, 128, 64
    a.Lq, a.Lkv = Lq, Lkv
    a.window_blk0, a.n_win_blk, a.topk = window_blk0, n_win_blk, topk
    a.q = vkv.vkv_tensor(q_ptr, *q_strides)
    a.k = vkv.vkv_tensor(k_ptr, *k_strides)
    a.out_idx = out_idx
    a.out_scores = out_scores
    a.workspace = None
    a.workspace_bytes = 0
    return a


def test_noalloc_refuses_requests_larger_than_its_scratch():
    # 2 x 40 heads x 1024 window blocks x 128 x 4 B = 41.9 MB > 4 MiB: refused before any device work
    need = vkv.vkv_block_select_workspace_size(2, 40, 512 * 64, 1024, 64, 128)
    assert need > vkv.NOALLOC_SCRATCH_BYTES
    a = _args(2, 40, 512 * 64, 2048 * 64, 1024, 1024, 9, 0x10000, 0x10000,
              (0, 40 * 128, 128), (0, 40 * 128, 128), 0x10000, None)
    assert vkv.vkv_block_select_noalloc(a, None) == 7  # VKV_ERR_WORKSPACE


def _case(seed, H, win_frames):
    return W.make_block_sparse("noalloc", seed=seed, H=H, d=128, frame_tokens=1536, block=64,
                               hist_frames=4, win_frames=win_frames, q_frames=3, n_persist=4)


def _noalloc_call(c, q, k, topk, kbar=None, order=False):
    dev = q.device
    idx = torch.full((c.B * c.H, c.n_qblk, topk), -1, dtype=torch.int32, device=dev)
    sc = torch.full((c.B * c.H, c.n_qblk, c.n_win_blk), float("nan"), dtype=torch.float32, device=dev)
    a = _args(c.B, c.H, c.Lq, c.k.shape[1], c.window_blk0, c.n_win_blk, topk, q.data_ptr(), k.data_ptr(),
              (q.stride(0), q.stride(1), q.stride(2)), (k.stride(0), k.stride(1), k.stride(2)),
              idx.data_ptr(), sc.data_ptr())
    od = None
    if kbar is not None:
        a.kbar = kbar.data_ptr()
    if order:
        od = torch.full((c.B * c.H, c.n_qblk), -1, dtype=torch.int32, device=dev)
        a.out_order = od.data_ptr()
    assert vkv.vkv_block_select_noalloc(a, torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    return idx, sc, od


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    """Calls in a row share the scratch array: a large call, then a smaller one with the
    same top-K on other inputs (if it read anything the first call left behind, its
    sets would differ from the workspace entry point's), then the first again."""
    dev = "cuda:0"
    for seed, H, win in ((2, 12, 6), (5, 3, 4), (2, 12, 6)):
        c = _case(seed, H, win)
        q, k = c.q.to(dev), c.k.to(dev)
        ref_idx, ref_sc = vkv.block_select(q, k, c.window_blk0, c.n_win_blk, 9, scores=True)
        idx, sc, _ = _noalloc_call(c, q, k, 9)
        assert torch.equal(idx, ref_idx), (seed, H, win)
        assert torch.equal(sc, ref_sc), (seed, H, win)  # same kernels: the same bits


@pytest.mark.gpu
def test_noalloc_with_cached_representatives_and_order():
    """The two other paths through the selection: window means passed in (kbar, no
    scratch needed) and the query-block order; idx, scores and order equal the
    workspace entry point's."""
    dev = "cuda:0"
    c = _case(7, 6, 6)
    q, k = c.q.to(dev), c.k.to(dev)
    kbar = vkv.block_pool(k, c.window_blk0, c.n_win_blk)
    ref_idx, ref_sc, ref_ord = vkv.block_select(q, k, c.window_blk0, c.n_win_blk, 18, scores=True, order=True,
                                                kbar=kbar)
    idx, sc, od = _noalloc_call(c, q, k, 18, kbar=kbar, order=True)
    assert torch.equal(idx, ref_idx)
    assert torch.equal(sc, ref_sc)
    assert torch.equal(od, ref_ord)
    idx2, _, od2 = _noalloc_call(c, q, k, 18, order=True)  # pooling the window itself: same sets and order
    assert torch.equal(idx2, ref_idx) and torch.equal(od2, ref_ord)
