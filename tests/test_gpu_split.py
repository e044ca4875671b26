"""GPU parity of key-axis split units against the fp64 oracle.

With a workspace the schedule may cut a unit's key steps into pieces that run
on different SMs; each piece leaves its partial output and LSE in the
workspace and the last piece to arrive combines them.  These cases have few
units over long caches, so the schedule is forced to split (checked through
the host-side schedule for this device's SM count), and cover: pieces that
start inside a branch and pieces that span the branch boundary, single-tile
units and a ragged last query tile, d = 64 and 128, ragged caches, a device
length table that differs from the host copy the pieces were cut from,
block-sparse units (whose pieces are fractions of a key count known only on
the device), and equality with the unsplit schedule up to rounding.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from kv_cache_attention_chunk_b200 import workloads as W
from parity_util import assert_bf16_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def vk():
    from kv_cache_attention_chunk_b200 import build, vkv
    build.build()
    vkv.lib()
    return vkv


def n_sm():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _seg_schedule(c):
    v = vk()
    a = v.vkv_attn_args()
    a.mode = v.MODE_SEGMENTS
    a.B, a.H, a.Lq, a.Lkv, a.d = c.B, c.H, c.q.shape[1], c.k.shape[1], c.d
    a.scale = c.scale
    a.n_branches = len(c.branches)
    keep = []
    for i, br in enumerate(c.branches):
        arr = (v.vkv_segment * max(1, len(br)))(*[v.vkv_segment(int(s), int(n)) for s, n in br])
        keep.append(arr)
        a.segs[i] = ctypes.cast(arr, ctypes.POINTER(v.vkv_segment))
        a.n_segs[i] = len(br)
    return v.attn_schedule(a, n_sm(), True)


def _run_segments(c, split):
    v = vk()
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    res = v.chunk_attn_segments(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV), c.branches, scale=c.scale, err=err,
                                split=split)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return res


def _check_segments(c, res):
    ref = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale)
    for i in range(len(c.branches)):
        assert_bf16_close(res["o"][i], ref["branch_o"][i], f"split O branch {i}")
        assert_lse_close(res["lse"][i], ref["branch_lse"][i], f"split LSE branch {i}")
    if len(c.branches) == 2:
        assert_bf16_close(res["o_merged"], ref["dense_o"], "split O merged")
        assert_lse_close(res["lse_merged"], ref["dense_lse"], "split LSE merged")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,q_tokens", [(2, 256), (3, 300), (1, 77)])
def test_split_dual_branch_matches_oracle(d, H, q_tokens):
    c = W.make_dual_branch("split", 300 + H + d, H=H, d=d, frame_tokens=128, q_frames=2, hist_frames=120,
                           q_tokens=q_tokens)
    sch = _seg_schedule(c)
    assert len(sch["pieces"]) > 0, "the schedule was expected to split"
    res = _run_segments(c, True)
    _check_segments(c, res)


def test_split_equals_unsplit():
    c = W.make_dual_branch("split", 77, H=2, d=128, frame_tokens=128, q_frames=2, hist_frames=100)
    a = _run_segments(c, True)
    b = _run_segments(c, False)
    for x, y in [(a["o"][0], b["o"][0]), (a["o"][1], b["o"][1]), (a["o_merged"], b["o_merged"])]:
        assert (x.float() - y.float()).abs().max().item() <= 2e-2
    for x, y in [(a["lse"][0], b["lse"][0]), (a["lse"][1], b["lse"][1]), (a["lse_merged"], b["lse_merged"])]:
        assert (x - y).abs().max().item() <= 1e-4


def test_split_single_branch_and_empty_branch():
    c = W.make_dual_branch("split1", 78, H=2, d=128, frame_tokens=128, q_frames=2, hist_frames=100)
    one = W.SegmentCase(c.name, c.B, c.H, c.d, c.frame_tokens, c.q, c.k, c.v,
                        [c.branches[0] + c.branches[1]], c.scale, c.meta)
    assert len(_seg_schedule(one)["pieces"]) > 0
    res = _run_segments(one, True)
    ref = oracle.segment_attention(one.q, one.k, one.v, one.branches, one.scale)
    assert_bf16_close(res["o"][0], ref["branch_o"][0], "split single branch O")
    assert_lse_close(res["lse"][0], ref["branch_lse"][0], "split single branch LSE")
    # an empty second branch: zeros and -inf, the merge equals the first branch
    emp = W.SegmentCase(c.name, c.B, c.H, c.d, c.frame_tokens, c.q, c.k, c.v,
                        [c.branches[0] + c.branches[1], []], c.scale, c.meta)
    res = _run_segments(emp, True)
    assert torch.equal(res["o"][1], torch.zeros_like(res["o"][1]))
    assert torch.isneginf(res["lse"][1]).all()
    assert_bf16_close(res["o_merged"], ref["branch_o"][0], "merge with an empty branch")
    assert_lse_close(res["lse_merged"], ref["branch_lse"][0], "merge LSE with an empty branch")


def _ragged_inputs(seed, Lq, lens, d=128):
    rng = np.random.default_rng(seed)
    H = len(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = torch.from_numpy(rng.standard_normal((1, Lq, H, d), dtype=np.float32)).to(torch.bfloat16)
    k = torch.from_numpy(rng.standard_normal((int(cu[-1]), d), dtype=np.float32)).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((int(cu[-1]), d), dtype=np.float32)).to(torch.bfloat16)
    return q, k, v, cu


@pytest.mark.parametrize("Lq,lens", [(200, [20000, 3000, 9000]), (130, [16000, 0, 129])])
def test_split_ragged_matches_oracle(Lq, lens):
    v = vk()
    q, k, vv, cu = _ragged_inputs(5 + Lq, Lq, lens)
    scale = 1.0 / np.sqrt(128.0)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, l = v.chunk_attn_ragged(q.to(DEV), k.to(DEV), vv.to(DEV), torch.from_numpy(cu).to(DEV), cu, scale=scale,
                               err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ro, rl = oracle.ragged_attention(q, k, vv, cu, scale)
    assert_bf16_close(o, ro, "split ragged O")
    assert_lse_close(l, rl, "split ragged LSE")


def test_split_ragged_device_lengths_differ_from_host():
    """Pieces are cut from the host lengths; the device table is authoritative: a
    longer or shorter device range is still covered exactly."""
    v = vk()
    q, k, vv, cu = _ragged_inputs(9, 180, [12000, 12000, 6000])
    dev_cu = cu.copy()
    dev_cu[1] += 2000  # sequence 0 longer, sequence 1 shorter on the device
    scale = 1.0 / np.sqrt(128.0)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, l = v.chunk_attn_ragged(q.to(DEV), k.to(DEV), vv.to(DEV), torch.from_numpy(dev_cu).to(DEV), cu,
                               scale=scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ro, rl = oracle.ragged_attention(q, k, vv, dev_cu, scale)
    assert_bf16_close(o, ro, "ragged O, device lengths")
    assert_lse_close(l, rl, "ragged LSE, device lengths")


def test_split_repeat_calls_identical():
    """The arrival counters are cleared by every call: repeated calls agree bit for bit."""
    c = W.make_dual_branch("rep", 79, H=3, d=128, frame_tokens=128, q_frames=2, hist_frames=60, q_tokens=300)
    a = _run_segments(c, True)
    for _ in range(3):
        b = _run_segments(c, True)
        assert torch.equal(a["o_merged"], b["o_merged"]) and torch.equal(a["lse"][1], b["lse"][1])


def test_workspace_too_small_is_refused():
    v = vk()
    c = W.make_dual_branch("ws", 80, H=2, d=128, frame_tokens=128, q_frames=2, hist_frames=120)
    assert len(_seg_schedule(c)["pieces"]) > 0
    small = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(v.VkvError) as e:
        v.chunk_attn_segments(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV), c.branches, scale=c.scale, workspace=small)
    assert e.value.status == 7  # VKV_ERR_WORKSPACE


def _sparse_schedule(c, topk, grouped):
    v = vk()
    a = v.vkv_attn_args()
    a.mode = v.MODE_BLOCK_SPARSE
    a.B, a.H, a.Lq, a.Lkv, a.d = c.B, c.H, c.q.shape[1], c.k.shape[1], c.d
    a.scale = c.scale
    a.block = 64
    a.n_persist = c.persist_idx.shape[1]
    a.topk = topk
    a.window_blk0, a.n_win_blk = c.window_blk0, c.n_win_blk
    a.qblk_order = 1 if grouped else None  # only NULL or not matters to the schedule
    return v.attn_schedule(a, n_sm(), True)


@pytest.mark.parametrize("topk,grouped", [(16, False), (6, True), (40, False)])
def test_split_block_sparse_matches_oracle(topk, grouped):
    """Block-sparse units learn their key count on the device; their pieces are cut
    as fractions of it.  Long persistent lists make every unit long enough to cut."""
    v = vk()
    c = W.make_block_sparse("sp", seed=90 + topk, H=2, d=128, frame_tokens=256, block=64, hist_frames=40,
                            win_frames=12, q_frames=1, n_persist=120)
    assert len(_sparse_schedule(c, topk, grouped)["pieces"]) > 0, "the schedule was expected to split"
    q, k, vv = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    order = None
    if grouped:
        idx, _, order = v.block_select(q, k, c.window_blk0, c.n_win_blk, topk, order=True)
        sel = idx.cpu().numpy()
    else:
        sel = W.random_selection(7 + topk, c.B * c.H, c.n_qblk, c.n_win_blk, topk)
        idx = torch.from_numpy(sel).to(DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, l = v.chunk_attn_block_sparse(q, k, vv, torch.from_numpy(c.persist_idx).to(DEV), idx, c.window_blk0,
                                     c.n_win_blk, scale=c.scale, err=err, qblk_order=order)
    o2, l2 = v.chunk_attn_block_sparse(q, k, vv, torch.from_numpy(c.persist_idx).to(DEV), idx, c.window_blk0,
                                       c.n_win_blk, scale=c.scale, err=err, qblk_order=order, split=False)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale)
    assert_bf16_close(o, ro, "split sparse O")
    assert_lse_close(l, rl, "split sparse LSE")
    assert (o.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l - l2).abs().max().item() <= 1e-4
