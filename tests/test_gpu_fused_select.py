"""GPU parity of the block-sparse attention that selects its own window blocks.

With cached window block means (kbar) the attention kernel pools each unit's
query blocks, scores them and keeps the top-K itself.  Its selection must be
the standalone selection's, index for index (both follow the same arithmetic),
and therefore the oracle's wherever the fp64 scores leave no near-tie; its
outputs must be those of the two-launch path (standalone selection, then the
attention from the selected ids) within the bounds a key-axis split is held
to, and within the parity tolerances of the fp64 oracle.  (A one-tile unit of
the selecting kernel splits its key steps over two accumulators and merges
them by LSE at the end, so its rows round differently from the two-launch
path's; pairs of tiles follow the same arithmetic in both.)
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_attention_chunk_b200 import workloads as W
from parity_util import assert_bf16_close, assert_lse_close, sparse_iid_case, to_np

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_attention_chunk_b200 import build, vkv
    build.build()
    vkv.lib()
    assert torch.cuda.is_available()
    yield


def vk():
    from kv_cache_attention_chunk_b200 import vkv
    return vkv


def err_word():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def _case(seed, H, d, qf, n_persist, win=4, B=1):
    return W.make_block_sparse("fused", seed=seed, H=H, d=d, frame_tokens=256, block=64, hist_frames=3,
                               win_frames=win, q_frames=qf, n_persist=n_persist, B=B)


def _run_pair(c, q, K, order=None, sel_out=True):
    """(fused o, lse, selection) and (two-launch o, lse, selection) on the same inputs."""
    k, v = c.k.to(DEV), c.v.to(DEV)
    pidx = torch.from_numpy(c.persist_idx).to(DEV)
    kbar = vk().block_pool(k, c.window_blk0, c.n_win_blk)
    n_qblk = -(-q.shape[1] // 64)
    sel = torch.full((c.B * c.H, n_qblk, K), -1, dtype=torch.int32, device=DEV) if sel_out else None
    err = err_word()
    o, l = vk().chunk_attn_block_sparse(q, k, v, pidx, None, c.window_blk0, c.n_win_blk, scale=c.scale, err=err,
                                        qblk_order=order, kbar=kbar, topk=K, sel_out=sel)
    idx, _ = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K, kbar=kbar)
    err2 = err_word()
    o2, l2 = vk().chunk_attn_block_sparse(q, k, v, pidx, idx, c.window_blk0, c.n_win_blk, scale=c.scale,
                                          err=err2, qblk_order=order, split=False)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and int(err2.item()) == 0
    return (o, l, sel), (o2, l2, idx)


def _same_as_two_launch(o, l, o2, l2):
    """Outputs of the two paths within 2e-2, LSEs within 1e-4: the bounds the key-axis
    split is held to against the whole unit, the same kind of LSE merge of two key
    subsets (each subset's P is rounded to bf16 against its own running maximum)."""
    return (o.float() - o2.float()).abs().max().item() <= 2e-2 and (l - l2).abs().max().item() <= 1e-4


def _gap_ok(qn, kn, c, K):
    s = oracle.block_scores(qn, kn, c.window_blk0, c.n_win_blk, c.block)
    return oracle.select_topk(s, K), oracle.topk_gap(s, K) > 1e-4


# (seed, H, d, q frames, persistent blocks, K, query-block order, query rows cut from the end)
SMALL = [
    (90, 2, 128, 2, 5, 3, None, 0),        # odd persistent count: the prefix ends inside a tile
    (91, 2, 128, 1, 0, 4, None, 0),        # no persistent blocks: everything waits for the selection
    (92, 3, 64, 2, 2, 1, None, 0),         # a one-step prefix
    (93, 2, 128, 3, 3, 16, "random", 0),   # every window block (K = n_win)
    (94, 2, 64, 2, 8, 7, "select", 0),
    (95, 2, 128, 2, 5, 3, None, 37),       # ragged tail: a partial last query block
    (96, 3, 128, 3, 4, 5, "random", 100),  # ragged tail under a permuted order
]


@pytest.mark.parametrize("seed,H,d,qf,npers,K,order,cut", SMALL)
def test_fused_select_small(seed, H, d, qf, npers, K, order, cut):
    c = _case(seed, H, d, qf, npers)
    qn = c.q[:, :c.q.shape[1] - cut] if cut else c.q
    q = qn.contiguous().to(DEV)
    n_qblk = -(-q.shape[1] // 64)
    perm = None
    if order == "random":
        rng = np.random.default_rng(seed)
        perm = torch.from_numpy(np.stack([rng.permutation(n_qblk) for _ in range(c.B * c.H)]).astype(np.int32)).to(DEV)
    elif order == "select":
        _, _, perm = vk().block_select(q, c.k.to(DEV), c.window_blk0, c.n_win_blk, K, order=True)
    (o, l, sel), (o2, l2, idx) = _run_pair(c, q, K, perm)
    assert torch.equal(sel, idx), "in-kernel selection differs from the standalone selection"
    ref_idx, ok = _gap_ok(qn, c.k, c, K)
    s = sel.cpu().numpy()
    assert np.array_equal(s[ok], ref_idx[ok])
    assert _same_as_two_launch(o, l, o2, l2), "outputs differ from the two-launch path"
    ro, rl = oracle.block_sparse_attention(qn, c.k, c.v, c.persist_idx, s, c.window_blk0, c.block, c.scale)
    assert_bf16_close(o, ro, "fused-select O")
    assert_lse_close(l, rl, "fused-select LSE")


@pytest.mark.parametrize("d", [128, 64])
def test_fused_select_several_units_per_cta(d):
    """More units than SMs: each CTA's selection warps run ahead over both list buffers."""
    c = _case(97, 96, d, 4, 6)
    q = c.q.to(DEV)
    (o, l, sel), (o2, l2, idx) = _run_pair(c, q, 5)
    assert torch.equal(sel, idx)
    assert _same_as_two_launch(o, l, o2, l2)
    heads, qblocks = [0, 47, 95], [0, 7, 15]
    s = sel.cpu().numpy()
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, s, c.window_blk0, c.block, c.scale,
                                           heads=heads, qblocks=qblocks)
    rows = [r for j in qblocks for r in range(j * 64, j * 64 + 64)]
    assert_bf16_close(to_np(o)[:, rows][:, :, heads], ro[:, rows][:, :, heads], "fused-select O (many units)")
    assert_lse_close(to_np(l)[:, heads][:, :, rows], rl[:, heads][:, :, rows], "fused-select LSE (many units)")


_IID = {}


def _iid():
    if "c" not in _IID:
        _IID["c"] = sparse_iid_case(name="iid")
    return _IID["c"]


@pytest.mark.parametrize("frac", W.SPARSE_TOPK_FRACTIONS)
def test_fused_select_full_config3(frac):
    """Config 3 (i.i.d. recipe) at full size, grouped order: the selection equals the
    oracle's at every K with no row masked, the outputs equal the two-launch path's."""
    c = _iid()
    K = W.topk_for_fraction(frac, c.n_win_blk)
    q, k = c.q.to(DEV), c.k.to(DEV)
    _, _, order = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K, order=True)
    (o, l, sel), (o2, l2, idx) = _run_pair(c, q, K, order)
    assert torch.equal(sel, idx)
    ref = oracle.block_select(c.q, c.k, c.window_blk0, c.n_win_blk, c.block, K)[0]
    assert np.array_equal(sel.cpu().numpy(), ref), f"K={K}"
    assert _same_as_two_launch(o, l, o2, l2), f"K={K}"


def test_order_from_a_fused_selection():
    """vkv_block_order on the in-kernel selection equals the order vkv_block_select
    writes with the same selection (a grouped order for the next call)."""
    c = _iid()
    K = W.topk_for_fraction(W.SPARSE_TOPK_FRACTIONS[1], c.n_win_blk)
    q, k = c.q.to(DEV), c.k.to(DEV)
    (o, l, sel), (_, _, idx) = _run_pair(c, q, K, None)
    _, _, ref_order = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K, order=True)
    order = vk().block_order(sel)
    torch.cuda.synchronize()
    assert torch.equal(sel, idx)
    assert torch.equal(order, ref_order)
    # and the grouped call with it reproduces the fused result of the grouped order
    (o2, l2, sel2), _ = _run_pair(c, q, K, order)
    assert torch.equal(sel2, sel)


def test_fused_select_full_config3_sampled_natural_order():
    c = _iid()
    K = W.topk_for_fraction(W.SPARSE_TOPK_FRACTIONS[0], c.n_win_blk)
    q = c.q.to(DEV)
    (o, l, sel), (o2, l2, idx) = _run_pair(c, q, K, None)
    assert torch.equal(sel, idx)
    assert _same_as_two_launch(o, l, o2, l2)
    s = sel.cpu().numpy()
    heads, qblocks = [2, 7, 11], [0, 3, 35, 70, 71]
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, s, c.window_blk0, c.block, c.scale,
                                           heads=heads, qblocks=qblocks)
    rows = [r for j in qblocks for r in range(j * 64, j * 64 + 64)]
    assert_bf16_close(to_np(o)[:, rows][:, :, heads], ro[:, rows][:, :, heads], "fused-select config 3 O")
    assert_lse_close(to_np(l)[:, heads][:, :, rows], rl[:, heads][:, :, rows], "fused-select config 3 LSE")


def test_fused_select_batch_of_two():
    c = _case(100, 3, 128, 3, 5, B=2)
    q = c.q.to(DEV)
    (o, l, sel), (o2, l2, idx) = _run_pair(c, q, 4)
    assert torch.equal(sel, idx)
    ref_idx, ok = _gap_ok(c.q, c.k, c, 4)
    assert np.array_equal(sel.cpu().numpy()[ok], ref_idx[ok])
    assert _same_as_two_launch(o, l, o2, l2)
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel.cpu().numpy(), c.window_blk0, c.block,
                                           c.scale)
    assert_bf16_close(o, ro, "fused-select O (B = 2)")
    assert_lse_close(l, rl, "fused-select LSE (B = 2)")


def test_fused_select_largest_window():
    """A window of 512 blocks, the largest the kernel's ranking keys hold (the
    standalone kernel then scores from L2 in another summation order: the planted
    margins keep the choice the same)."""
    c = W.make_block_sparse("fused", seed=101, H=1, d=128, frame_tokens=256, block=64, hist_frames=3,
                            win_frames=128, q_frames=2, n_persist=6)
    assert c.n_win_blk == 512
    q = c.q.to(DEV)
    (o, l, sel), (o2, l2, idx) = _run_pair(c, q, 16)
    assert torch.equal(sel, idx)
    ref_idx, ok = _gap_ok(c.q, c.k, c, 16)
    assert ok.all() and np.array_equal(sel.cpu().numpy(), ref_idx)
    assert _same_as_two_launch(o, l, o2, l2)
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, ref_idx, c.window_blk0, c.block, c.scale)
    assert_bf16_close(o, ro, "fused-select O (512-block window)")
    assert_lse_close(l, rl, "fused-select LSE (512-block window)")


def test_fused_select_without_selection_output():
    c = _case(98, 2, 128, 2, 5)
    q = c.q.to(DEV)
    (o, l, _), (o2, l2, _) = _run_pair(c, q, 3, sel_out=False)
    assert _same_as_two_launch(o, l, o2, l2)


def test_fused_select_bad_order_sets_error_word():
    c = _case(99, 2, 128, 2, 5)
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    n_qblk = c.n_qblk
    perm = np.tile(np.arange(n_qblk, dtype=np.int32), (c.B * c.H, 1))
    perm[1, 2] = n_qblk + 3  # not a query block
    kbar = vk().block_pool(k, c.window_blk0, c.n_win_blk)
    err = err_word()
    vk().chunk_attn_block_sparse(q, k, v, torch.from_numpy(c.persist_idx).to(DEV), None, c.window_blk0,
                                 c.n_win_blk, scale=c.scale, err=err, qblk_order=torch.from_numpy(perm).to(DEV),
                                 kbar=kbar, topk=3)
    torch.cuda.synchronize()
    assert int(err.item()) == vk().DEVERR_BAD_INDEX
    # the device stays usable
    (o, l, sel), (o2, l2, idx) = _run_pair(c, q, 3)
    assert torch.equal(sel, idx) and _same_as_two_launch(o, l, o2, l2)
