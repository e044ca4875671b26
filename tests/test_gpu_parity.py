"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases are compared element by element; the full-size configurations
are run in the launch configuration the benchmark times and checked on
sampled rows the oracle computes one by one.
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


def run_segments(c, merged=True):
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    err = err_word()
    res = vk().chunk_attn_segments(q, k, v, c.branches, scale=c.scale, merged=merged, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return res


def check_segments_full(c, res):
    ref = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale)
    for i in range(len(c.branches)):
        assert_bf16_close(res["o"][i], ref["branch_o"][i], f"O branch {i}")
        assert_lse_close(res["lse"][i], ref["branch_lse"][i], f"LSE branch {i}")
    if len(c.branches) == 2 and res.get("o_merged") is not None:
        assert_bf16_close(res["o_merged"], ref["dense_o"], "O merged vs dense")
        assert_lse_close(res["lse_merged"], ref["dense_lse"], "LSE merged vs dense")


# ---------------------------------------------------------------------------
# mode 1: segments (dual branch)
# ---------------------------------------------------------------------------
def test_tiny_dual_branch_config():
    c = W.cfg_tiny()
    check_segments_full(c, run_segments(c))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("frame,qf,hf", [(200, 2, 5), (96, 3, 2), (130, 1, 3)])
def test_dual_branch_ragged_tiles(d, frame, qf, hf):
    """Segments and query chunks that are not multiples of the 128-row tile."""
    c = W.make_dual_branch("mid", 40 + d + frame, H=3, d=d, frame_tokens=frame, q_frames=qf, hist_frames=hf)
    check_segments_full(c, run_segments(c))


def test_single_branch_and_batch():
    c = W.make_dual_branch("b2", 51, H=2, d=128, frame_tokens=160, q_frames=2, hist_frames=3, B=2)
    c.branches = [c.branches[0] + c.branches[1]]
    res = run_segments(c, merged=False)
    ref = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale)
    assert_bf16_close(res["o"][0], ref["branch_o"][0], "O")
    assert_lse_close(res["lse"][0], ref["branch_lse"][0], "LSE")


def test_empty_branch_gives_zero_and_neg_inf():
    c = W.make_dual_branch("e", 52, H=2, d=128, frame_tokens=128, q_frames=1, hist_frames=2)
    c.branches = [c.branches[0], []]
    res = run_segments(c)
    ref = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale)
    assert_bf16_close(res["o"][0], ref["branch_o"][0], "O local")
    assert np.all(to_np(res["o"][1]) == 0)
    assert np.all(np.isneginf(to_np(res["lse"][1])))
    assert_bf16_close(res["o_merged"], ref["dense_o"], "O merged")
    assert_lse_close(res["lse_merged"], ref["dense_lse"], "LSE merged")


def test_short_query_chunks():
    for Lq in (1, 17, 127, 129):
        c = W.make_dual_branch("s", 60 + Lq, H=2, d=128, frame_tokens=192, q_frames=1, hist_frames=2,
                               q_tokens=Lq)
        check_segments_full(c, run_segments(c))


def test_large_logit_range_rescaling():
    """Keys with growing norm force the running maximum to move many times."""
    c = W.make_dual_branch("r", 70, H=2, d=128, frame_tokens=256, q_frames=1, hist_frames=3)
    scale = torch.linspace(0.2, 6.0, c.Lkv).reshape(1, -1, 1, 1)
    c.k = (c.k.float() * scale).to(torch.bfloat16)
    check_segments_full(c, run_segments(c))


def test_repeat_calls_are_deterministic():
    c = W.make_dual_branch("d", 71, H=4, d=128, frame_tokens=300, q_frames=2, hist_frames=4)
    a = run_segments(c)
    b = run_segments(c)
    for x, y in zip(a["o"] + [a["o_merged"]], b["o"] + [b["o_merged"]]):
        assert torch.equal(x, y)


def _sampled_rows(Lq):
    return sorted(set([0, 1, 63, 64, 127, 128, Lq // 2, Lq - 73, Lq - 72, Lq - 1]))


@pytest.mark.parametrize("cfg", ["wan13b", "wan14b"])
def test_full_size_dense_configs_sampled(cfg):
    c = W.cfg_wan13b() if cfg == "wan13b" else W.cfg_wan14b()
    res = run_segments(c)
    rows = _sampled_rows(c.Lq)
    heads = [0, c.H // 2, c.H - 1]
    ref = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale, heads=heads, rows=rows)
    sel = lambda t: to_np(t)[:, rows][:, :, heads]  # noqa: E731
    sel_l = lambda t: to_np(t)[:, heads][:, :, rows]  # noqa: E731
    for i in range(2):
        assert_bf16_close(sel(res["o"][i]), ref["branch_o"][i], f"{cfg} O{i}")
        assert_lse_close(sel_l(res["lse"][i]), ref["branch_lse"][i], f"{cfg} LSE{i}")
    assert_bf16_close(sel(res["o_merged"]), ref["dense_o"], f"{cfg} merged")
    assert_lse_close(sel_l(res["lse_merged"]), ref["dense_lse"], f"{cfg} merged LSE")
    # property over every row: merged LSE = logaddexp of the branch LSEs
    la, lb, lm = (to_np(x) for x in (res["lse"][0], res["lse"][1], res["lse_merged"]))
    assert np.abs(np.logaddexp(la, lb) - lm).max() < 1e-3
    assert np.isfinite(to_np(res["o_merged"])).all()


@pytest.mark.parametrize("H,q_tokens", [(160, 300), (300, 100)])
def test_many_heads_odd_tile_count(H, q_tokens):
    """Many heads with an odd number of query tiles (one-tile units beside pairs,
    more units than SMs): every output of every head matches the oracle."""
    c = W.make_dual_branch("m", 90 + H, H=H, d=128, frame_tokens=100, q_frames=3, hist_frames=2,
                           q_tokens=q_tokens)
    res = run_segments(c)
    ref = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale)
    for i in range(2):
        assert_bf16_close(res["o"][i], ref["branch_o"][i], f"H{H} O{i}")
        assert_lse_close(res["lse"][i], ref["branch_lse"][i], f"H{H} LSE{i}")
    assert_bf16_close(res["o_merged"], ref["dense_o"], f"H{H} merged")
    assert_lse_close(res["lse_merged"], ref["dense_lse"], f"H{H} merged LSE")


def test_stalled_pipeline_reports_timeout_and_device_stays_usable():
    """A cache-tile copy that never arrives (withheld on purpose): the bounded wait
    for it runs out, the call reports VKV_DEVERR_TIMEOUT and the next call on the
    same context is correct."""
    v = vk()
    c = W.cfg_tiny()
    q, k, vv = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    err = err_word()
    with v.using_test_library():  # the test aid exists only in the test build
        assert v.vkv_debug_withhold_copy(1) == 0
        try:
            v.chunk_attn_segments(q, k, vv, c.branches, scale=c.scale, err=err)
            torch.cuda.synchronize()
        finally:
            v.vkv_debug_withhold_copy(0)
        assert int(err.item()) == v.DEVERR_TIMEOUT
        check_segments_full(c, run_segments(c))
    check_segments_full(c, run_segments(c))  # and the production library on the same context


# ---------------------------------------------------------------------------
# standalone LSE merge
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("neg_inf", [0.0, 0.2])
def test_lse_merge_kernel(neg_inf):
    oa, la, ob, lb = W.make_merge_inputs(5, 2, 333, 3, 128, neg_inf_frac=neg_inf)
    o, l = vk().lse_merge(oa.to(DEV), la.to(DEV), ob.to(DEV), lb.to(DEV))
    torch.cuda.synchronize()
    ro, rl = oracle.lse_merge(to_np(oa), np.moveaxis(to_np(la), 1, 2), to_np(ob), np.moveaxis(to_np(lb), 1, 2))
    assert_bf16_close(o, ro, "merge O")
    assert_lse_close(l, np.moveaxis(rl, 2, 1), "merge LSE")


def test_lse_merge_matches_fused_merge():
    c = W.make_dual_branch("m", 72, H=3, d=128, frame_tokens=256, q_frames=2, hist_frames=4)
    res = run_segments(c)
    o, l = vk().lse_merge(res["o"][0], res["lse"][0], res["o"][1], res["lse"][1])
    torch.cuda.synchronize()
    ref = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale)
    assert_bf16_close(o, ref["dense_o"], "standalone merge vs dense")
    assert_lse_close(l, ref["dense_lse"], "standalone merge LSE")


# ---------------------------------------------------------------------------
# mode 2: block selection + persistent/top-K block-sparse attention
# ---------------------------------------------------------------------------
def _small_sparse(seed=80, H=2, d=128, hist=3, win=4, qf=2, n_persist=5):
    return W.make_block_sparse("small", seed=seed, H=H, d=d, frame_tokens=256, block=64, hist_frames=hist,
                               win_frames=win, q_frames=qf, n_persist=n_persist)


@pytest.mark.parametrize("topk", [1, 3, 7, 16])
def test_block_select_exact_small(topk):
    c = _small_sparse()
    q, k = c.q.to(DEV), c.k.to(DEV)
    idx, sc = vk().block_select(q, k, c.window_blk0, c.n_win_blk, topk, scores=True)
    torch.cuda.synchronize()
    ref_idx, ref_sc = oracle.block_select(c.q, c.k, c.window_blk0, c.n_win_blk, c.block, topk)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.abs(to_np(sc) - ref_sc).max() < 1e-3


def test_block_select_exact_full_sparse_config():
    c = W.cfg_sparse()
    q, k = c.q.to(DEV), c.k.to(DEV)
    ref_s = oracle.block_scores(c.q, c.k, c.window_blk0, c.n_win_blk, c.block)
    for frac in W.SPARSE_TOPK_FRACTIONS:
        K = W.topk_for_fraction(frac, c.n_win_blk)
        idx, _ = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), oracle.select_topk(ref_s, K)), f"K={K}"


_IID = {}


def _iid_sparse():
    """Config 3 as stated: i.i.d. N(0,1) keys plus the planted offsets, query blocks
    redrawn until the fp64 top-K gap is >= 0.05 at K = 9, 18, 36 (built once)."""
    if "c" not in _IID:
        _IID["c"] = sparse_iid_case(name="iid")
    return _IID["c"]


def test_block_select_exact_iid_config3():
    """Every selected index set bit-exact at K = 9 / 18 / 36 / 144 on the i.i.d.
    recipe, no row masked; scores within 1e-3; the cached-representative path and
    the no-workspace entry point give the same sets."""
    c = _iid_sparse()
    q, k = c.q.to(DEV), c.k.to(DEV)
    ref_s = oracle.block_scores(c.q, c.k, c.window_blk0, c.n_win_blk, c.block)
    kbar = vk().block_pool(k, c.window_blk0, c.n_win_blk)
    for frac in W.SPARSE_TOPK_FRACTIONS:
        K = W.topk_for_fraction(frac, c.n_win_blk)
        ref_idx = oracle.select_topk(ref_s, K)
        idx, sc = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K, scores=True)
        idx_c, _ = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K, kbar=kbar)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), ref_idx), f"K={K}"
        assert np.array_equal(idx_c.cpu().numpy(), ref_idx), f"K={K} (cached representatives)"
        assert np.abs(to_np(sc) - ref_s).max() < 1e-3


@pytest.mark.parametrize("K", [9, 36])
def test_iid_config3_attention_sampled(K):
    c = _iid_sparse()
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    idx, _, order = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K, order=True)
    err = err_word()
    o, l = vk().chunk_attn_block_sparse(q, k, v, torch.from_numpy(c.persist_idx).to(DEV), idx,
                                        c.window_blk0, c.n_win_blk, scale=c.scale, err=err, qblk_order=order)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    sel = idx.cpu().numpy()
    assert np.array_equal(sel, oracle.block_select(c.q, c.k, c.window_blk0, c.n_win_blk, c.block, K)[0])
    heads, qblocks = [1, 6, 10], [0, 2, 36, 69, 71]
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale,
                                           heads=heads, qblocks=qblocks)
    rows = [r for j in qblocks for r in range(j * 64, j * 64 + 64)]
    assert_bf16_close(to_np(o)[:, rows][:, :, heads], ro[:, rows][:, :, heads], f"iid sparse K={K}")
    assert_lse_close(to_np(l)[:, heads][:, :, rows], rl[:, heads][:, :, rows], f"iid sparse LSE K={K}")


@pytest.mark.parametrize("topk", [1, 4, 16])
def test_block_sparse_attention_small_random_selection(topk):
    c = _small_sparse(seed=81)
    sel = W.random_selection(9 + topk, c.B * c.H, c.n_qblk, c.n_win_blk, topk)
    err = err_word()
    o, l = vk().chunk_attn_block_sparse(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV),
                                        torch.from_numpy(c.persist_idx).to(DEV), torch.from_numpy(sel).to(DEV),
                                        c.window_blk0, c.n_win_blk, scale=c.scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale)
    assert_bf16_close(o, ro, "sparse O")
    assert_lse_close(l, rl, "sparse LSE")


def test_block_sparse_no_persistent_blocks():
    c = _small_sparse(seed=82, n_persist=0)
    sel = W.random_selection(3, c.B * c.H, c.n_qblk, c.n_win_blk, 5)
    o, l = vk().chunk_attn_block_sparse(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV),
                                        torch.zeros((c.B * c.H, 0), dtype=torch.int32, device=DEV),
                                        torch.from_numpy(sel).to(DEV), c.window_blk0, c.n_win_blk, scale=c.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx[:, :0], sel, c.window_blk0, c.block,
                                           c.scale)
    assert_bf16_close(o, ro, "sparse O (no persistent)")
    assert_lse_close(l, rl, "sparse LSE (no persistent)")


def test_block_sparse_all_blocks_equals_dense_segments():
    c = _small_sparse(seed=83)
    K = c.n_win_blk
    sel = np.tile(np.arange(K, dtype=np.int32), (c.B * c.H, c.n_qblk, 1))
    o, l = vk().chunk_attn_block_sparse(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV),
                                        torch.from_numpy(c.persist_idx).to(DEV), torch.from_numpy(sel).to(DEV),
                                        c.window_blk0, c.n_win_blk, scale=c.scale)
    torch.cuda.synchronize()
    for h in range(c.H):
        blocks = list(c.persist_idx[h]) + list(range(c.window_blk0, c.window_blk0 + K))
        segs = [(int(b) * 64, 64) for b in blocks]
        ref = oracle.segment_attention(c.q, c.k, c.v, [segs], c.scale, heads=[h])
        assert_bf16_close(to_np(o)[:, :, h:h + 1], ref["dense_o"], "K=all vs dense")
        assert_lse_close(to_np(l)[:, h:h + 1], ref["dense_lse"], "K=all vs dense LSE")


@pytest.mark.parametrize("frac", W.SPARSE_TOPK_FRACTIONS)
def test_full_sparse_config_sampled(frac):
    c = W.cfg_sparse()
    K = W.topk_for_fraction(frac, c.n_win_blk)
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    idx, _ = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K)
    err = err_word()
    o, l = vk().chunk_attn_block_sparse(q, k, v, torch.from_numpy(c.persist_idx).to(DEV), idx,
                                        c.window_blk0, c.n_win_blk, scale=c.scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    sel = idx.cpu().numpy()
    heads, qblocks = [0, 7, 11], [0, 1, 35, 70, 71]
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale,
                                           heads=heads, qblocks=qblocks)
    rows = [r for j in qblocks for r in range(j * 64, j * 64 + 64)]
    assert_bf16_close(to_np(o)[:, rows][:, :, heads], ro[:, rows][:, :, heads], f"sparse K={K}")
    assert_lse_close(to_np(l)[:, heads][:, :, rows], rl[:, heads][:, :, rows], f"sparse LSE K={K}")


def test_sparse_bad_index_sets_error_word():
    c = _small_sparse(seed=84)
    sel = W.random_selection(4, c.B * c.H, c.n_qblk, c.n_win_blk, 3)
    sel[0, 0, 0] = c.n_win_blk + 5  # outside the window
    err = err_word()
    vk().chunk_attn_block_sparse(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV), torch.from_numpy(c.persist_idx).to(DEV),
                                 torch.from_numpy(sel).to(DEV), c.window_blk0, c.n_win_blk, scale=c.scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == vk().DEVERR_BAD_INDEX


def _order_reference(sel):
    """Query-block order of the grouping aid: ascending (first six selected ids, 10 bits
    each, first id most significant), then ascending block index."""
    BH, nq, K = sel.shape
    out = np.zeros((BH, nq), dtype=np.int32)
    for s in range(BH):
        keys = []
        for j in range(nq):
            key = 0
            for e in range(6):
                key = (key << 10) | ((int(sel[s, j, e]) & 1023) if e < K else 0)
            keys.append((key, j))
        out[s] = [j for _, j in sorted(keys)]
    return out


@pytest.mark.parametrize("topk", [1, 9, 36, 144])
def test_block_select_order_definition(topk):
    c = W.cfg_sparse()
    q, k = c.q.to(DEV), c.k.to(DEV)
    idx, _, order = vk().block_select(q, k, c.window_blk0, c.n_win_blk, topk, order=True)
    torch.cuda.synchronize()
    sel = idx.cpu().numpy()
    got = order.cpu().numpy()
    assert np.array_equal(np.sort(got, axis=1), np.tile(np.arange(c.n_qblk), (c.B * c.H, 1)))
    assert np.array_equal(got, _order_reference(sel))


@pytest.mark.parametrize("frame_tokens,qf,topk", [(256, 2, 3), (192, 1, 4), (192, 3, 2)])
def test_block_sparse_grouped_order_matches_oracle(frame_tokens, qf, topk):
    # (192, 1): three query blocks, so the second tile's second block is missing
    c = W.make_block_sparse("grp", seed=85, H=2, d=128, frame_tokens=frame_tokens, block=64, hist_frames=3,
                            win_frames=4, q_frames=qf, n_persist=5)
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    idx, _, order = vk().block_select(q, k, c.window_blk0, c.n_win_blk, topk, order=True)
    err = err_word()
    o, l = vk().chunk_attn_block_sparse(q, k, v, torch.from_numpy(c.persist_idx).to(DEV), idx, c.window_blk0,
                                        c.n_win_blk, scale=c.scale, err=err, qblk_order=order)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, idx.cpu().numpy(), c.window_blk0,
                                           c.block, c.scale)
    assert_bf16_close(o, ro, "sparse O (grouped order)")
    assert_lse_close(l, rl, "sparse LSE (grouped order)")


@pytest.mark.parametrize("seed", [0, 1])
def test_block_sparse_random_query_block_order(seed):
    c = _small_sparse(seed=86 + seed, qf=3)
    sel = W.random_selection(20 + seed, c.B * c.H, c.n_qblk, c.n_win_blk, 4)
    rng = np.random.default_rng(90 + seed)
    perm = np.stack([rng.permutation(c.n_qblk) for _ in range(c.B * c.H)]).astype(np.int32)
    err = err_word()
    o, l = vk().chunk_attn_block_sparse(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV),
                                        torch.from_numpy(c.persist_idx).to(DEV), torch.from_numpy(sel).to(DEV),
                                        c.window_blk0, c.n_win_blk, scale=c.scale, err=err,
                                        qblk_order=torch.from_numpy(perm).to(DEV))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale)
    assert_bf16_close(o, ro, "sparse O (random order)")
    assert_lse_close(l, rl, "sparse LSE (random order)")


@pytest.mark.parametrize("frac", [W.SPARSE_TOPK_FRACTIONS[0], W.SPARSE_TOPK_FRACTIONS[2]])
def test_full_sparse_config_grouped_sampled(frac):
    c = W.cfg_sparse()
    K = W.topk_for_fraction(frac, c.n_win_blk)
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    idx, _, order = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K, order=True)
    err = err_word()
    o, l = vk().chunk_attn_block_sparse(q, k, v, torch.from_numpy(c.persist_idx).to(DEV), idx,
                                        c.window_blk0, c.n_win_blk, scale=c.scale, err=err, qblk_order=order)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    sel = idx.cpu().numpy()
    heads, qblocks = [0, 5, 11], [0, 1, 36, 70, 71]
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale,
                                           heads=heads, qblocks=qblocks)
    rows = [r for j in qblocks for r in range(j * 64, j * 64 + 64)]
    assert_bf16_close(to_np(o)[:, rows][:, :, heads], ro[:, rows][:, :, heads], f"grouped sparse K={K}")
    assert_lse_close(to_np(l)[:, heads][:, :, rows], rl[:, heads][:, :, rows], f"grouped sparse LSE K={K}")


def test_sparse_bad_query_block_order_sets_error_word():
    c = _small_sparse(seed=88)
    sel = W.random_selection(5, c.B * c.H, c.n_qblk, c.n_win_blk, 3)
    perm = np.tile(np.arange(c.n_qblk, dtype=np.int32), (c.B * c.H, 1))
    perm[1, 2] = c.n_qblk + 3  # not a query block
    err = err_word()
    vk().chunk_attn_block_sparse(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV), torch.from_numpy(c.persist_idx).to(DEV),
                                 torch.from_numpy(sel).to(DEV), c.window_blk0, c.n_win_blk, scale=c.scale, err=err,
                                 qblk_order=torch.from_numpy(perm).to(DEV))
    torch.cuda.synchronize()
    assert int(err.item()) == vk().DEVERR_BAD_INDEX


@pytest.mark.parametrize("d", [128, 64])
def test_block_pool_matches_oracle(d):
    c = _small_sparse(seed=89, d=d)
    k = c.k.to(DEV)
    blk0, n = 3, 20  # the cache holds 7 frames x 4 blocks
    kb = vk().block_pool(k, blk0, n)
    torch.cuda.synchronize()
    kk = oracle.to64(c.k)
    ref = np.stack([oracle.pool_blocks(kk[b, blk0 * 64:(blk0 + n) * 64, h], 64)
                    for b in range(c.B) for h in range(c.H)])
    assert np.abs(to_np(kb) - ref).max() < 1e-5


@pytest.mark.parametrize("topk", [3, 9])
def test_block_select_with_cached_representatives(topk):
    c = W.cfg_sparse()
    q, k = c.q.to(DEV), c.k.to(DEV)
    idx, sc, order = vk().block_select(q, k, c.window_blk0, c.n_win_blk, topk, scores=True, order=True)
    kbar = vk().block_pool(k, c.window_blk0, c.n_win_blk)
    # the cached path must not need k: pass a tensor of the right shape filled with garbage
    junk = torch.full_like(k, float("nan"))
    idx2, sc2, order2 = vk().block_select(q, junk, c.window_blk0, c.n_win_blk, topk, scores=True, order=True,
                                          kbar=kbar)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx2)
    assert torch.equal(sc, sc2)
    assert torch.equal(order, order2)


# ---------------------------------------------------------------------------
# mode 3: ragged per-head cache
# ---------------------------------------------------------------------------
def _run_ragged(c, host=True):
    err = err_word()
    o, l = vk().chunk_attn_ragged(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV),
                                  torch.from_numpy(c.cu_seqlens).to(DEV),
                                  c.cu_seqlens if host else None, scale=c.scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return o, l


@pytest.mark.parametrize("host", [True, False])
def test_ragged_small(host):
    pol = [("anchor", 3), ("wave", 2), ("veil", 0), ("full", 0)]
    c = W.make_ragged("small", seed=90, H=4, d=128, frame_tokens=100, hist_frames=12, q_frames=2, policies=pol)
    o, l = _run_ragged(c, host)
    ro, rl = oracle.ragged_attention(c.q, c.k, c.v, c.cu_seqlens, c.scale)
    assert_bf16_close(o, ro, "ragged O")
    assert_lse_close(l, rl, "ragged LSE")


def test_ragged_all_full_equals_dense():
    pol = [("full", 0)] * 2
    c = W.make_ragged("full", seed=91, H=2, d=128, frame_tokens=96, hist_frames=5, q_frames=2, policies=pol)
    o, l = _run_ragged(c)
    for h in range(2):
        a, b = int(c.cu_seqlens[h]), int(c.cu_seqlens[h + 1])
        kd = c.k[a:b].reshape(1, b - a, 1, 128).expand(1, b - a, 2, 128)
        vd = c.v[a:b].reshape(1, b - a, 1, 128).expand(1, b - a, 2, 128)
        ref = oracle.segment_attention(c.q, kd, vd, [[(0, b - a)]], c.scale, heads=[h])
        assert_bf16_close(to_np(o)[:, :, h:h + 1], ref["dense_o"], "ragged full vs dense")


def test_full_ragged_config_sampled():
    c = W.cfg_ragged()
    assert c.cu_seqlens.tolist()[-1] == 299520
    o, l = _run_ragged(c)
    rows = _sampled_rows(c.Lq)
    heads = [0, 4, 5, 7, 8, 11]
    ro, rl = oracle.ragged_attention(c.q, c.k, c.v, c.cu_seqlens, c.scale, heads=heads, rows=rows)
    assert_bf16_close(to_np(o)[:, rows][:, :, heads], ro, "ragged cfg O")
    assert_lse_close(to_np(l)[:, heads][:, :, rows], rl, "ragged cfg LSE")


def test_ragged_bad_offsets_set_error_word():
    pol = [("anchor", 3), ("wave", 2)]
    c = W.make_ragged("bad", seed=92, H=2, d=128, frame_tokens=64, hist_frames=8, q_frames=1, policies=pol)
    cu = c.cu_seqlens.copy()
    cu[1] = cu[2] + 10  # decreasing
    err = err_word()
    vk().chunk_attn_ragged(c.q.to(DEV), c.k.to(DEV), c.v.to(DEV), torch.from_numpy(cu).to(DEV), None,
                           scale=c.scale, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == vk().DEVERR_BAD_OFFSETS


# ---------------------------------------------------------------------------
# selection edge cases: ties, larger windows, d = 64; merge at d = 64
# ---------------------------------------------------------------------------
def test_block_select_all_ties_pick_lowest_indices():
    """Identical window blocks: every score ties, so top-K = the K lowest block ids."""
    c = _small_sparse(seed=85)
    k = c.k.clone()
    w0 = c.window_blk0 * 64
    blk = k[:, w0:w0 + 64].clone()
    for b in range(c.n_win_blk):
        k[:, w0 + b * 64:w0 + (b + 1) * 64] = blk
    for topk in (1, 5, c.n_win_blk - 1):
        idx, _ = vk().block_select(c.q.to(DEV), k.to(DEV), c.window_blk0, c.n_win_blk, topk)
        torch.cuda.synchronize()
        ref, _ = oracle.block_select(c.q, k, c.window_blk0, c.n_win_blk, c.block, topk)
        assert np.array_equal(ref, np.tile(np.arange(topk), ref.shape[:-1] + (1,)))
        assert np.array_equal(idx.cpu().numpy(), ref)


@pytest.mark.parametrize("win_frames,d", [(75, 128), (175, 64), (40, 64)])
def test_block_select_large_windows(win_frames, d):
    """Windows of 300 / 700 / 160 blocks exercise the wider per-lane instantiations."""
    c = W.make_block_sparse("wide", seed=86 + win_frames, H=2, d=d, frame_tokens=256, block=64, hist_frames=1,
                            win_frames=win_frames, q_frames=1, n_persist=2)
    for topk in (7, c.n_win_blk // 3):
        idx, sc = vk().block_select(c.q.to(DEV), c.k.to(DEV), c.window_blk0, c.n_win_blk, topk, scores=True)
        torch.cuda.synchronize()
        ref_s = oracle.block_scores(c.q, c.k, c.window_blk0, c.n_win_blk, c.block)
        assert np.abs(to_np(sc) - ref_s).max() < 1e-3
        gap = oracle.topk_gap(ref_s, topk)
        exact = gap > 1e-4  # rows whose ranking fp32 scores can resolve
        got = idx.cpu().numpy()
        ref = oracle.select_topk(ref_s, topk)
        assert np.array_equal(got[exact], ref[exact])
        # every row holds topk distinct ascending window ids
        assert np.all(np.diff(got, axis=-1) > 0) and got.min() >= 0 and got.max() < c.n_win_blk


def test_lse_merge_kernel_d64():
    oa, la, ob, lb = W.make_merge_inputs(6, 3, 77, 5, 64, neg_inf_frac=0.1)
    o, l = vk().lse_merge(oa.to(DEV), la.to(DEV), ob.to(DEV), lb.to(DEV))
    torch.cuda.synchronize()
    ro, rl = oracle.lse_merge(to_np(oa), np.moveaxis(to_np(la), 1, 2), to_np(ob), np.moveaxis(to_np(lb), 1, 2))
    assert_bf16_close(o, ro, "merge O d64")
    assert_lse_close(l, np.moveaxis(rl, 2, 1), "merge LSE d64")


def test_lse_merge_in_place():
    oa, la, ob, lb = W.make_merge_inputs(7, 1, 200, 4, 128)
    ref_o, ref_l = oracle.lse_merge(to_np(oa), np.moveaxis(to_np(la), 1, 2), to_np(ob), np.moveaxis(to_np(lb), 1, 2))
    a, al = oa.to(DEV), la.to(DEV)
    vk().lse_merge(a, al, ob.to(DEV), lb.to(DEV), out=(a, al))
    torch.cuda.synchronize()
    assert_bf16_close(a, ref_o, "in-place merge O")
    assert_lse_close(al, np.moveaxis(ref_l, 2, 1), "in-place merge LSE")


# ---------------------------------------------------------------------------
# full size, every row (the launch configuration the bench times, split
# schedules with key-axis pieces included)
# ---------------------------------------------------------------------------
def test_full_size_wan13b_every_row():
    """Wan-1.3B-shaped chunk (its schedule cuts units into ~190 key-axis pieces):
    both branch outputs, their LSEs and the merged output, every element."""
    c = W.cfg_wan13b()
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    assert vk().vkv_chunk_attn_workspace_size(vk().segments_args(q, k, v, c.branches, c.scale)) > 0
    check_segments_full(c, run_segments(c))


def test_full_size_wan14b_every_row():
    """The headline workload (Wan-14B-shaped, 40 heads) in the launch configuration the
    bench times (head-major split schedule, combine kernel, fused merge): both branch
    outputs, their LSEs and the merged output, every element."""
    c = W.cfg_wan14b()
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    assert vk().vkv_chunk_attn_workspace_size(vk().segments_args(q, k, v, c.branches, c.scale)) > 0
    check_segments_full(c, run_segments(c))


def test_full_size_ragged_every_row():
    c = W.cfg_ragged()
    o, l = _run_ragged(c)
    ro, rl = oracle.ragged_attention(c.q, c.k, c.v, c.cu_seqlens, c.scale)
    assert_bf16_close(o, ro, "ragged full O")
    assert_lse_close(l, rl, "ragged full LSE")


@pytest.mark.parametrize("K", [9, 144])
def test_full_size_iid_sparse_every_row(K):
    c = _iid_sparse()
    q, k, v = c.q.to(DEV), c.k.to(DEV), c.v.to(DEV)
    idx, _, order = vk().block_select(q, k, c.window_blk0, c.n_win_blk, K, order=True)
    err = err_word()
    o, l = vk().chunk_attn_block_sparse(q, k, v, torch.from_numpy(c.persist_idx).to(DEV), idx,
                                        c.window_blk0, c.n_win_blk, scale=c.scale, err=err, qblk_order=order)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    sel = idx.cpu().numpy()
    ro, rl = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale)
    assert_bf16_close(o, ro, f"iid sparse full O K={K}")
    assert_lse_close(l, rl, f"iid sparse full LSE K={K}")
