"""Pins for the CPU oracle: it is checked against things other than itself.

* brute force: an independent pure-Python loop (no matrix products, the LSE
  taken first and the weights as exp(s - LSE)) on small inputs;
* hand-worked cases in tests/golden/hand_cases.json;
* the decomposition the ISPA summary relies on (section 2 step 1): merging
  the local and history branches by their LSE equals attention over the union;
* closed forms: constant keys give the mean of V and LSE = s + ln|J|;
* invariances: key order, a common shift of all keys, a constant added to V;
* reductions: top-K with K = every block equals dense attention over
  persistent + window blocks (Sparse Forcing summary, PBSA); a ragged cache in
  which every head keeps every frame equals dense attention (Pyramid Forcing
  summary, section 3);
* generator recipe checks (frame lists, offsets, the planted top-K margin).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from kv_cache_attention_chunk_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _f(x):
    return -math.inf if x == "-inf" else float(x)


def brute_attend(q, k, v, scale):
    """Pure-Python softmax attention: LSE first, then O = sum exp(s - LSE) v."""
    n, m, dv = len(q), len(k), len(v[0]) if len(v) else 0
    o, lse = [], []
    for i in range(n):
        s = [scale * math.fsum(q[i][c] * k[j][c] for c in range(len(q[i]))) for j in range(m)]
        mx = max(s)
        L = mx + math.log(math.fsum(math.exp(x - mx) for x in s))
        o.append([math.fsum(math.exp(s[j] - L) * v[j][c] for j in range(m)) for c in range(dv)])
        lse.append(L)
    return np.array(o), np.array(lse)


# ---------------------------------------------------------------------------
# hand-worked cases
# ---------------------------------------------------------------------------
with open(os.path.join(GOLD, "hand_cases.json")) as fh:
    HAND = json.load(fh)


@pytest.mark.parametrize("case", HAND["attend"], ids=lambda c: c["name"])
def test_attend_hand_cases(case):
    o, lse = oracle.attend(np.array(case["q"], float), np.array(case["k"], float),
                           np.array(case["v"], float), case["scale"])
    np.testing.assert_allclose(o, np.array(case["o"], float), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.array(case["lse"], float), rtol=0, atol=1e-12)


@pytest.mark.parametrize("case", HAND["merge"], ids=lambda c: c["name"])
def test_merge_hand_cases(case):
    o, lse = oracle.lse_merge(np.array([case["o_a"]], float), np.array([_f(case["lse_a"])]),
                              np.array([case["o_b"]], float), np.array([_f(case["lse_b"])]))
    np.testing.assert_allclose(o[0], np.array(case["o"], float), rtol=0, atol=1e-12)
    exp = _f(case["lse"])
    if math.isinf(exp):
        assert np.isneginf(lse[0])
    else:
        assert abs(lse[0] - exp) < 1e-12


@pytest.mark.parametrize("case", HAND["topk"], ids=lambda c: f"{c['scores']}-k{c['k']}")
def test_topk_hand_cases(case):
    idx = oracle.select_topk(np.array(case["scores"], float), case["k"])
    assert idx.tolist() == case["idx"]


# ---------------------------------------------------------------------------
# brute force
# ---------------------------------------------------------------------------
def test_attend_brute_force_small():
    rng = np.random.default_rng(11)
    for n, m, d in [(1, 1, 1), (3, 5, 4), (7, 2, 3), (4, 9, 8)]:
        q, k, v = rng.standard_normal((n, d)), rng.standard_normal((m, d)), rng.standard_normal((m, d + 1))
        o, lse = oracle.attend(q, k, v, 0.7)
        bo, bl = brute_attend(q.tolist(), k.tolist(), v.tolist(), 0.7)
        np.testing.assert_allclose(o, bo, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, bl, rtol=0, atol=1e-12)


def test_segment_attention_brute_force_tiny_config():
    """Config 1 (tiny dual-branch), a sample of rows, checked loop by loop."""
    c = W.cfg_tiny()
    rows = [0, 17, 63]
    res = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale, rows=rows)
    q, k, v = oracle.to64(c.q), oracle.to64(c.k), oracle.to64(c.v)
    for h in range(c.H):
        for bi, br in enumerate(c.branches):
            toks = [t for s, n in br for t in range(s, s + n)]
            bo, bl = brute_attend(q[0, rows, h].tolist(), k[0, toks, h].tolist(), v[0, toks, h].tolist(), c.scale)
            np.testing.assert_allclose(res["branch_o"][bi][0, :, h], bo, rtol=0, atol=1e-11)
            np.testing.assert_allclose(res["branch_lse"][bi][0, h], bl, rtol=0, atol=1e-11)
        toks = [t for br in c.branches for s, n in br for t in range(s, s + n)]
        bo, bl = brute_attend(q[0, rows, h].tolist(), k[0, toks, h].tolist(), v[0, toks, h].tolist(), c.scale)
        np.testing.assert_allclose(res["merged_o"][0, :, h], bo, rtol=0, atol=1e-11)
        np.testing.assert_allclose(res["merged_lse"][0, h], bl, rtol=0, atol=1e-11)


# ---------------------------------------------------------------------------
# decomposition, closed forms, invariances
# ---------------------------------------------------------------------------
def test_branch_merge_equals_dense_tiny():
    c = W.cfg_tiny()
    res = oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale)
    np.testing.assert_allclose(res["merged_o"], res["dense_o"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["merged_lse"], res["dense_lse"], rtol=0, atol=1e-12)
    # the branch LSEs themselves combine by log-add-exp
    la, lb = res["branch_lse"]
    np.testing.assert_allclose(np.logaddexp(la, lb), res["dense_lse"], rtol=0, atol=1e-12)


def test_merge_three_way_split_equals_dense():
    rng = np.random.default_rng(5)
    q, k, v = rng.standard_normal((6, 16)), rng.standard_normal((40, 16)), rng.standard_normal((40, 16))
    parts = [oracle.attend(q, k[a:b], v[a:b], 0.25) for a, b in [(0, 7), (7, 31), (31, 40)]]
    o, l = parts[0]
    for po, pl in parts[1:]:
        o, l = oracle.lse_merge(o, l, po, pl)
    do, dl = oracle.attend(q, k, v, 0.25)
    np.testing.assert_allclose(o, do, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, dl, rtol=0, atol=1e-12)


def test_constant_keys_give_mean_of_v():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((5, 8))
    kk = rng.standard_normal(8)
    k = np.tile(kk, (13, 1))
    v = rng.standard_normal((13, 6))
    o, lse = oracle.attend(q, k, v, 0.3)
    np.testing.assert_allclose(o, np.tile(v.mean(axis=0), (5, 1)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, 0.3 * q @ kk + math.log(13), rtol=0, atol=1e-12)


def test_invariances():
    rng = np.random.default_rng(4)
    q, k, v = rng.standard_normal((4, 8)), rng.standard_normal((11, 8)), rng.standard_normal((11, 5))
    o, lse = oracle.attend(q, k, v, 0.5)
    p = rng.permutation(11)
    o2, l2 = oracle.attend(q, k[p], v[p], 0.5)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(l2, lse, atol=1e-12)
    w = rng.standard_normal(8)
    o3, l3 = oracle.attend(q, k + w, v, 0.5)
    np.testing.assert_allclose(o3, o, atol=1e-12)
    np.testing.assert_allclose(l3, lse + 0.5 * q @ w, atol=1e-12)
    c = rng.standard_normal(5)
    o4, l4 = oracle.attend(q, k, v + c, 0.5)
    np.testing.assert_allclose(o4, o + c, atol=1e-12)
    np.testing.assert_allclose(l4, lse, atol=1e-12)


def test_empty_key_set():
    o, lse = oracle.attend(np.ones((2, 4)), np.zeros((0, 4)), np.zeros((0, 3)), 1.0)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_merge_is_symmetric_and_handles_infinities():
    rng = np.random.default_rng(8)
    oa, ob = rng.standard_normal((50, 4)), rng.standard_normal((50, 4))
    la, lb = rng.standard_normal(50) * 3, rng.standard_normal(50) * 3
    la[::7] = -np.inf
    lb[::11] = -np.inf
    o1, l1 = oracle.lse_merge(oa, la, ob, lb)
    o2, l2 = oracle.lse_merge(ob, lb, oa, la)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_array_equal(np.isneginf(l1), np.isneginf(l2))
    only_b = np.isneginf(la) & ~np.isneginf(lb)
    np.testing.assert_allclose(o1[only_b], ob[only_b], atol=0)
    np.testing.assert_allclose(l1[only_b], lb[only_b], atol=0)


# ---------------------------------------------------------------------------
# blockified scoring and top-K
# ---------------------------------------------------------------------------
def test_pool_blocks_closed_forms():
    x = np.repeat(np.arange(5.0)[:, None], 4, axis=0).reshape(20, 1) * np.ones((1, 3))
    p = oracle.pool_blocks(x, 4)
    np.testing.assert_allclose(p, np.arange(5.0)[:, None] * np.ones((1, 3)))
    y = np.arange(10.0)[:, None]
    np.testing.assert_allclose(oracle.pool_blocks(y, 4)[:, 0], [1.5, 5.5, 8.5])  # last block: mean of 8, 9


def test_select_topk_brute_force_with_ties():
    rng = np.random.default_rng(9)
    for trial in range(50):
        n = int(rng.integers(1, 40))
        s = np.round(rng.standard_normal(n), 1)  # many ties
        kk = int(rng.integers(1, n + 1))
        ref = sorted(sorted(range(n), key=lambda i: (-s[i], i))[:kk])
        assert oracle.select_topk(s, kk).tolist() == ref


def test_block_scores_match_pooled_dot_products_by_loop():
    c = W.make_block_sparse("small", seed=21, H=2, d=16, frame_tokens=64, block=16,
                            hist_frames=2, win_frames=2, q_frames=1, n_persist=3)
    s = oracle.block_scores(c.q, c.k, c.window_blk0, c.n_win_blk, c.block)
    q, k = oracle.to64(c.q), oracle.to64(c.k)
    for h in range(c.H):
        for j in range(c.n_qblk):
            qbar = [math.fsum(q[0, j * 16 + t, h, x] for t in range(16)) / 16 for x in range(16)]
            for b in range(c.n_win_blk):
                r0 = (c.window_blk0 + b) * 16
                kbar = [math.fsum(k[0, r0 + t, h, x] for t in range(16)) / 16 for x in range(16)]
                assert abs(s[h, j, b] - math.fsum(a * bb for a, bb in zip(qbar, kbar))) < 1e-12


def test_sparse_with_all_blocks_equals_dense():
    c = W.make_block_sparse("small", seed=22, H=2, d=32, frame_tokens=128, block=32,
                            hist_frames=3, win_frames=2, q_frames=1, n_persist=4)
    K = c.n_win_blk
    sel, _ = oracle.block_select(c.q, c.k, c.window_blk0, c.n_win_blk, c.block, K)
    assert np.all(sel == np.arange(K))
    o, lse = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale)
    for h in range(c.H):
        blocks = list(c.persist_idx[h]) + list(range(c.window_blk0, c.window_blk0 + K))
        segs = [(int(b) * c.block, c.block) for b in blocks]
        res = oracle.segment_attention(c.q, c.k, c.v, [segs], c.scale, heads=[h])
        np.testing.assert_allclose(o[:, :, h:h + 1], res["dense_o"], atol=1e-12)
        np.testing.assert_allclose(lse[:, h:h + 1], res["dense_lse"], atol=1e-12)


def test_sparse_brute_force_one_block():
    c = W.make_block_sparse("small", seed=23, H=1, d=8, frame_tokens=32, block=8,
                            hist_frames=2, win_frames=2, q_frames=1, n_persist=2)
    sel = W.random_selection(1, 1, c.n_qblk, c.n_win_blk, 3)
    o, lse = oracle.block_sparse_attention(c.q, c.k, c.v, c.persist_idx, sel, c.window_blk0, c.block, c.scale,
                                           qblocks=[2])
    q, k, v = oracle.to64(c.q), oracle.to64(c.k), oracle.to64(c.v)
    blocks = list(c.persist_idx[0]) + [c.window_blk0 + int(x) for x in sel[0, 2]]
    toks = [b * 8 + t for b in blocks for t in range(8)]
    bo, bl = brute_attend(q[0, 16:24, 0].tolist(), k[0, toks, 0].tolist(), v[0, toks, 0].tolist(), c.scale)
    np.testing.assert_allclose(o[0, 16:24, 0], bo, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0, 16:24], bl, atol=1e-12)
    assert np.isnan(o[0, 0, 0]).all()  # unsampled rows stay NaN


# ---------------------------------------------------------------------------
# ragged
# ---------------------------------------------------------------------------
def test_ragged_all_full_equals_dense():
    pol = [("full", 0)] * 3
    c = W.make_ragged("full", seed=31, H=3, d=16, frame_tokens=8, hist_frames=6, q_frames=2, policies=pol)
    o, lse = oracle.ragged_attention(c.q, c.k, c.v, c.cu_seqlens, c.scale)
    L = c.cu_seqlens[1] - c.cu_seqlens[0]
    for h in range(3):
        kk = c.k[c.cu_seqlens[h]:c.cu_seqlens[h + 1]]
        vv = c.v[c.cu_seqlens[h]:c.cu_seqlens[h + 1]]
        kd = kk.reshape(1, L, 1, 16).expand(1, L, 3, 16)
        vd = vv.reshape(1, L, 1, 16).expand(1, L, 3, 16)
        res = oracle.segment_attention(c.q, kd, vd, [[(0, int(L))]], c.scale, heads=[h])
        np.testing.assert_allclose(o[:, :, h:h + 1], res["dense_o"], atol=1e-12)
        np.testing.assert_allclose(lse[:, h:h + 1], res["dense_lse"], atol=1e-12)


def test_ragged_brute_force_small():
    pol = [("anchor", 2), ("wave", 2), ("veil", 0)]
    c = W.make_ragged("small", seed=32, H=3, d=4, frame_tokens=3, hist_frames=8, q_frames=1, policies=pol)
    o, lse = oracle.ragged_attention(c.q, c.k, c.v, c.cu_seqlens, c.scale)
    q = oracle.to64(c.q)
    kf, vf = oracle.to64(c.k), oracle.to64(c.v)
    for h in range(3):
        a, b = int(c.cu_seqlens[h]), int(c.cu_seqlens[h + 1])
        bo, bl = brute_attend(q[0, :, h].tolist(), kf[a:b].tolist(), vf[a:b].tolist(), c.scale)
        np.testing.assert_allclose(o[0, :, h], bo, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], bl, atol=1e-12)


# ---------------------------------------------------------------------------
# input recipes
# ---------------------------------------------------------------------------
def test_ragged_frames_and_offsets_match_hand_worked_recipe():
    g = json.load(open(os.path.join(GOLD, "ragged_cfg4.json")))
    names = ["anchor"] * 4 + ["wave2", "wave3", "wave4", "wave5"] + ["veil"] * 4
    for (pol, par), name in zip(W.pyramid_policies(12), names):
        fr = W.pyramid_head_frames(pol, 60, 3, par)
        exp = [tuple(x) if isinstance(x, list) else x for x in g["frames"][name]]
        assert fr == exp
    lens = [len(W.pyramid_head_frames(p, 60, 3, a)) * g["frame_tokens"] for p, a in W.pyramid_policies(12)]
    assert lens == g["lengths"] and sum(lens) == g["total"]
    assert np.cumsum([0] + lens).tolist() == g["cu_seqlens"]


def test_veil_merge_is_pairwise_token_mean():
    pol = [("veil", 0)]
    c = W.make_ragged("v", seed=33, H=1, d=4, frame_tokens=2, hist_frames=12, q_frames=1, policies=pol)
    fr = c.frames[0]
    assert fr[1] == (2, 3) and fr[-1] == 12
    assert c.cu_seqlens.tolist() == [0, len(fr) * 2]


def test_dual_branch_layout():
    c = W.cfg_tiny()
    assert c.branches == [[(0, 64), (320, 64)], [(64, 256)]]
    assert (c.Lq, c.Lkv, c.H, c.d) == (64, 384, 2, 64)
    loc, hist = W.dual_branch_layout(1560, 1, 20, 3)
    assert loc == [(0, 1560), (32760, 4680)] and hist == [(1560, 31200)]


def test_wan13b_shape_matches_cache_size_on_videomla_page():
    """12 heads x 128 x 1560 tokens x 21 frames x K,V x 2 B x 30 layers ~ 6.0 GB."""
    gb = 12 * 128 * 1560 * 21 * 2 * 2 * 30 / 1e9
    assert abs(gb - 6.0) < 0.05


def test_visited_flop_counts():
    loc, hist = W.dual_branch_layout(1560, 1, 20, 3)
    assert oracle.visited_flops_segments(1, 40, 4680, 128, [loc, hist]) == 4 * 128 * 40 * 4680 * 37440
    assert abs(oracle.visited_flops_segments(1, 12, 4680, 128, [loc, hist]) / 1e12 - 1.0765) < 1e-3
    assert abs(oracle.visited_flops_sparse(1, 12, 4608, 128, 64, 32, 9) / 1e9 - 74.3) < 0.1
    cu = json.load(open(os.path.join(GOLD, "ragged_cfg4.json")))["cu_seqlens"]
    assert abs(oracle.visited_flops_ragged(1, 12, 4680, 128, cu) / 1e9 - 717.7) < 0.1


@pytest.mark.slow
def test_planted_topk_margin_full_sparse_config():
    """Config 3: every (head, query block) has a margin >= 0.05 at K = 9, 18, 36."""
    c = W.cfg_sparse()
    s = oracle.block_scores(c.q, c.k, c.window_blk0, c.n_win_blk, c.block)
    for frac in W.SPARSE_TOPK_FRACTIONS[:3]:
        K = W.topk_for_fraction(frac, c.n_win_blk)
        assert oracle.topk_gap(s, K).min() >= 0.05


def test_planted_topk_margin_reduced_sparse_config():
    c = W.make_block_sparse("mid", seed=2, H=2, d=128, frame_tokens=1536, block=64,
                            hist_frames=2, win_frames=6, q_frames=3, n_persist=4)
    s = oracle.block_scores(c.q, c.k, c.window_blk0, c.n_win_blk, c.block)
    for K in (9, 18, 36):
        assert oracle.topk_gap(s, K).min() >= 0.05


# ---------------------------------------------------------------------------
# planted mistakes: each plausible error in the oracle must trip a pin above
# ---------------------------------------------------------------------------
def _attend_no_scale(q, k, v, scale):
    return _ORIG_ATTEND(q, k, v, 1.0)


def _attend_log2(q, k, v, scale):
    o, l = _ORIG_ATTEND(q, k, v, scale)
    return o, l / math.log(2)


def _attend_transposed_v(q, k, v, scale):
    o, l = _ORIG_ATTEND(q, k, v[::-1], scale)
    return o, l


def _merge_wrong_sign(o_a, lse_a, o_b, lse_b):
    return _ORIG_MERGE(o_a, lse_a, o_b, -np.asarray(lse_b))


def _topk_wrong_tiebreak(scores, topk):
    n = scores.shape[-1]
    flat = scores.reshape(-1, n)
    out = np.empty((flat.shape[0], topk), dtype=np.int32)
    for i, s in enumerate(flat):
        order = sorted(range(n), key=lambda j: (-s[j], -j))
        out[i] = np.sort(order[:topk])
    return out.reshape(scores.shape[:-1] + (topk,))


_ORIG_ATTEND = oracle.attention.attend
_ORIG_MERGE = oracle.attention.lse_merge


@pytest.mark.parametrize("mutant,target,pins", [
    (_attend_no_scale, "attend", ["test_attend_brute_force_small"]),
    (_attend_log2, "attend", ["test_attend_hand_cases"]),
    (_attend_transposed_v, "attend", ["test_attend_brute_force_small"]),
    (_merge_wrong_sign, "lse_merge", ["test_merge_three_way_split_equals_dense"]),
    (_topk_wrong_tiebreak, "select_topk", ["test_topk_hand_cases"]),
])
def test_planted_mistakes_are_caught(monkeypatch, mutant, target, pins):
    monkeypatch.setattr(oracle.attention, target, mutant)
    monkeypatch.setattr(oracle, target, mutant)
    g = globals()
    caught = False
    for name in pins:
        fn = g[name]
        try:
            if name == "test_attend_hand_cases":
                for c in HAND["attend"]:
                    fn(c)
            elif name == "test_topk_hand_cases":
                for c in HAND["topk"]:
                    fn(c)
            else:
                fn()
        except AssertionError:
            caught = True
    assert caught, f"mutant {mutant.__name__} slipped past {pins}"


@pytest.mark.slow
def test_iid_sparse_config_margin_and_noise():
    """Config 3 with i.i.d. key noise: the redraw loop leaves every (head, query block)
    with a margin >= 0.05 at K = 9, 18, 36, recomputed here on the final tensors, and
    the window keys' noise does not cancel inside a block (it is not antithetic)."""
    from parity_util import sparse_iid_case
    c = sparse_iid_case(name="iid")
    s = oracle.block_scores(c.q, c.k, c.window_blk0, c.n_win_blk, c.block)
    for K in (9, 18, 36):
        assert oracle.topk_gap(s, K).min() >= W.MIN_TOPK_GAP
    assert c.meta["min_topk_gap"] >= W.MIN_TOPK_GAP
    k = oracle.to64(c.k)[0]
    u = c.meta["u"][0]
    w0 = c.window_blk0 * c.block
    for h in (0, 5, 11):
        kw = k[w0:w0 + c.n_win_blk * c.block, h, :].reshape(c.n_win_blk, c.block, -1)
        planted = (c.meta["a"][0, h][:, None] * u[h][None, :])
        resid = kw.mean(axis=1) - planted  # block mean of the noise alone
        # N(0, 1) noise: each coordinate of a 64-row mean has std 1/8
        assert 0.09 < resid.std() < 0.16


def test_iid_sparse_reduced_margin():
    from parity_util import sparse_iid_case
    c = sparse_iid_case(name="iid-mid", seed=5, H=2, d=128, frame_tokens=1536, block=64, hist_frames=2,
                        win_frames=6, q_frames=3, n_persist=4)
    s = oracle.block_scores(c.q, c.k, c.window_blk0, c.n_win_blk, c.block)
    for K in (9, 18, 36):
        assert oracle.topk_gap(s, K).min() >= 0.05
    assert c.meta["redraw_rounds"] >= 1  # the i.i.d. recipe does need redraws


def test_iid_generator_refuses_without_margin_check():
    with pytest.raises(ValueError):
        W.make_block_sparse("x", seed=1, H=1, d=16, frame_tokens=64, block=16, hist_frames=1, win_frames=2,
                            q_frames=1, n_persist=1, noise="iid")
