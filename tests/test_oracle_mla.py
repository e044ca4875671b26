"""Pins of the latent-attention oracle (CPU only).

The absorbed latent form is checked against things other than itself:

* the per-head form with explicit up-projections (VideoMLA technical summary,
  "Methodology": keys and values rebuilt from the shared latent, a separate
  head-shared rotary key) on random weights;
* a pure-Python brute-force loop on tiny inputs;
* closed forms (identical cached rows; one dominant key) and invariances
  (row order, a common shift of the rotary keys);
* the memory figures the pages print (92.7 % fewer cached scalars; about
  6.0 GB of dense cache for 21 latent frames of Wan-1.3B);
* planted mistakes that the expanded-form pin must catch.
"""
import math

import numpy as np
import pytest

from oracle import mla as M
from oracle.attention import attend


def _weights(rng, H, d_nope, d_v, d_c):
    w_k = rng.standard_normal((H, d_nope, d_c)) / math.sqrt(d_c)
    w_v = rng.standard_normal((H, d_v, d_c)) / math.sqrt(d_c)
    return w_k, w_v


def _expanded_case(seed=0, B=2, H=3, Lq=7, Lkv=29, d_nope=12, d_rope=4, d_c=10, d_v=9):
    rng = np.random.default_rng(seed)
    q_nope = rng.standard_normal((B, Lq, H, d_nope))
    q_rope = rng.standard_normal((B, Lq, H, d_rope))
    c = rng.standard_normal((B, Lkv, d_c))
    k_rope = rng.standard_normal((B, Lkv, d_rope))
    w_k, w_v = _weights(rng, H, d_nope, d_v, d_c)
    return q_nope, q_rope, c, k_rope, w_k, w_v


def _absorbed(q_nope, q_rope, c, k_rope, w_k, w_v, scale, fn=M.latent_attention):
    qa = M.absorb_query(q_nope, q_rope, w_k)
    kv = np.concatenate([c, k_rope], axis=-1)
    o_lat, lse = fn(qa, kv, c.shape[-1], scale)
    return M.up_project_output(o_lat, w_v), lse


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_absorbed_equals_expanded_heads(seed):
    case = _expanded_case(seed)
    scale = 1 / math.sqrt(16)
    o_ref, lse_ref = M.expanded_attention(*case, scale)
    o, lse = _absorbed(*case, scale)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def _brute_latent(q, kv, d_c, scale):
    """Pure-Python loops: LSE first, then O = sum exp(s - LSE) c."""
    B, Lq, H, dq = q.shape
    Lkv = kv.shape[1]
    o = np.zeros((B, Lq, H, d_c))
    lse = np.zeros((B, H, Lq))
    for b in range(B):
        for h in range(H):
            for i in range(Lq):
                s = [scale * math.fsum(float(q[b, i, h, e]) * float(kv[b, t, e]) for e in range(dq))
                     for t in range(Lkv)]
                mx = max(s)
                L = mx + math.log(math.fsum(math.exp(x - mx) for x in s))
                lse[b, h, i] = L
                for e in range(d_c):
                    o[b, i, h, e] = math.fsum(math.exp(s[t] - L) * float(kv[b, t, e]) for t in range(Lkv))
    return o, lse


def test_brute_force_tiny():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 4, 2, 6))
    kv = rng.standard_normal((1, 9, 6))
    o, lse = M.latent_attention(q, kv, 4, 0.37)
    ob, lb = _brute_latent(q, kv, 4, 0.37)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-12)


def test_identical_rows_give_the_row():
    rng = np.random.default_rng(3)
    r = rng.standard_normal(7)
    kv = np.tile(r, (1, 50, 1))
    q = rng.standard_normal((1, 5, 2, 7))
    o, lse = M.latent_attention(q, kv, 5, 0.5)
    np.testing.assert_allclose(o, np.broadcast_to(r[:5], o.shape), rtol=0, atol=1e-13)
    want = 0.5 * np.einsum("lhe,e->hl", q[0], r) + math.log(50)
    np.testing.assert_allclose(lse[0], want, rtol=0, atol=1e-12)


def test_one_dominant_key():
    rng = np.random.default_rng(4)
    kv = rng.standard_normal((1, 40, 6)) * 0.01
    kv[0, 17, 4:] = [30.0, -30.0]
    q = np.zeros((1, 3, 1, 6))
    q[..., 4:] = [1.0, -1.0]
    o, _ = M.latent_attention(q, kv, 4, 1.0)
    np.testing.assert_allclose(o[0, :, 0, :], np.broadcast_to(kv[0, 17, :4], (3, 4)), atol=1e-20)


def test_row_order_invariance():
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 6, 2, 8))
    kv = rng.standard_normal((1, 33, 8))
    perm = rng.permutation(33)
    o1, l1 = M.latent_attention(q, kv, 6, 0.3)
    o2, l2 = M.latent_attention(q, kv[:, perm], 6, 0.3)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_rotary_shift_moves_lse_only():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 6, 2, 8))
    kv = rng.standard_normal((1, 33, 8))
    w = rng.standard_normal(2)
    kv2 = kv.copy()
    kv2[..., 6:] += w
    o1, l1 = M.latent_attention(q, kv, 6, 0.3)
    o2, l2 = M.latent_attention(q, kv2, 6, 0.3)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    shift = 0.3 * np.einsum("lhe,e->hl", q[0, :, :, 6:], w)
    np.testing.assert_allclose(l2[0], l1[0] + shift, rtol=0, atol=1e-12)


def test_single_head_reduces_to_attend():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 5, 1, 9))
    kv = rng.standard_normal((1, 12, 9))
    o, lse = M.latent_attention(q, kv, 7, 0.4)
    o_ref, l_ref = attend(q[0, :, 0, :], kv[0], kv[0, :, :7], 0.4)
    np.testing.assert_allclose(o[0, :, 0, :], o_ref, rtol=0, atol=0)
    np.testing.assert_allclose(lse[0, 0], l_ref, rtol=0, atol=0)


def test_memory_figures_of_the_pages():
    dense, latent = M.cache_scalars_per_token(12, 128, 192, 32)
    assert (dense, latent) == (3072, 224)
    assert round(100 * (1 - latent / dense), 1) == 92.7
    # 21 latent frames of 1560 tokens, 30 layers, bf16: about 6.0 GB dense
    gb = dense * 2 * 21 * 1560 * 30 / 1e9
    assert abs(gb - 6.0) < 0.05


def test_flop_count():
    assert M.visited_flops_latent(1, 12, 4680, 32760, 192, 32) == 2.0 * 12 * 4680 * 32760 * 416
    # brute count on a tiny case: one multiply-add per (query, key, feature)
    B, H, Lq, Lkv, dc, dr = 2, 3, 5, 7, 4, 2
    macs = sum(1 for _ in range(B * H * Lq * Lkv) for _ in range(dc + dr + dc))
    assert M.visited_flops_latent(B, H, Lq, Lkv, dc, dr) == 2 * macs


# ---------------------------------------------------------------------------
# planted mistakes: each must break the expanded-form pin
# ---------------------------------------------------------------------------
def _latent_wrong_value_slice(q, kv, d_c, scale):
    q = np.asarray(q, float)
    kv = np.asarray(kv, float)
    B, Lq, H, _ = q.shape
    o = np.empty((B, Lq, H, d_c))
    lse = np.empty((B, H, Lq))
    for b in range(B):
        for h in range(H):
            o[b, :, h, :], lse[b, h] = attend(q[b, :, h, :], kv[b], kv[b, :, -d_c:], scale)
    return o, lse


def _latent_no_rope(q, kv, d_c, scale):
    q = np.asarray(q, float)
    kv = np.asarray(kv, float)
    B, Lq, H, _ = q.shape
    o = np.empty((B, Lq, H, d_c))
    lse = np.empty((B, H, Lq))
    for b in range(B):
        for h in range(H):
            o[b, :, h, :], lse[b, h] = attend(q[b, :, h, :d_c], kv[b, :, :d_c], kv[b, :, :d_c], scale)
    return o, lse


@pytest.mark.parametrize("mutant", [_latent_wrong_value_slice, _latent_no_rope])
def test_planted_mistakes_are_caught(mutant):
    case = _expanded_case(11)
    scale = 0.25
    o_ref, lse_ref = M.expanded_attention(*case, scale)
    o, lse = _absorbed(*case, scale, fn=mutant)
    assert np.abs(o - o_ref).max() > 1e-3 or np.abs(lse - lse_ref).max() > 1e-3


def test_untransposed_absorption_is_caught():
    case = list(_expanded_case(12, d_nope=10, d_c=10))
    q_nope, q_rope, c, k_rope, w_k, w_v = case
    scale = 0.25
    o_ref, _ = M.expanded_attention(q_nope, q_rope, c, k_rope, w_k, w_v, scale)
    qa = np.concatenate([np.einsum("blhn,hcn->blhc", q_nope, w_k), q_rope], axis=-1)
    o_lat, _ = M.latent_attention(qa, np.concatenate([c, k_rope], -1), 10, scale)
    assert np.abs(M.up_project_output(o_lat, w_v) - o_ref).max() > 1e-3
