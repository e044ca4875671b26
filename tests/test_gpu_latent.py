"""GPU parity of latent (VideoMLA) attention against the fp64 oracle.

Same bar as the other attention modes: bf16 latent outputs max-abs <= 2e-2
and mean-abs <= 2e-3, fp32 LSE <= 1e-3 absolute.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_attention_chunk_b200 import workloads as W
from parity_util import assert_bf16_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def vk():
    from kv_cache_attention_chunk_b200 import vkv
    vkv.lib()
    return vkv


def _run(case, **kw):
    v = vk()
    q = case.q.to(DEV)
    kv = case.kv.to(DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = v.latent_attn(q, kv, case.d_c, scale=case.scale, err=err, **kw)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return o, lse


def _check_full(case, o, lse, what):
    o_ref, l_ref = oracle.latent_attention(case.q, case.kv, case.d_c, case.scale)
    assert_bf16_close(o, o_ref, what)
    assert_lse_close(lse, l_ref, what)


@pytest.mark.parametrize("d_c,B,H,Lq,Lkv,q_std", [
    (192, 2, 3, 300, 1000, 1.0),    # several tiles of both kinds, ragged tails
    (192, 1, 2, 128, 128, 3.0),     # exact single tiles, peaked softmax
    (192, 1, 4, 77, 50, 1.0),       # one partial cache tile
    (192, 1, 1, 5, 1, 1.0),         # a single cached row
    (128, 2, 3, 300, 1000, 1.0),    # the smaller latent budget
    (192, 1, 40, 512, 600, 2.0),    # more query tiles than SMs: several tiles per CTA
    (192, 4, 12, 300, 700, 1.0),    # a batch of chunks, each over its own cache
])
def test_latent_matches_oracle(d_c, B, H, Lq, Lkv, q_std):
    case = W.make_latent("t", seed=11 + Lq, B=B, H=H, Lq=Lq, Lkv=Lkv, d_c=d_c, q_std=q_std)
    o, lse = _run(case)
    _check_full(case, o, lse, f"latent d_c={d_c} B={B} H={H} Lq={Lq} Lkv={Lkv}")


def test_growing_scores_force_rescales():
    """Scores rise along the cache, so the running maximum moves by more than 2^8
    many times within a row: the output rescaling path is exercised."""
    rng = np.random.default_rng(3)
    B, H, Lq, Lkv, d_c = 1, 2, 200, 2000, 192
    q = rng.standard_normal((B, Lq, H, 224)).astype(np.float32) * 0.5
    q[..., 192:] = 0.0
    q[..., 192] = 4.0
    kv = rng.standard_normal((B, Lkv, 224)).astype(np.float32)
    kv[..., 192:] = 0.0
    kv[0, :, 192] = np.linspace(0.0, 60.0, Lkv, dtype=np.float32)
    case = W.LatentCase("ramp", B, H, d_c, 32, torch.from_numpy(q).to(torch.bfloat16),
                        torch.from_numpy(kv).to(torch.bfloat16), 1.0 / np.sqrt(128.0))
    o, lse = _run(case)
    _check_full(case, o, lse, "rising scores")


def test_separate_rotary_keys_equal_pair_layout():
    case = W.make_latent("t", seed=5, B=2, H=3, Lq=200, Lkv=700)
    o1, l1 = _run(case)
    kv = case.kv.to(DEV)
    c_only = torch.zeros((2, 700, 192 + 64), dtype=torch.bfloat16, device=DEV)[..., :192]
    c_only.copy_(kv[..., :192])
    kr = kv[..., 192:].contiguous()
    o2, l2 = vk().latent_attn(case.q.to(DEV), c_only, 192, scale=case.scale, kr=kr)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_strided_query_and_output():
    case = W.make_latent("t", seed=6, B=2, H=3, Lq=260, Lkv=500)
    big = torch.zeros((2, 260, 5, 256), dtype=torch.bfloat16, device=DEV)
    q = big[:, :, 1:4, :224]
    q.copy_(case.q.to(DEV))
    out_big = torch.full((2, 300, 3, 256), float("nan"), dtype=torch.bfloat16, device=DEV)
    o = out_big[:, 20:280, :, 32:224]
    lse = torch.empty((2, 3, 260), dtype=torch.float32, device=DEV)
    vk().latent_attn(q, case.kv.to(DEV), 192, scale=case.scale, out=(o, lse))
    torch.cuda.synchronize()
    _check_full(case, o, lse, "strided")
    assert torch.isnan(out_big[:, :20]).all() and torch.isnan(out_big[:, 280:]).all()
    assert torch.isnan(out_big[..., :32]).all() and torch.isnan(out_big[..., 224:]).all()


def test_empty_cache():
    case = W.make_latent("t", seed=7, B=1, H=2, Lq=130, Lkv=0)
    o, lse = _run(case)
    assert torch.equal(o, torch.zeros_like(o))
    assert torch.isneginf(lse).all()


def test_latent_output_projects_to_expanded_heads():
    """Up-projecting the kernel's latent output reproduces per-head attention with
    keys and values rebuilt from the latent (the absorption the method relies on)."""
    rng = np.random.default_rng(9)
    B, H, Lq, Lkv, d_c, d_nope, d_v = 1, 2, 150, 400, 192, 96, 128
    c = rng.standard_normal((B, Lkv, d_c)).astype(np.float32)
    k_r = rng.standard_normal((B, Lkv, 32)).astype(np.float32)
    q_nope = rng.standard_normal((B, Lq, H, d_nope))
    q_r = rng.standard_normal((B, Lq, H, 32))
    w_k = rng.standard_normal((H, d_nope, d_c)) / np.sqrt(d_c)
    w_v = rng.standard_normal((H, d_v, d_c)) / np.sqrt(d_c)
    qa = torch.from_numpy(oracle.mla.absorb_query(q_nope, q_r, w_k).astype(np.float32)).to(torch.bfloat16)
    kv = torch.from_numpy(np.concatenate([c, k_r], -1)).to(torch.bfloat16)
    scale = 1 / np.sqrt(128.0)
    o, lse = vk().latent_attn(qa.to(DEV), kv.to(DEV), d_c, scale=scale)
    torch.cuda.synchronize()
    # the reference sees the same bf16-rounded query and cache
    qa64, kv64 = to_np(qa), to_np(kv)
    o_ref, l_ref = oracle.latent_attention(qa64, kv64, d_c, scale)
    assert_bf16_close(o, o_ref, "absorbed")
    assert_lse_close(lse, l_ref, "absorbed")
    up = oracle.mla.up_project_output(to_np(o), w_v)
    up_ref = oracle.mla.up_project_output(o_ref, w_v)
    assert np.abs(up - up_ref).max() <= 2e-2


def test_full_size_sampled():
    """The benchmarked VideoMLA chunk (12 heads, 4680 queries, 21-frame cache of 32 760
    rows): every head's first, middle and last query rows against the oracle."""
    case = W.cfg_latent()
    o, lse = _run(case)
    rows = np.array([0, 1, 127, 128, 2339, 4607, 4608, 4679])
    o_ref, l_ref = oracle.latent_attention(case.q, case.kv, case.d_c, case.scale, rows=rows)
    assert_bf16_close(to_np(o)[:, rows], o_ref[:, rows], "full size")
    assert_lse_close(to_np(lse)[:, :, rows], l_ref[:, :, rows], "full size lse")
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()


def test_stalled_pipeline_reports_timeout_and_device_stays_usable():
    """A withheld cache-tile copy makes the bounded wait run out: VKV_DEVERR_TIMEOUT,
    then a normal call on the same context matches the oracle."""
    v = vk()
    case = W.make_latent("t", seed=8, B=1, H=2, Lq=200, Lkv=400)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    with v.using_test_library():  # the test aid exists only in the test build
        assert v.vkv_debug_withhold_copy(1) == 0
        try:
            v.latent_attn(case.q.to(DEV), case.kv.to(DEV), case.d_c, scale=case.scale, err=err)
            torch.cuda.synchronize()
        finally:
            v.vkv_debug_withhold_copy(0)
        assert int(err.item()) == v.DEVERR_TIMEOUT
        o, lse = _run(case)
        _check_full(case, o, lse, "after a timeout")
    o, lse = _run(case)
    _check_full(case, o, lse, "production library after a timeout")
