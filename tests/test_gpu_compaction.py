"""GPU parity of the head-aware cache compaction (bit-exact against the oracle)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import compaction as OC
from parity_util import assert_bf16_close, assert_lse_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def vk():
    from kv_cache_attention_chunk_b200 import vkv
    vkv.lib()
    return vkv


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _dense(seed, B, H, d, ft, hist, cur):
    g = torch.Generator().manual_seed(seed)
    L = (hist + cur) * ft
    k = torch.randn((B, L, H, d), generator=g).to(torch.bfloat16)
    v = torch.randn((B, L, H, d), generator=g).to(torch.bfloat16)
    return k, v


def _run(k, v, rules, ft, hist, cur, recent):
    kv = vk()
    ko, vo, cu_dev, cu_host = kv.compact_cache(k.to(DEV), v.to(DEV), rules, ft, hist, cur, recent)
    torch.cuda.synchronize()
    return ko, vo, cu_dev, cu_host


@pytest.mark.parametrize("d,ft", [(128, 70), (64, 64), (128, 5)])
def test_compaction_small_bit_exact(d, ft):
    B, H, hist, cur, recent = 2, 4, 12, 2, 2
    rules = [(OC.ANCHOR, 4), (OC.WAVE, 3), (OC.VEIL, 6), (OC.FULL, 0)]
    k, v = _dense(11 + d + ft, B, H, d, ft, hist, cur)
    ko, vo, cu_dev, cu_host = _run(k, v, rules, ft, hist, cur, recent)
    rk, rv, rcu, _ = oracle.compact_cache(_bits(k), _bits(v), rules, ft, hist, cur, recent)
    assert np.array_equal(cu_host, rcu)
    assert np.array_equal(cu_dev.cpu().numpy(), rcu)
    assert np.array_equal(_bits(ko), rk)
    assert np.array_equal(_bits(vo), rv)


def test_compaction_pyramid_config_full_size():
    # config-4 shape: B=1, 12 heads, d=128, 1560 tokens per frame, 60 history + 3 current frames
    ft, hist, cur, recent = 1560, 60, 3, 2
    rules = [(OC.ANCHOR, 8)] * 4 + [(OC.WAVE, p) for p in (2, 3, 4, 5)] + [(OC.VEIL, 8)] * 4
    k, v = _dense(12, 1, 12, 128, ft, hist, cur)
    ko, vo, cu_dev, cu_host = _run(k, v, rules, ft, hist, cur, recent)
    rk, rv, rcu, _ = oracle.compact_cache(_bits(k), _bits(v), rules, ft, hist, cur, recent)
    assert cu_host.tolist()[-1] == 299520
    assert np.array_equal(cu_host, rcu)
    assert np.array_equal(cu_dev.cpu().numpy(), rcu)
    assert np.array_equal(_bits(ko), rk)
    assert np.array_equal(_bits(vo), rv)


def test_compaction_then_ragged_attention():
    B, H, d, ft, hist, cur, recent = 1, 4, 128, 96, 10, 2, 2
    rules = [(OC.ANCHOR, 3), (OC.WAVE, 2), (OC.VEIL, 4), (OC.FULL, 0)]
    k, v = _dense(13, B, H, d, ft, hist, cur)
    g = torch.Generator().manual_seed(14)
    q = torch.randn((B, cur * ft, H, d), generator=g).to(torch.bfloat16)
    ko, vo, cu_dev, cu_host = _run(k, v, rules, ft, hist, cur, recent)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, l = vk().chunk_attn_ragged(q.to(DEV), ko, vo, cu_dev, cu_host, scale=d ** -0.5, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    rk, rv, rcu, _ = oracle.compact_cache(_bits(k), _bits(v), rules, ft, hist, cur, recent)
    kf = torch.from_numpy(rk.view(np.int16).copy()).view(torch.bfloat16)
    vf = torch.from_numpy(rv.view(np.int16).copy()).view(torch.bfloat16)
    ro, rl = oracle.ragged_attention(q, kf, vf, rcu, d ** -0.5)
    assert_bf16_close(o, ro, "compacted ragged O")
    assert_lse_close(l, rl, "compacted ragged LSE")


def test_compaction_rejects_bad_rule():
    k, v = _dense(15, 1, 2, 64, 8, 6, 1)
    with pytest.raises(Exception):
        vk().compact_cache(k.to(DEV), v.to(DEV), [(OC.VEIL, 3), (OC.FULL, 0)], 8, 6, 1, 2)
