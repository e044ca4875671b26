"""One chunk split over ranks (kv_cache_attention_chunk_b200.shard), on CPU.

The split/exchange/merge plumbing runs as gloo ranks (world size 2 and 3) on
the tiny dual-branch config, with the fp64 oracle standing in for the attention
and merge kernels (test infrastructure: the product path passes the library's
own kernels); rank 0's merged output is compared with the oracle's attention
over the whole key set.  The key cuts and head ranges are checked on their own.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from kv_cache_attention_chunk_b200 import shard  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_head_ranges_cover_every_head_once():
    for H in (1, 2, 12, 40):
        for world in (1, 2, 3, 4, 8):
            got = [shard.head_range(H, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == H
            assert all(got[r][1] == got[r + 1][0] for r in range(world - 1))
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
def test_key_parts_partition_the_key_set(world):
    from kv_cache_attention_chunk_b200 import workloads as W
    loc, hist = W.dual_branch_layout(1560, 1, 20, 3)
    parts = shard.key_parts([loc, hist], world)
    rows = np.concatenate([np.arange(a, a + n) for p in parts for a, n in p])
    ref = np.concatenate([np.arange(a, a + n) for br in (loc, hist) for a, n in br])
    assert np.array_equal(rows, ref)  # every key once, in order
    sizes = [sum(n for _, n in p) for p in parts]
    assert max(sizes) - min(sizes) <= 128
    assert all(s % 128 == 0 for s in sizes[:-1])  # cuts on tile boundaries
    by = shard.key_parts([loc, hist], 2, by_branch=True)
    assert by == [loc, hist]


def _oracle_attn_keys(q, k, v, segments):
    import oracle
    r = oracle.segment_attention(q, k, v, [segments], _SCALE[0])
    return (torch.from_numpy(r["branch_o"][0]).to(torch.bfloat16),
            torch.from_numpy(r["branch_lse"][0]).to(torch.float32))


def _oracle_attn_heads(q, k, v, branches):
    import oracle
    r = oracle.segment_attention(q, k, v, branches, _SCALE[0])
    out = {"o": [torch.from_numpy(x).to(torch.bfloat16) for x in r["branch_o"]],
           "lse": [torch.from_numpy(x).to(torch.float32) for x in r["branch_lse"]]}
    out["o_merged"] = torch.from_numpy(r["dense_o"]).to(torch.bfloat16)
    out["lse_merged"] = torch.from_numpy(r["dense_lse"]).to(torch.float32)
    return out


def _oracle_merge(o_a, lse_a, o_b, lse_b):
    """The merge kernel's stand-in: LSEs [B, H, Lq] as the library lays them out."""
    import oracle
    f = lambda t: t.to(torch.float64).numpy()  # noqa: E731
    g = lambda t: np.moveaxis(f(t), 1, 2)  # noqa: E731  [B, H, Lq] -> [B, Lq, H]
    o, l = oracle.lse_merge(f(o_a), g(lse_a), f(o_b), g(lse_b))
    return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(np.moveaxis(l, 2, 1).copy()).to(torch.float32)


_SCALE = [0.125]


def _worker(rank, world, port, mode, by_branch, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    from kv_cache_attention_chunk_b200 import shard as S, workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    c = W.cfg_tiny()
    _SCALE[0] = c.scale
    if mode == "keys":
        o, l = S.attend_key_split(c.q, c.k, c.v, c.branches, rank, world, attn=_oracle_attn_keys,
                                  merge=_oracle_merge, by_branch=by_branch)
        q.put((rank, o.float().numpy(), l.numpy()))
    else:
        h0, h1, res, full = S.attend_heads(c.q, c.k, c.v, c.branches, rank, world, attn=_oracle_attn_heads,
                                           gather=True)
        q.put((rank, full.float().numpy(), (h0, h1)))
    dist.barrier()
    dist.destroy_process_group()


def _run(world, mode, by_branch=False):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, by_branch, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def _dense_ref():
    import oracle
    from kv_cache_attention_chunk_b200 import workloads as W
    c = W.cfg_tiny()
    return oracle.segment_attention(c.q, c.k, c.v, c.branches, c.scale)


@pytest.mark.parametrize("world,by_branch", [(2, False), (2, True), (3, False)])
def test_key_split_merge_equals_dense(world, by_branch):
    from parity_util import assert_bf16_close, assert_lse_close
    res = _run(world, "keys", by_branch)
    ref = _dense_ref()
    _, o, l = res[0]
    assert_bf16_close(o, ref["dense_o"], "key split merged O")
    assert_lse_close(l, ref["dense_lse"], "key split merged LSE")
    if by_branch:
        # rank 1 holds the history branch's own partial (the method's split)
        assert_bf16_close(res[1][1], ref["branch_o"][1], "history branch O on rank 1")


def test_head_split_all_gather_equals_dense():
    from parity_util import assert_bf16_close
    res = _run(2, "heads")
    ref = _dense_ref()
    assert [r[2] for r in res] == [(0, 1), (1, 2)]
    for _, full, _ in res:
        assert_bf16_close(full, ref["dense_o"], "head split gathered O")


def test_key_split_single_rank_is_whole_key_set():
    from kv_cache_attention_chunk_b200 import workloads as W
    c = W.cfg_tiny()
    parts = shard.key_parts(c.branches, 1)
    assert parts == [[s for br in c.branches for s in br]]


def test_compact_part_keeps_the_key_set():
    from kv_cache_attention_chunk_b200 import workloads as W
    import oracle
    c = W.cfg_tiny()
    parts = shard.key_parts(c.branches, 3)
    for p in parts:
        kr, vr, seg = shard.compact_part(c.k, c.v, p)
        a = oracle.segment_attention(c.q, c.k, c.v, [p], c.scale)
        b = oracle.segment_attention(c.q, kr, vr, [seg], c.scale)
        assert np.array_equal(a["branch_o"][0], b["branch_o"][0])
        assert np.array_equal(a["branch_lse"][0], b["branch_lse"][0])
