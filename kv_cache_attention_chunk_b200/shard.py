"""One chunk's attention split over several GPUs (one process per GPU).

Two exact splits of the dense dual-branch chunk, each rank working on its own
GPU's memory only (no kernel reads a peer's memory; the one exchange step is
an NCCL send/recv or all-gather into local buffers):

* by head (``attend_heads``): rank r computes heads [h0_r, h1_r) -- heads are
  independent in every mode -- and, when asked, the ranks all-gather the
  merged output so that each holds the whole [B, Lq, H, d] tensor;
* by key range (``attend_key_split``): the decomposable-attention split of the
  ISPA summary (section 2 step 1, "Dual-Stream Warmup": branch outputs tracked
  by their log-sum-exp and recombined afterwards).  The chunk's key set (the
  local and history branches' segments) is cut into one part per rank; rank r
  attends over its part and produces a partial output and its LSE; rank 0
  receives every other rank's partial (one send/recv each, into its own
  memory) and folds them in with the LSE merge.  With two ranks and
  ``by_branch=True`` the parts are exactly the two branches (local on rank 0,
  history on rank 1).

The attention and merge steps are callables: by default the library's own
(``vkv.chunk_attn_segments`` and ``vkv.lse_merge``, hand-written CUDA through
the C ABI); the functions here only slice, exchange and order the work.
"""
from __future__ import annotations

import torch


def head_range(H: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous heads of `rank`: the first H % world ranks take one more."""
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def key_parts(branches, world: int, tile: int = 128, by_branch: bool = False) -> list:
    """Cut the chunk's key set into `world` parts, each a list of (start, len) segments.

    The key set is the branches' segments in order (local, then history).  By
    default the cuts fall at multiples of `tile` keys, as even as possible, so
    the ranks get equal work; a part may span segments of both branches.  With
    by_branch the parts are the branches themselves (world must equal their
    number).  Every key lies in exactly one part, in the original order.
    """
    if by_branch:
        if world != len(branches):
            raise ValueError("by_branch needs one rank per branch")
        return [[s for s in br if s[1] > 0] for br in branches]
    segs = [(int(a), int(n)) for br in branches for a, n in br if n > 0]
    total = sum(n for _, n in segs)
    n_tiles = -(-total // tile)
    cuts = [min(total, ((n_tiles * r) // world) * tile) for r in range(world)] + [total]
    parts = []
    for r in range(world):
        lo, hi = cuts[r], cuts[r + 1]
        part, off = [], 0
        for a, n in segs:
            s0, s1 = max(lo, off), min(hi, off + n)
            if s1 > s0:
                part.append((a + s0 - off, s1 - s0))
            off += n
        parts.append(part)
    return parts


def _default_attn_heads(q, k, v, branches):
    from kv_cache_attention_chunk_b200 import vkv
    return vkv.chunk_attn_segments(q, k, v, branches)


def _default_attn_keys(q, k, v, segments):
    from kv_cache_attention_chunk_b200 import vkv
    res = vkv.chunk_attn_segments(q, k, v, [segments], merged=False)
    return res["o"][0], res["lse"][0]


def _default_merge(o_a, lse_a, o_b, lse_b):
    from kv_cache_attention_chunk_b200 import vkv
    return vkv.lse_merge(o_a, lse_a, o_b, lse_b)


def gather_heads(o, H: int, rank: int, world: int, group=None):
    """All-gather the ranks' head slices o [B, Lq, h1 - h0, d] into the whole
    [B, Lq, H, d] on every rank (each slice padded to the largest head count)."""
    import torch.distributed as dist
    B, Lq, _, d = o.shape
    h0, h1 = head_range(H, world, rank)
    hmax = head_range(H, world, 0)[1]
    mine = torch.zeros((B, Lq, hmax, d), dtype=o.dtype, device=o.device)
    mine[:, :, :h1 - h0] = o
    if world > 1:
        bufs = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(bufs, mine, group=group)
    else:
        bufs = [mine]
    full = torch.empty((B, Lq, H, d), dtype=o.dtype, device=o.device)
    for r in range(world):
        a, b = head_range(H, world, r)
        full[:, :, a:b] = bufs[r][:, :, :b - a]
    return full


def attend_heads(q, k, v, branches, rank: int, world: int, attn=None, gather: bool = False, group=None):
    """Heads [h0, h1) of this rank (strided views of q, k, v: no copies).

    Returns (h0, h1, res, full): res is the attention result for the rank's heads
    (dict o, lse, o_merged, lse_merged, as vkv.chunk_attn_segments returns it);
    full is the merged output of all heads [B, Lq, H, d] gathered from every rank
    when `gather`, else None.
    """
    attn = attn or _default_attn_heads
    H = q.shape[2]
    h0, h1 = head_range(H, world, rank)
    res = attn(q[:, :, h0:h1], k[:, :, h0:h1], v[:, :, h0:h1], branches)
    full = None
    if gather:
        o = res["o_merged"] if res.get("o_merged") is not None else res["o"][0]
        full = gather_heads(o, H, rank, world, group=group)
    return h0, h1, res, full


def compact_part(k, v, segments):
    """This rank's key part as its own compact K/V: the part's rows [B, n, H, d]
    gathered in order, and the one segment [(0, n)] that covers them (attention
    over a key set does not depend on where the keys sit in the cache)."""
    idx = torch.cat([torch.arange(a, a + n, device=k.device) for a, n in segments]) if segments else \
        torch.zeros(0, dtype=torch.long, device=k.device)
    return k[:, idx].contiguous(), v[:, idx].contiguous(), [(0, int(idx.numel()))] if segments else []


def merge_to_rank0(o, lse, rank: int, world: int, merge=None, group=None):
    """Rank 0 receives every other rank's partial (o, lse) into its own memory and
    folds them in, in rank order, with the exact LSE merge; the other ranks send
    theirs.  Returns the merged (o, lse) on rank 0, the rank's own partial elsewhere."""
    import torch.distributed as dist
    merge = merge or _default_merge
    if world == 1:
        return o, lse
    if rank != 0:
        dist.send(o.contiguous(), dst=0, group=group)
        dist.send(lse.contiguous(), dst=0, group=group)
        return o, lse
    acc_o, acc_l = o, lse
    for r in range(1, world):
        ro, rl = torch.empty_like(o), torch.empty_like(lse)
        dist.recv(ro, src=r, group=group)
        dist.recv(rl, src=r, group=group)
        acc_o, acc_l = merge(acc_o, acc_l, ro, rl)
    return acc_o, acc_l


def attend_key_split(q, k, v, branches, rank: int, world: int, attn=None, merge=None, by_branch: bool = False,
                     group=None):
    """Partial attention over this rank's key part; rank 0 merges every part.

    Returns (o, lse) of the whole key set on rank 0 -- the exact LSE merge of the
    ranks' partials, folded in rank order -- and this rank's own partial on the
    other ranks (after its send has completed).
    """
    attn = attn or _default_attn_keys
    parts = key_parts(branches, world, by_branch=by_branch)
    o, lse = attn(q, k, v, parts[rank])
    return merge_to_rank0(o, lse, rank, world, merge=merge, group=group)
