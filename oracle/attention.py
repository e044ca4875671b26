"""fp64 CPU oracle for chunk attention over a segmented KV cache.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plain reference that the
CUDA path is checked against.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it; the library itself
never does, and it shares no code with the CUDA kernels.

Every step is the textbook definition, computed in float64 from the exact
bf16 inputs.  For one query row q_i and an explicitly gathered key set J:

    s_j   = scale * <q_i, k_j>
    m     = max_j s_j
    l     = sum_j exp(s_j - m)
    O_i   = sum_j exp(s_j - m) v_j / l
    LSE_i = m + ln l                      (natural log, scale included)

Sources (page title, section):

* ISPA summary, section 2 step 1 "Dual-Stream Warmup" and contribution 2:
  attention is split into a local and a history branch, each tracked with its
  log-sum-exp, and the two are recombined afterwards (online softmax).
* Sparse Forcing summary, section 2 component 2 "Blockified Compression" and
  component 3 "PBSA": one representative per block for coarse scoring; dense
  attention on persistent blocks plus top-K window blocks.
* Pyramid Forcing summary, methodology section 3 "Ragged-Cache Attention":
  per-head variable-length caches stored flattened with boundary indices.

Layouts: Q, K, V, O are [B, L, H, d]; LSE is [B, H, Lq]; ragged K/V are
[sum L_s, d] with sequence s = b*H + h at rows cu[s]..cu[s+1].
"""
from __future__ import annotations

import numpy as np

ROW_CHUNK = 512


def to64(t) -> np.ndarray:
    """Exact upcast of a (bf16) torch tensor or array to float64."""
    if hasattr(t, "detach"):
        t = t.detach().cpu().float().numpy()
    return np.asarray(t, dtype=np.float64)


# ---------------------------------------------------------------------------
# softmax attention over an explicit key set
# ---------------------------------------------------------------------------
def attend(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """Softmax attention of rows q [n, d] over keys k [m, d] / values v [m, dv].

    Returns (O [n, dv], LSE [n]).  An empty key set gives O = 0 and
    LSE = -inf (the empty branch has no mass).
    """
    n = q.shape[0]
    if k.shape[0] == 0:
        return np.zeros((n, v.shape[1])), np.full(n, -np.inf)
    o = np.empty((n, v.shape[1]))
    lse = np.empty(n)
    for r0 in range(0, n, ROW_CHUNK):
        r1 = min(n, r0 + ROW_CHUNK)
        s = scale * (q[r0:r1] @ k.T)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        o[r0:r1] = (e @ v) / l
        lse[r0:r1] = m[:, 0] + np.log(l[:, 0])
    return o, lse


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Exact recombination of two partial attentions over disjoint key sets.

    With M = max(LSE_a, LSE_b), w_x = exp(LSE_x - M):
        O   = (w_a O_a + w_b O_b) / (w_a + w_b)
        LSE = M + ln(w_a + w_b)
    Rows where both LSEs are -inf (no keys at all) give O = 0, LSE = -inf.
    o_* have a trailing feature axis; lse_* match o_* without it.
    """
    o_a = np.asarray(o_a, dtype=np.float64)
    o_b = np.asarray(o_b, dtype=np.float64)
    lse_a = np.asarray(lse_a, dtype=np.float64)
    lse_b = np.asarray(lse_b, dtype=np.float64)
    M = np.maximum(lse_a, lse_b)
    empty = np.isneginf(M)
    Ms = np.where(empty, 0.0, M)
    wa = np.exp(lse_a - Ms)
    wb = np.exp(lse_b - Ms)
    den = wa + wb
    safe = np.where(empty, 1.0, den)
    o = (wa[..., None] * o_a + wb[..., None] * o_b) / safe[..., None]
    o = np.where(empty[..., None], 0.0, o)
    lse = np.where(empty, -np.inf, Ms + np.log(safe))
    return o, lse


# ---------------------------------------------------------------------------
# mode 1: token segments (local / history branches)
# ---------------------------------------------------------------------------
def segment_rows(segments) -> np.ndarray:
    """Token indices of a list of (start, len) segments, in list order."""
    parts = [np.arange(s, s + n, dtype=np.int64) for s, n in segments]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def _sel(n, idx):
    return range(n) if idx is None else idx


def segment_attention(q, k, v, branches, scale, heads=None, rows=None, batches=None):
    """Per-branch attention, their LSE merge, and dense attention over the union.

    q [B, Lq, H, d], k/v [B, Lkv, H, d] (any array-likes, upcast to fp64).
    ``heads`` / ``rows`` / ``batches`` restrict the computation to a sample.
    Returns a dict with 'branch_o' (list of [b, r, h, d]), 'branch_lse'
    (list of [b, h, r]), 'merged_o', 'merged_lse', 'dense_o', 'dense_lse'.
    """
    q = to64(q)
    k = to64(k)
    v = to64(v)
    B, Lq, H, d = q.shape
    bs = list(_sel(B, batches))
    hs = list(_sel(H, heads))
    rs = np.asarray(list(_sel(Lq, rows)), dtype=np.int64)
    nb = len(branches)
    bo = [np.zeros((len(bs), len(rs), len(hs), v.shape[-1])) for _ in range(nb)]
    bl = [np.zeros((len(bs), len(hs), len(rs))) for _ in range(nb)]
    do = np.zeros((len(bs), len(rs), len(hs), v.shape[-1]))
    dl = np.zeros((len(bs), len(hs), len(rs)))
    idx = [segment_rows(br) for br in branches]
    union = np.concatenate(idx) if idx else np.zeros(0, dtype=np.int64)
    for ib, b in enumerate(bs):
        for ih, h in enumerate(hs):
            qq = q[b, rs, h, :]
            for i in range(nb):
                o, l = attend(qq, k[b, idx[i], h, :], v[b, idx[i], h, :], scale)
                bo[i][ib, :, ih, :] = o
                bl[i][ib, ih, :] = l
            o, l = attend(qq, k[b, union, h, :], v[b, union, h, :], scale)
            do[ib, :, ih, :] = o
            dl[ib, ih, :] = l
    mo, ml = bo[0], bl[0]
    for i in range(1, nb):
        mo, ml = lse_merge(mo, np.moveaxis(ml, 1, 2), bo[i], np.moveaxis(bl[i], 1, 2))
        ml = np.moveaxis(ml, 2, 1)
    return dict(branch_o=bo, branch_lse=bl, merged_o=mo, merged_lse=ml, dense_o=do, dense_lse=dl)


# ---------------------------------------------------------------------------
# mode 2: blockified coarse scoring, top-K, persistent + selected blocks
# ---------------------------------------------------------------------------
def pool_blocks(x: np.ndarray, block: int) -> np.ndarray:
    """Representative token of each block = mean of its rows.

    x [L, d]; block i covers rows [i*block, min(L, (i+1)*block)).
    """
    L = x.shape[0]
    nblk = -(-L // block)
    out = np.empty((nblk, x.shape[1]))
    for i in range(nblk):
        out[i] = x[i * block:min(L, (i + 1) * block)].mean(axis=0)
    return out


def select_topk(scores: np.ndarray, topk: int) -> np.ndarray:
    """Indices of the ``topk`` highest scores, ascending.

    Ties rank the lower block index first.  scores [..., n] -> [..., topk].
    """
    n = scores.shape[-1]
    flat = scores.reshape(-1, n)
    out = np.empty((flat.shape[0], topk), dtype=np.int32)
    ar = np.arange(n)
    for i, s in enumerate(flat):
        order = np.lexsort((ar, -s))  # primary: score descending; secondary: index ascending
        out[i] = np.sort(order[:topk])
    return out.reshape(scores.shape[:-1] + (topk,))


def block_scores(q, k, window_blk0: int, n_win_blk: int, block: int):
    """Coarse scores <mean-pooled query block, mean-pooled window key block>.

    Returns scores [B*H, n_qblk, n_win_blk] (no softmax scale: a positive
    factor does not change the ranking).
    """
    q = to64(q)
    k = to64(k)
    B, Lq, H, d = q.shape
    n_qblk = -(-Lq // block)
    w0 = window_blk0 * block
    out = np.empty((B * H, n_qblk, n_win_blk))
    for b in range(B):
        for h in range(H):
            qb = pool_blocks(q[b, :, h, :], block)
            kb = pool_blocks(k[b, w0:w0 + n_win_blk * block, h, :], block)
            out[b * H + h] = qb @ kb.T
    return out


def block_select(q, k, window_blk0: int, n_win_blk: int, block: int, topk: int):
    """Top-K window blocks per query block: (idx [B*H, n_qblk, topk], scores)."""
    s = block_scores(q, k, window_blk0, n_win_blk, block)
    return select_topk(s, topk), s


def topk_gap(scores: np.ndarray, topk: int) -> np.ndarray:
    """Score gap between the topk-th and (topk+1)-th best block (inf if topk = n)."""
    n = scores.shape[-1]
    if topk >= n:
        return np.full(scores.shape[:-1], np.inf)
    srt = -np.sort(-scores, axis=-1)
    return srt[..., topk - 1] - srt[..., topk]


def block_sparse_attention(q, k, v, persist_idx, sel_idx, window_blk0: int, block: int,
                           scale: float, heads=None, qblocks=None):
    """Persistent blocks (every query) + each query block's selected window blocks.

    persist_idx [B*H, n_persist] absolute block ids; sel_idx [B*H, n_qblk, K]
    window-relative block ids.  One softmax over the union (the two sets are
    disjoint).  Returns (O [B, Lq, H, d], LSE [B, H, Lq]); rows outside the
    sampled query blocks are left NaN.
    """
    q = to64(q)
    k = to64(k)
    v = to64(v)
    B, Lq, H, d = q.shape
    n_qblk = -(-Lq // block)
    o = np.full((B, Lq, H, v.shape[-1]), np.nan)
    lse = np.full((B, H, Lq), np.nan)
    for b in range(B):
        for h in list(_sel(H, heads)):
            bh = b * H + h
            pers = np.asarray(persist_idx[bh], dtype=np.int64)
            for j in list(_sel(n_qblk, qblocks)):
                blocks = np.concatenate([pers, window_blk0 + np.asarray(sel_idx[bh, j], dtype=np.int64)])
                toks = (blocks[:, None] * block + np.arange(block)[None, :]).reshape(-1)
                r0, r1 = j * block, min(Lq, (j + 1) * block)
                oo, ll = attend(q[b, r0:r1, h, :], k[b, toks, h, :], v[b, toks, h, :], scale)
                o[b, r0:r1, h, :] = oo
                lse[b, h, r0:r1] = ll
    return o, lse


# ---------------------------------------------------------------------------
# mode 3: ragged per-head caches, flattened with boundary offsets
# ---------------------------------------------------------------------------
def ragged_attention(q, k_flat, v_flat, cu_seqlens, scale, heads=None, rows=None, batches=None):
    """Sequence s = b*H + h attends over rows cu[s]..cu[s+1] of the flat K/V.

    Returns (O [b, r, h, d], LSE [b, h, r]) over the sampled batches/rows/heads.
    """
    q = to64(q)
    kf = to64(k_flat)
    vf = to64(v_flat)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B, Lq, H, d = q.shape
    bs = list(_sel(B, batches))
    hs = list(_sel(H, heads))
    rs = np.asarray(list(_sel(Lq, rows)), dtype=np.int64)
    o = np.zeros((len(bs), len(rs), len(hs), vf.shape[-1]))
    lse = np.zeros((len(bs), len(hs), len(rs)))
    for ib, b in enumerate(bs):
        for ih, h in enumerate(hs):
            s = b * H + h
            oo, ll = attend(q[b, rs, h, :], kf[cu[s]:cu[s + 1]], vf[cu[s]:cu[s + 1]], scale)
            o[ib, :, ih, :] = oo
            lse[ib, ih, :] = ll
    return o, lse


# ---------------------------------------------------------------------------
# counting (for the effective-throughput metric)
# ---------------------------------------------------------------------------
def visited_flops_segments(B, H, Lq, d, branches) -> int:
    """4*d per visited (query, key) pair: QK^T and PV multiply-adds."""
    n = sum(int(n) for br in branches for _, n in br)
    return 4 * d * B * H * Lq * n


def visited_flops_sparse(B, H, Lq, d, block, n_persist, topk) -> int:
    return 4 * d * B * H * Lq * (n_persist + topk) * block


def visited_flops_ragged(B, H, Lq, d, cu_seqlens) -> int:
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    return int(4 * d * Lq * int((cu[1:] - cu[:-1]).sum()))
