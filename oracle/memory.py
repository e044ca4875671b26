"""Persistent-memory management oracle (fp64 NumPy).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it; the library never does, and it
shares no code with the CUDA path.

Source: Sparse Forcing summary, section 2 component 1 "Structured Memory
Decomposition": the persistent memory P_t keeps the most important blocks of
the whole history; the blocks evicted from the local window become
candidates, and the top C by a coarse-grained score are kept in (or replace
blocks of) the persistent memory; component 2: each block is compressed to one
representative token for coarse scoring.

Readings (the page names the candidates and "coarse-grained score" only):

* the candidates are the current persistent blocks and the evicted blocks;
* a block's representative is the mean of its 64 rows; the chunk's query
  representative is the mean of all its query rows; the score is their inner
  product (no softmax scale: a positive factor does not change the ranking);
* the C highest scores are kept, equal scores taking the lower block id first,
  and returned in ascending block order (the top-K conventions of PBSA).
"""
from __future__ import annotations

import numpy as np

from .attention import to64


def persist_update(q, k, persist_idx, evict_blk0: int, n_evict: int, block: int = 64):
    """Returns (new persistent ids [B*H, C] ascending, candidate scores [B*H, C + n_evict])."""
    q64, k64 = to64(q), to64(k)
    B, Lq, H, d = q64.shape
    persist_idx = np.asarray(persist_idx)
    C = persist_idx.shape[-1]
    out = np.zeros((B * H, C), dtype=np.int32)
    scores = np.zeros((B * H, C + n_evict))
    for b in range(B):
        for h in range(H):
            s = b * H + h
            qbar = q64[b, :, h].mean(axis=0)
            cands = [int(c) for c in persist_idx[s]] + list(range(evict_blk0, evict_blk0 + n_evict))
            sc = [float(qbar @ k64[b, c * block:(c + 1) * block, h].mean(axis=0)) for c in cands]
            scores[s] = sc
            best = sorted(range(len(cands)), key=lambda i: (-sc[i], cands[i]))[:C]
            out[s] = sorted(cands[i] for i in best)
    return out, scores
