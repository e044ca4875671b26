"""fp64 CPU oracle for latent (multi-head latent) attention over a video KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; the library never does.

Source: VideoMLA technical summary, "Methodology: VideoMLA".  Each cached
token t keeps one head-shared content latent c_t (dimension d_c, the
down-projection of the token) and one head-shared rotary key k^R_t
(dimension d_rope, already rotated by the 3D-RoPE).  Head h rebuilds its
content key and its value from the latent with its own up-projections,

    k_{t,h} = [ W^K_h c_t ; k^R_t ],      v_{t,h} = W^V_h c_t,

with W^K_h of shape [d_nope, d_c] and W^V_h of shape [d_v, d_c], and a query
split the same way, q_h = [ q^nope_h ; q^R_h ].  Attention per head is the
textbook softmax attention over these keys and values.

Because <q^nope_h, W^K_h c_t> = <(W^K_h)^T q^nope_h, c_t>, the key
up-projection can be moved onto the query ("absorbed"): with

    qa_h = [ (W^K_h)^T q^nope_h ; q^R_h ]      (dimension d_c + d_rope)

the score is scale * <qa_h, [c_t ; k^R_t]>, one dot product against the
cached row itself.  Likewise sum_t p_t W^V_h c_t = W^V_h (sum_t p_t c_t), so
attention can return the latent output o_h = sum_t p_t c_t (dimension d_c)
and leave W^V_h to the output projection.  ``latent_attention`` computes
exactly that absorbed form; ``expanded_attention`` computes the per-head form
from explicit up-projections, and the two agree by the identities above.

Readings where the pages leave a step open:
* the query arriving at the kernel is already absorbed and rotated; no RoPE
  and no projection happen inside attention;
* scale is an argument (the workloads use 1/sqrt(128), the per-head width
  d_nope + d_rope = d_h = 128 of the Wan-1.3B backbone);
* the cached row is stored as the pair [c_t ; k^R_t], d_c values then d_rope
  values; the latent output is [B, Lq, H, d_c] and the LSE [B, H, Lq]
  (natural log, scale included), as in the other attention modes.

Parity status: pinned by ``tests/test_oracle_mla.py`` (expanded form with
explicit up-projections, pure-Python brute force, closed forms, invariances,
planted mistakes).
"""
from __future__ import annotations

import numpy as np

from .attention import attend, to64


def latent_attention(q, kv, d_c: int, scale: float, heads=None, rows=None, batches=None):
    """Absorbed latent attention.

    q  [B, Lq, H, d_c + d_rope]  absorbed, rotated queries
    kv [B, Lkv, d_c + d_rope]    cached rows [c_t ; k^R_t]
    Returns (O [B, Lq, H, d_c] latent outputs, LSE [B, H, Lq]) in float64;
    ``heads``/``rows``/``batches`` restrict the computed entries (others NaN).
    """
    q = to64(q)
    kv = to64(kv)
    B, Lq, H, dq = q.shape
    if kv.shape[-1] != dq or not 0 < d_c <= dq:
        raise ValueError("query and cached row widths disagree")
    o = np.full((B, Lq, H, d_c), np.nan)
    lse = np.full((B, H, Lq), np.nan)
    bs = range(B) if batches is None else batches
    hs = range(H) if heads is None else heads
    rs = np.arange(Lq) if rows is None else np.asarray(rows)
    for b in bs:
        keys = kv[b]
        vals = kv[b, :, :d_c]
        for h in hs:
            ob, lb = attend(q[b, rs, h, :], keys, vals, scale)
            o[b, rs, h, :] = ob
            lse[b, h, rs] = lb
    return o, lse


def absorb_query(q_nope, q_rope, w_k):
    """qa_h = [ (W^K_h)^T q^nope_h ; q^R_h ].

    q_nope [B, Lq, H, d_nope], q_rope [B, Lq, H, d_rope], w_k [H, d_nope, d_c].
    """
    q_nope = to64(q_nope)
    q_rope = to64(q_rope)
    w_k = np.asarray(w_k, dtype=np.float64)
    qc = np.einsum("blhn,hnc->blhc", q_nope, w_k)
    return np.concatenate([qc, q_rope], axis=-1)


def expanded_attention(q_nope, q_rope, c, k_rope, w_k, w_v, scale):
    """Per-head attention with keys and values rebuilt from the latent.

    c [B, Lkv, d_c], k_rope [B, Lkv, d_rope], w_k [H, d_nope, d_c],
    w_v [H, d_v, d_c].  Returns (O [B, Lq, H, d_v], LSE [B, H, Lq]).
    """
    q_nope = to64(q_nope)
    q_rope = to64(q_rope)
    c = to64(c)
    k_rope = to64(k_rope)
    w_k = np.asarray(w_k, dtype=np.float64)
    w_v = np.asarray(w_v, dtype=np.float64)
    B, Lq, H, _ = q_nope.shape
    d_v = w_v.shape[1]
    o = np.empty((B, Lq, H, d_v))
    lse = np.empty((B, H, Lq))
    for b in range(B):
        for h in range(H):
            k_h = np.concatenate([c[b] @ w_k[h].T, k_rope[b]], axis=-1)
            v_h = c[b] @ w_v[h].T
            q_h = np.concatenate([q_nope[b, :, h, :], q_rope[b, :, h, :]], axis=-1)
            o[b, :, h, :], lse[b, h, :] = attend(q_h, k_h, v_h, scale)
    return o, lse


def up_project_output(o_latent, w_v):
    """o_h = W^V_h o^latent_h: [B, Lq, H, d_c] -> [B, Lq, H, d_v]."""
    return np.einsum("blhc,hvc->blhv", to64(o_latent), np.asarray(w_v, dtype=np.float64))


def cache_scalars_per_token(n_heads: int, d_head: int, d_c: int, d_rope: int):
    """Cached scalars per token and layer: dense per-head K and V vs the latent pair."""
    return 2 * n_heads * d_head, d_c + d_rope


def visited_flops_latent(B: int, H: int, Lq: int, Lkv: int, d_c: int, d_rope: int) -> float:
    """QK^T over d_c + d_rope and PV over d_c, two flops per multiply-add."""
    return 2.0 * B * H * Lq * Lkv * ((d_c + d_rope) + d_c)
