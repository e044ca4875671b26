"""Shared helpers for the parity tests: tolerances and comparisons.

Tolerances (bf16 outputs: max-abs 2e-2 and mean-abs 2e-3; fp32 LSE: 1e-3
absolute; indices and offsets: exact) are the parity bar of the chunk-attention
path.  Expected values always come from the fp64 oracle.
"""
import numpy as np

BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
LSE_ABS = 1e-3


def to_np(t):
    if hasattr(t, "detach"):
        t = t.detach().float().cpu().numpy()
    return np.asarray(t, dtype=np.float64)


def assert_bf16_close(gpu, ref, what=""):
    g = to_np(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    d = np.abs(g - r)
    assert d.max() <= BF16_MAX_ABS, f"{what}: max-abs {d.max():.3e} > {BF16_MAX_ABS}"
    assert d.mean() <= BF16_MEAN_ABS, f"{what}: mean-abs {d.mean():.3e} > {BF16_MEAN_ABS}"
    return float(d.max()), float(d.mean())


def assert_lse_close(gpu, ref, what=""):
    g = to_np(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    ninf = np.isneginf(r)
    assert np.array_equal(np.isneginf(g), ninf), f"{what}: -inf pattern differs"
    if (~ninf).any():
        d = np.abs(g[~ninf] - r[~ninf])
        assert d.max() <= LSE_ABS, f"{what}: LSE max-abs {d.max():.3e} > {LSE_ABS}"
        return float(d.max())
    return 0.0


def config3_gap_fn(topks, block=64):
    """Margin check for the i.i.d. config-3 generator (test infrastructure).

    Returns gap_fn(q_h, k_win_h) -> per query block, the smallest fp64 score gap
    between the K-th and (K+1)-th window block over K in `topks`, with the
    scores taken from the oracle (mean-pooled blocks, inner product).
    """
    import oracle

    def fn(qh, kwin):
        n_win = kwin.shape[0] // block
        s = oracle.block_scores(qh[None, :, None, :], kwin[None, :, None, :], 0, n_win, block)[0]
        return np.min([oracle.topk_gap(s, K) for K in topks], axis=0)

    return fn


def sparse_iid_case(**kw):
    """Config 3 with i.i.d. N(0,1) window-key noise, redrawn until every query block
    has an fp64 top-K gap >= 0.05 at K = 9, 18, 36 (6.25 / 12.5 / 25 % of 144)."""
    from kv_cache_attention_chunk_b200 import workloads as W
    topks = kw.pop("topks", (9, 18, 36))
    return W.make_block_sparse(noise="iid", gap_fn=config3_gap_fn(topks), **kw)
