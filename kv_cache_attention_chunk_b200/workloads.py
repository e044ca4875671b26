"""Seeded synthetic inputs for chunk attention over a segmented KV cache.

This module only *builds inputs*: tensor shapes, seeded random draws and the
cache layouts that the three attention modes read (token segments, persistent
block lists, per-head frame lists and their boundary offsets).  It computes no
attention, softmax, log-sum-exp, pooling, scoring or selection.  The CPU
oracle and the CUDA path both consume exactly the tensors returned here, so
the two sides see identical bytes.

Shapes follow the workloads the pages describe:

* Wan-1.3B-shaped latents: 12 heads, head dim 128, 1560 tokens per latent
  frame (VideoMLA technical summary, "Problem statement": a 21-latent-frame
  dense cache of about 6.0 GB for Wan-1.3B).
* Dual-branch cache = sink frames + history + current chunk (ISPA summary,
  section 2, step 1 "Dual-Stream Warmup": local context = current frames plus
  sink tokens).
* Persistent blocks + local window (Sparse Forcing summary, section 2,
  component 1 "Structured Memory Decomposition").
* Per-head anchor / wave / veil caches (Pyramid Forcing summary, methodology
  section 2 "Head-aware pyramid KV cache policy"), stored flattened with
  boundary offsets (methodology section 3 "Ragged-Cache Attention").

All random draws use ``numpy.random.default_rng(seed)`` in float32 and are cast
to bfloat16 with round-to-nearest-even by ``torch.Tensor.to``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

BF16 = torch.bfloat16


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(BF16)


def _bf16_values(a: np.ndarray) -> np.ndarray:
    """float64 copy of the bf16 values (round to nearest even) of a float32 array."""
    return _bf16(a).to(torch.float64).numpy()


# ---------------------------------------------------------------------------
# Mode 1: dual-branch chunk over a segmented cache (configs 1, 2 and 5)
# ---------------------------------------------------------------------------
@dataclass
class SegmentCase:
    name: str
    B: int
    H: int
    d: int
    frame_tokens: int
    q: torch.Tensor  # [B, Lq, H, d] bf16
    k: torch.Tensor  # [B, Lkv, H, d] bf16
    v: torch.Tensor  # [B, Lkv, H, d] bf16
    branches: list  # list of branches; each a list of (start, len) token segments
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def Lq(self) -> int:
        return self.q.shape[1]

    @property
    def Lkv(self) -> int:
        return self.k.shape[1]


def dual_branch_layout(frame_tokens: int, sink_frames: int, hist_frames: int, cur_frames: int):
    """Token segments of the local and history branches.

    Cache order is chronological: sink frames, then history frames, then the
    current chunk's own frames.  Local = sink + current, history = the rest.
    """
    sink = (0, sink_frames * frame_tokens)
    hist = (sink_frames * frame_tokens, hist_frames * frame_tokens)
    cur = ((sink_frames + hist_frames) * frame_tokens, cur_frames * frame_tokens)
    local = [s for s in (sink, cur) if s[1] > 0]
    history = [hist] if hist[1] > 0 else []
    return local, history


def make_dual_branch(name: str, seed: int, H: int, d: int, frame_tokens: int,
                     q_frames: int, hist_frames: int, sink_frames: int = 1,
                     B: int = 1, q_tokens: int | None = None) -> SegmentCase:
    """N(0,1) bf16 Q, K, V; Q is the current chunk, K/V the whole cache."""
    rng = np.random.default_rng(seed)
    Lq = q_frames * frame_tokens if q_tokens is None else q_tokens
    Lkv = (sink_frames + hist_frames + q_frames) * frame_tokens
    q = _bf16(rng.standard_normal((B, Lq, H, d), dtype=np.float32))
    k = _bf16(rng.standard_normal((B, Lkv, H, d), dtype=np.float32))
    v = _bf16(rng.standard_normal((B, Lkv, H, d), dtype=np.float32))
    local, history = dual_branch_layout(frame_tokens, sink_frames, hist_frames, q_frames)
    return SegmentCase(name, B, H, d, frame_tokens, q, k, v, [local, history],
                       1.0 / float(np.sqrt(d)),
                       dict(seed=seed, sink_frames=sink_frames, hist_frames=hist_frames,
                            q_frames=q_frames))


def cfg_tiny() -> SegmentCase:
    """B=1, H=2, d=64, 8x8=64-token frames; Q 1 frame; KV 1 sink + 4 history + current."""
    return make_dual_branch("tiny", 0, H=2, d=64, frame_tokens=64, q_frames=1, hist_frames=4)


def cfg_wan13b() -> SegmentCase:
    """Wan-1.3B-shaped dense chunk: H=12, d=128, 1560 tok/frame, Q 3 frames, KV 1+20+3 frames."""
    return make_dual_branch("wan13b", 1, H=12, d=128, frame_tokens=1560, q_frames=3, hist_frames=20)


def cfg_wan14b() -> SegmentCase:
    """Wan-14B-shaped dense chunk: as Wan-1.3B with 40 heads."""
    return make_dual_branch("wan14b", 4, H=40, d=128, frame_tokens=1560, q_frames=3, hist_frames=20)


# ---------------------------------------------------------------------------
# Mode 2: persistent blocks + top-K local window blocks (config 3)
# ---------------------------------------------------------------------------
@dataclass
class SparseCase:
    name: str
    B: int
    H: int
    d: int
    block: int
    q: torch.Tensor  # [B, Lq, H, d]
    k: torch.Tensor  # [B, Lkv, H, d]  (history blocks, then the local window)
    v: torch.Tensor
    persist_idx: np.ndarray  # int32 [B*H, n_persist], absolute block ids, ascending
    window_blk0: int  # first block of the local window
    n_win_blk: int
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def Lq(self) -> int:
        return self.q.shape[1]

    @property
    def n_qblk(self) -> int:
        return -(-self.Lq // self.block)


MIN_TOPK_GAP = 0.05  # fp64 score gap at every ranking boundary the selection tests use


def make_block_sparse(name: str = "sparse", seed: int = 2, H: int = 12, d: int = 128,
                      frame_tokens: int = 32 * 48, block: int = 64, hist_frames: int = 30,
                      win_frames: int = 6, q_frames: int = 3, n_persist: int = 32,
                      B: int = 1, planted: bool = True, noise: str = "antithetic",
                      gap_fn=None, max_tries: int = 64) -> SparseCase:
    """Cache of ``hist_frames`` history frames followed by a ``win_frames`` local window.

    The query chunk is the window's last ``q_frames`` frames (its keys sit in
    the window, so each query block can pick its own "diagonal" block).

    Planted structure (``planted=True``), per head h with a random unit
    direction u_h:

    * window block b carries the offset a_{h,b} = 0.25 * (r_{h,b} - (n_win-1)/2)
      along u_h, r_{h,b} a random permutation of 0..n_win-1, added to every
      key of the block;
    * query block j carries beta_{h,j} = +/-(1 + U[0,1)) along u_h, added to
      every query of the block.

    Key noise of the window blocks (``noise``):

    * ``"antithetic"``: drawn as pairs (z, -z), randomly placed inside the
      block, so that it sums to zero over the block.  The block ranking of
      query block j is then the order of beta_{h,j} * a_{h,b} up to bf16
      rounding, neighbouring ranks at least about 0.25 * |beta| apart: the
      selection is unambiguous by construction, with no scoring needed here.
    * ``"iid"``: plain N(0, 1), as every other key.  The ranking margin then
      has to be checked: ``gap_fn(q_h, k_win_h)`` (supplied by the caller; this
      module computes no scores) receives one head's query rows [Lq, d] and
      window key rows [n_win * block, d] as float64 copies of the bf16 values
      and returns, per query block, the smallest score gap at the ranking
      boundaries the caller cares about.  Every query block whose gap is below
      MIN_TOPK_GAP gets a new beta and new query noise, drawn from the sub-seed
      (seed, b, h, j, try), until all pass (at most ``max_tries`` rounds).

    Persistent blocks carry no offset.
    """
    assert frame_tokens % block == 0
    rng = np.random.default_rng(seed)
    bpf = frame_tokens // block
    n_hist_blk = hist_frames * bpf
    n_win_blk = win_frames * bpf
    Lkv = (n_hist_blk + n_win_blk) * block
    Lq = q_frames * frame_tokens
    n_qblk = Lq // block
    q = rng.standard_normal((B, Lq, H, d), dtype=np.float32)
    k = rng.standard_normal((B, Lkv, H, d), dtype=np.float32)
    v = rng.standard_normal((B, Lkv, H, d), dtype=np.float32)
    persist = np.zeros((B * H, n_persist), dtype=np.int32)
    meta = dict(seed=seed, hist_frames=hist_frames, win_frames=win_frames, q_frames=q_frames,
                frame_tokens=frame_tokens, planted=planted)
    if noise not in ("antithetic", "iid"):
        raise ValueError(noise)
    if planted:
        u = rng.standard_normal((B, H, d))
        u /= np.linalg.norm(u, axis=-1, keepdims=True)
        r = np.stack([rng.permutation(n_win_blk) for _ in range(B * H)]).reshape(B, H, n_win_blk)
        a = 0.25 * (r - (n_win_blk - 1) / 2.0)
        sign = rng.choice(np.array([-1.0, 1.0]), size=(B, H, n_qblk))
        beta = sign * (1.0 + rng.random((B, H, n_qblk)))
        half = block // 2
        w0 = n_hist_blk * block
        for b in range(B):
            for h in range(H):
                for wb in range(n_win_blk):
                    s = w0 + wb * block
                    if noise == "antithetic":
                        z = rng.standard_normal((half, d), dtype=np.float32)
                        rows = np.concatenate([z, -z], axis=0)[rng.permutation(block)]
                    else:
                        rows = k[b, s:s + block, h, :]
                    k[b, s:s + block, h, :] = rows + (a[b, h, wb] * u[b, h]).astype(np.float32)
                for j in range(n_qblk):
                    q[b, j * block:(j + 1) * block, h, :] += (beta[b, h, j] * u[b, h]).astype(np.float32)
        meta.update(a=a, beta=beta, u=u, noise=noise)
        if noise == "iid":
            if gap_fn is None:
                raise ValueError("noise='iid' needs gap_fn to check the ranking margin")
            min_gap = np.inf
            tries = 0
            for b in range(B):
                for h in range(H):
                    kw = _bf16_values(k[b, w0:w0 + n_win_blk * block, h, :])
                    for t in range(max_tries + 1):
                        gaps = np.asarray(gap_fn(_bf16_values(q[b, :, h, :]), kw), dtype=np.float64)
                        bad = np.nonzero(gaps < MIN_TOPK_GAP)[0]
                        if len(bad) == 0:
                            min_gap = min(min_gap, float(gaps.min()))
                            tries = max(tries, t)
                            break
                        if t == max_tries:
                            raise RuntimeError(f"query blocks {bad.tolist()} of (b={b}, h={h}) still have a "
                                               f"top-K gap below {MIN_TOPK_GAP} after {max_tries} redraws")
                        for j in bad:
                            sub = np.random.default_rng([seed, b, h, int(j), t + 1])
                            bj = sub.choice(np.array([-1.0, 1.0])) * (1.0 + sub.random())
                            lo, hi = j * block, min(Lq, (j + 1) * block)
                            q[b, lo:hi, h, :] = (sub.standard_normal((hi - lo, d), dtype=np.float32) +
                                                 (bj * u[b, h]).astype(np.float32))
                            beta[b, h, j] = bj
            meta.update(min_topk_gap=min_gap, redraw_rounds=tries)
    for bh in range(B * H):
        persist[bh] = np.sort(rng.choice(n_hist_blk, size=n_persist, replace=False)).astype(np.int32)
    return SparseCase(name, B, H, d, block, _bf16(q), _bf16(k), _bf16(v), persist,
                      n_hist_blk, n_win_blk, 1.0 / float(np.sqrt(d)), meta)


def cfg_sparse() -> SparseCase:
    """12 heads, d=128, 32x48-token frames in 64-token blocks; 30 history + 6 window frames."""
    return make_block_sparse()


SPARSE_TOPK_FRACTIONS = (0.0625, 0.125, 0.25, 1.0)


def topk_for_fraction(frac: float, n_win_blk: int) -> int:
    return max(1, int(round(frac * n_win_blk)))


def random_selection(seed: int, BH: int, n_qblk: int, n_win_blk: int, topk: int) -> np.ndarray:
    """Arbitrary ascending window-block index sets (for kernel tests that bypass scoring)."""
    rng = np.random.default_rng(seed)
    out = np.zeros((BH, n_qblk, topk), dtype=np.int32)
    for i in range(BH):
        for j in range(n_qblk):
            out[i, j] = np.sort(rng.choice(n_win_blk, size=topk, replace=False))
    return out


# ---------------------------------------------------------------------------
# Mode 3: ragged per-head cache, flattened with boundary offsets (config 4)
# ---------------------------------------------------------------------------
@dataclass
class RaggedCase:
    name: str
    B: int
    H: int
    d: int
    frame_tokens: int
    q: torch.Tensor  # [B, Lq, H, d]
    k: torch.Tensor  # [sum L, d]  sequence s = b*H + h occupies rows cu[s]..cu[s+1]
    v: torch.Tensor
    cu_seqlens: np.ndarray  # int32 [B*H + 1]
    frames: list  # per sequence: list of frame labels (int, or (f0, f1) for a merged pair)
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def Lq(self) -> int:
        return self.q.shape[1]


def pyramid_head_frames(policy: str, hist_frames: int, q_frames: int, param: int = 0,
                        recent: int = 2, veil_frames: int = 8) -> list:
    """Frame list of one head under the anchor / wave / veil policies.

    Every head keeps frame 0 (sink) and the last ``recent`` history frames; the
    policy picks from the middle history [1, hist_frames - recent - 1]; the
    current chunk's ``q_frames`` frames follow.  Order is chronological.

    * ``anchor``: ``param`` evenly spaced middle frames, both ends included.
    * ``wave``: middle frames f with (hist_frames - f) % param == 0, i.e. a
      period-``param`` comb aligned to the current frame.
    * ``veil``: the ``veil_frames`` middle frames just before the recent ones,
      merged in adjacent pairs (a merged pair is written as a tuple).
    * ``full``: every history frame (used to reduce ragged mode to dense).
    """
    lo, hi = 1, hist_frames - recent - 1
    if policy == "anchor":
        mid = [int(x) for x in np.linspace(lo, hi, param)]
    elif policy == "wave":
        mid = [f for f in range(lo, hi + 1) if (hist_frames - f) % param == 0]
    elif policy == "veil":
        first = hi - veil_frames + 1
        mid = [(f, f + 1) for f in range(first, hi + 1, 2)]
    elif policy == "full":
        mid = list(range(lo, hi + 1))
    else:
        raise ValueError(policy)
    recent_frames = list(range(hist_frames - recent, hist_frames))
    cur = list(range(hist_frames, hist_frames + q_frames))
    return [0] + mid + recent_frames + cur


def pyramid_policies(H: int = 12):
    """Heads 0-3 anchor (8 frames), 4-7 wave (P = 2, 3, 4, 5), 8-11 veil."""
    assert H == 12
    return ([("anchor", 8)] * 4 + [("wave", p) for p in (2, 3, 4, 5)] + [("veil", 0)] * 4)


def make_ragged(name: str = "ragged", seed: int = 3, H: int = 12, d: int = 128,
                frame_tokens: int = 1560, hist_frames: int = 60, q_frames: int = 3,
                policies=None, B: int = 1) -> RaggedCase:
    """Per-head caches built from one seeded dense cache of hist+q frames.

    Each sequence's K/V are its frames' tokens concatenated chronologically; a
    veil pair is stored as the token-wise fp32 mean of its two bf16 frames,
    rounded to bf16 (cache construction, before any attention runs).
    """
    if policies is None:
        policies = pyramid_policies(H)
    rng = np.random.default_rng(seed)
    F = hist_frames + q_frames
    q = _bf16(rng.standard_normal((B, q_frames * frame_tokens, H, d), dtype=np.float32))
    ks, vs, frames_all, lens = [], [], [], []
    for b in range(B):
        for h in range(H):
            kd = _bf16(rng.standard_normal((F, frame_tokens, d), dtype=np.float32)).float()
            vd = _bf16(rng.standard_normal((F, frame_tokens, d), dtype=np.float32)).float()
            pol, par = policies[h]
            frames = pyramid_head_frames(pol, hist_frames, q_frames, par)
            kk, vv = [], []
            for f in frames:
                if isinstance(f, tuple):
                    kk.append(((kd[f[0]] + kd[f[1]]) * 0.5).to(BF16))
                    vv.append(((vd[f[0]] + vd[f[1]]) * 0.5).to(BF16))
                else:
                    kk.append(kd[f].to(BF16))
                    vv.append(vd[f].to(BF16))
            ks.append(torch.cat(kk, 0))
            vs.append(torch.cat(vv, 0))
            frames_all.append(frames)
            lens.append(len(frames) * frame_tokens)
    cu = np.zeros(B * H + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    assert cu[-1] < 2 ** 31
    return RaggedCase(name, B, H, d, frame_tokens, q, torch.cat(ks, 0).contiguous(),
                      torch.cat(vs, 0).contiguous(), cu.astype(np.int32), frames_all,
                      1.0 / float(np.sqrt(d)),
                      dict(seed=seed, hist_frames=hist_frames, q_frames=q_frames))


def cfg_ragged() -> RaggedCase:
    """12 heads, d=128, 1560 tok/frame, 60 history frames, Q a 3-frame chunk."""
    return make_ragged()


# ---------------------------------------------------------------------------
# Standalone merge inputs
# ---------------------------------------------------------------------------
def make_merge_inputs(seed: int, B: int, Lq: int, H: int, d: int, neg_inf_frac: float = 0.0):
    """Two bf16 partial outputs and fp32 LSEs of plausible magnitude."""
    rng = np.random.default_rng(seed)
    oa = _bf16(rng.standard_normal((B, Lq, H, d), dtype=np.float32) * 0.1)
    ob = _bf16(rng.standard_normal((B, Lq, H, d), dtype=np.float32) * 0.1)
    la = (rng.standard_normal((B, H, Lq)) * 2 + 8).astype(np.float32)
    lb = (rng.standard_normal((B, H, Lq)) * 2 + 9).astype(np.float32)
    if neg_inf_frac > 0:
        la[rng.random(la.shape) < neg_inf_frac] = -np.inf
        lb[rng.random(lb.shape) < neg_inf_frac] = -np.inf
    return oa, torch.from_numpy(la), ob, torch.from_numpy(lb)


# ---------------------------------------------------------------------------
# Latent (VideoMLA) cache: one head-shared [c_t ; k^R_t] row per token
# ---------------------------------------------------------------------------
@dataclass
class LatentCase:
    name: str
    B: int
    H: int
    d_c: int
    d_rope: int
    q: torch.Tensor   # [B, Lq, H, d_c + d_rope] bf16, absorbed and rotated queries
    kv: torch.Tensor  # [B, Lkv, d_c + d_rope] bf16, cached rows [c ; k_R]
    scale: float
    meta: dict = field(default_factory=dict)

    @property
    def Lq(self) -> int:
        return self.q.shape[1]

    @property
    def Lkv(self) -> int:
        return self.kv.shape[1]


def make_latent(name: str = "latent", seed: int = 5, B: int = 1, H: int = 12, Lq: int = 4680,
                Lkv: int = 32760, d_c: int = 192, d_rope: int = 32, d_head: int = 128,
                q_std: float = 1.0) -> LatentCase:
    """N(0, q_std^2) queries and N(0, 1) cached rows, both bf16.

    Defaults: the Wan-1.3B shape (12 heads of width 128, 1560 tokens per latent
    frame) with a 3-frame query chunk over a 21-latent-frame cache, and the
    default latent budget d_c = 192, d_rope = 32 (VideoMLA technical summary,
    "Methodology", memory reduction).  Scale 1/sqrt(d_head).
    """
    rng = np.random.default_rng(seed)
    dq = d_c + d_rope
    q = _bf16(rng.standard_normal((B, Lq, H, dq), dtype=np.float32) * np.float32(q_std))
    kv = _bf16(rng.standard_normal((B, Lkv, dq), dtype=np.float32))
    return LatentCase(name, B, H, d_c, d_rope, q, kv, 1.0 / float(np.sqrt(d_head)),
                      dict(seed=seed, q_std=q_std))


def cfg_latent() -> LatentCase:
    """VideoMLA-shaped chunk on Wan-1.3B: H=12, Q 3 frames (4680), cache 21 frames (32 760)."""
    return make_latent()
