"""Head-aware cache compaction oracle (plain NumPy, exact).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it; the library never does, and it
shares no code with the CUDA path.

Source: Pyramid Forcing summary, methodology section 2 "head-aware pyramid KV
cache policies" (anchor heads: an adaptive-stride window that samples
representative frames uniformly; wave heads: frames kept at the head's period
P; veil heads: adjacent frames merged; every head shares the sink frames and
the forced recent frames) and section 3 (variable-length caches stored as one
flattened sequence with boundary indices).

Readings taken where the page leaves a step open (each is a test pin):

* the sink is frame 0; ``recent`` forced history frames precede the current
  chunk's frames; the policy chooses among the middle frames
  [1, hist - recent - 1];
* anchor keeps ``n`` middle frames evenly spaced with both ends included,
  position lo + i (hi - lo) / (n - 1) rounded down;
* wave keeps the middle frames f with (hist - f) mod P = 0;
* veil keeps the last ``n`` (even) middle frames, merged in adjacent pairs; a
  merged frame is the mean of the two bf16 frames (exact in fp32) rounded to
  the nearest bf16, ties to even;
* a head's frames are stored in chronological order; sequence s = b*H + h
  occupies rows cu[s] .. cu[s+1] of the flattened cache.

Arrays of bf16 values are handled as their uint16 bit patterns, so copies are
exact and the only arithmetic is the merge.
"""
from __future__ import annotations

import numpy as np

FULL, ANCHOR, WAVE, VEIL = 0, 1, 2, 3


def head_frames(policy: int, param: int, hist: int, cur: int, recent: int) -> list:
    """Frames one head keeps, in order; a merged pair is a tuple (f, f + 1)."""
    lo, hi = 1, hist - recent - 1
    middle = list(range(lo, hi + 1))
    if policy == FULL:
        mid = middle
    elif policy == ANCHOR:
        if not 1 <= param <= len(middle):
            raise ValueError("anchor count outside the middle range")
        mid = [lo] if param == 1 else [lo + (i * (hi - lo)) // (param - 1) for i in range(param)]
    elif policy == WAVE:
        if param < 1:
            raise ValueError("wave period must be >= 1")
        mid = [f for f in middle if (hist - f) % param == 0]
    elif policy == VEIL:
        if param < 0 or param % 2 or param > len(middle):
            raise ValueError("veil count must be even and within the middle range")
        tail = middle[len(middle) - param:]
        mid = [(tail[i], tail[i + 1]) for i in range(0, param, 2)]
    else:
        raise ValueError(policy)
    return [0] + mid + list(range(hist - recent, hist)) + list(range(hist, hist + cur))


def bf16_bits_round(x32: np.ndarray) -> np.ndarray:
    """float32 -> nearest bf16 (ties to even), as uint16 bit patterns (finite inputs)."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def merge_frames(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Mean of two bf16 frames, rounded to bf16 (the sum and the halving are exact in fp32)."""
    return bf16_bits_round((bf16_bits_to_f32(a_bits) + bf16_bits_to_f32(b_bits)) * np.float32(0.5))


def compact_cache(k_bits: np.ndarray, v_bits: np.ndarray, rules, frame_tokens: int, hist: int, cur: int,
                  recent: int):
    """Flatten a dense cache [B, L, H, d] (uint16 bf16 bits) under per-head rules.

    Returns (k_flat [rows, d], v_flat [rows, d], cu int32 [B*H + 1], frames per sequence).
    """
    B, L, H, d = k_bits.shape
    assert L == (hist + cur) * frame_tokens and len(rules) == H
    ks, vs, frames_all, lens = [], [], [], []
    for b in range(B):
        for h in range(H):
            frames = head_frames(rules[h][0], rules[h][1], hist, cur, recent)
            for f in frames:
                if isinstance(f, tuple):
                    ra = slice(f[0] * frame_tokens, (f[0] + 1) * frame_tokens)
                    rb = slice(f[1] * frame_tokens, (f[1] + 1) * frame_tokens)
                    ks.append(merge_frames(k_bits[b, ra, h], k_bits[b, rb, h]))
                    vs.append(merge_frames(v_bits[b, ra, h], v_bits[b, rb, h]))
                else:
                    r = slice(f * frame_tokens, (f + 1) * frame_tokens)
                    ks.append(k_bits[b, r, h])
                    vs.append(v_bits[b, r, h])
            frames_all.append(frames)
            lens.append(len(frames) * frame_tokens)
    cu = np.zeros(B * H + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    k_flat = np.concatenate(ks, 0) if ks else np.zeros((0, d), np.uint16)
    v_flat = np.concatenate(vs, 0) if vs else np.zeros((0, d), np.uint16)
    return k_flat, v_flat, cu.astype(np.int32), frames_all
