#!/usr/bin/env python
"""Benchmark of chunk attention over a segmented KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload: the Wan-14B-shaped dense dual-branch chunk (B=1, 40 heads,
d=128, 1560 tokens per latent frame; Q = a 3-frame chunk of 4680 tokens; KV =
1 sink + 20 history + 3 current frames = 37 440 tokens; local branch = sink +
current, history branch = the 20 history frames; both branch outputs with
their LSEs plus the LSE-merged output).  One step = one vkv_chunk_attn call.
Metric: effective TFLOP/s counting 4*d per visited (query, key) pair, its
fraction of the measured bf16 dense peak, and ms per chunk.

Multi-GPU (torchrun, one process per GPU): by default every rank runs its own
chunk (independent seeds) with no collective on the data path (weak scaling).
--split heads / --split keys instead split ONE chunk over the ranks (strong
scaling): by head (each rank its heads; --gather all-gathers the merged
output), or by key range (each rank attends over one part of the key set and
rank 0 merges the partials it receives with the LSE merge).  The time is the
max over ranks; rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle on the host cores (bounded samples
of the same workload); under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_attention_chunk_b200 import workloads as W  # noqa: E402

METRIC = "chunk-attn effective TFLOP/s & % of bf16 tensor peak; ms per 3-frame chunk"
WORKLOAD = ("wan14b dense dual-branch chunk: B=1, H=40, d=128, 1560 tok/frame, Q 4680 (3 frames), "
            "KV 37440 (1 sink + 20 history + 3 current frames), local=sink+current, history=20 frames, "
            "outputs O/LSE per branch + LSE-merged O/LSE")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# distributed plumbing (also exercised by the gloo tests)
# ---------------------------------------------------------------------------
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)), int(os.environ.get("WORLD_SIZE", 1))


def dist_setup(backend: str | None = None):
    import torch.distributed as dist
    rank, local, world = dist_env()
    if world > 1 and not dist.is_initialized():
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        import datetime
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, local, world


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device="cpu") -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws an independent chunk of the same shape."""
    return base + 7919 * rank


def headline_case(rank: int = 0):
    return W.make_dual_branch("wan14b", rank_seed(4, rank), H=40, d=128, frame_tokens=1560, q_frames=3,
                              hist_frames=20)


def headline_flops() -> int:
    loc, hist = W.dual_branch_layout(1560, 1, 20, 3)
    n = sum(l for _, l in loc) + sum(l for _, l in hist)
    return 4 * 128 * 40 * 4680 * n


# ---------------------------------------------------------------------------
# peaks, clocks, profiles
# ---------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


ATTN_SOURCES = ("vkv_attn.cu", "vkv_attn_kernel.cuh", "vkv_internal.h", "vkv_ptx.cuh", "vkv_topk.cuh")


def headline_split(vkv, q, k, v, branches, scale) -> bool:
    """True when the call's schedule cuts units along the key axis (a non-zero
    workspace): the piece-enabled attention instantiation runs, then the combine kernel."""
    return vkv.vkv_chunk_attn_workspace_size(vkv.segments_args(q, k, v, branches, scale)) > 0


def headline_kernel_name(vkv, q, k, v, case) -> str:
    """The attention instantiation the headline call runs."""
    pc = headline_split(vkv, q, k, v, case.branches, case.scale)
    return f"chunk_attn_kernel<128, 0, {int(pc)}>"


def mcycles(ms, clocks):
    """Milliseconds at the median SM clock under load, as millions of SM cycles."""
    mhz = (clocks or {}).get("sm_mhz")
    return ms * mhz / 1000.0 if mhz else None


def kernel_source_hash() -> str:
    """Hash of the attention kernel's code (ties recorded ncu counters to a kernel version).

    Comments and whitespace are left out, so an edit of the prose alone keeps the record.
    """
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kv_cache_attention_chunk_b200", "csrc")
    for name in ATTN_SOURCES:
        with open(os.path.join(csrc, name)) as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        src = " ".join(src.split())
        h.update(name.encode() + src.encode())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it matches this source."""
    p = os.path.join(ROOT, "profiles", "attn_wan14b_traffic.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        if d.get("kernel_source_hash") == kernel_source_hash():
            return float(d["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.idx, self.period, self.proc, self.out = gpu_index, period_ms, None, ""

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", f"-lms={self.period}"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            self.out = ""
        rows = [r.split(", ") for r in self.out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        loaded = [s for s, p in zip(sm, pw) if p > 200] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "reasons": reasons}


def host_cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info()]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


# ---------------------------------------------------------------------------
# the oracle on the host (CPU baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(case, rows: int, head: int = 0):
    """Run the fp64 oracle (both branches + their LSE merge) on `rows` query rows of one head."""
    import oracle
    q = oracle.to64(case.q[0, :rows, head])
    k = oracle.to64(case.k[0, :, head])
    v = oracle.to64(case.v[0, :, head])
    t0 = time.perf_counter()
    parts = []
    for br in case.branches:
        idx = oracle.segment_rows(br)
        parts.append(oracle.attend(q, k[idx], v[idx], case.scale))
    oracle.lse_merge(parts[0][0], parts[0][1], parts[1][0], parts[1][1])
    dt = time.perf_counter() - t0
    n_keys = sum(l for br in case.branches for _, l in br)
    return dt, 4 * case.d * rows * n_keys


def calibrate_rows(case, seconds: float) -> int:
    dt, _ = oracle_sample(case, 32)
    rows = int(32 * seconds / max(dt, 1e-3))
    return max(16, min(case.Lq, rows))


def cpu_baseline(case, seconds: float = 15.0):
    """The oracle as it stands on the host cores, on about `seconds` of work."""
    rows = calibrate_rows(case, seconds)
    heads = 1
    if rows >= case.Lq:
        dt1, _ = oracle_sample(case, case.Lq, head=0)
        heads = max(1, min(case.H, int(seconds / max(dt1, 1e-3))))
    t = 0.0
    fl = 0
    for h in range(heads):
        dt, f = oracle_sample(case, rows, head=h)
        t += dt
        fl += f
    return {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
            "sample": f"heads 0..{heads - 1}, query rows 0..{rows - 1} of the wan14b chunk (both branches "
                      f"+ LSE merge, fp64 NumPy), {t:.1f} s"}


def headline_config(world: int) -> dict:
    """The workload of the headline line (the same for every arm of the same launch)."""
    return {"workload": WORKLOAD, "parallelism": f"independent chunk per GPU x{world}",
            "l2": "no flush: each step reads 961 MB of inputs, larger than the 126 MB L2",
            "flops_per_chunk": headline_flops()}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    case = headline_case(0)
    budget = 150.0
    per_step = max(0.05, budget / max(1, args.steps + args.warmup))
    rows = calibrate_rows(case, per_step)
    for _ in range(args.warmup):
        oracle_sample(case, rows)
    tot_t, tot_f = 0.0, 0
    for _ in range(args.steps):
        dt, fl = oracle_sample(case, rows)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": headline_config(world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": host_cores(), "kind": "oracle",
                             "sample": f"head 0, query rows 0..{rows - 1} of the chunk per step (both branches "
                                       f"+ LSE merge, fp64 NumPy)"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
class L2Flush:
    """Leaves L2 without the next call's inputs, outside the timed interval.

    A buffer larger than L2 is written, then another one is read: the call
    then starts with a cold L2 that holds only clean lines.  (After the write
    alone, L2 is full of dirty lines whose write-back to DRAM would run during
    the timed call and be charged to it: ~30 MB on the Wan-1.3B merge.)
    """

    def __init__(self, dev, nbytes: int):
        self.w = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(nbytes // 4, dtype=torch.float32, device=dev)
        self.acc = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.acc)


def timed(fn, iters: int, stream, flush=None) -> list:
    """Device time of each call of `fn` (ms), CUDA events on `stream`.

    The calls are queued behind a device-side sleep, so the host-side cost of
    each call (argument marshalling, launch) is hidden and only GPU time is
    measured.  With `flush` (an L2Flush), L2 is emptied of the call's inputs
    before every call, outside the timed interval, so each call starts with a
    cold L2.
    """
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    torch.cuda._sleep(int(4e5) * iters + int(2e6))  # ~0.2 ms of host enqueue time per call at ~2 GHz
    for a, b in evs:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


L2_FLUSH_BYTES = 256 << 20  # twice the B200 L2


def extras(dev, peaks):
    """Per-mode timings of the other workloads (parity cases, reported for context)."""
    from kv_cache_attention_chunk_b200 import vkv
    import oracle
    out = {}
    st = torch.cuda.current_stream()
    flush = L2Flush(dev, L2_FLUSH_BYTES)
    # Wan-1.3B-shaped dense dual-branch chunk
    c = W.cfg_wan13b()
    q, k, v = c.q.to(dev), c.k.to(dev), c.v.to(dev)
    res = vkv.chunk_attn_segments(q, k, v, c.branches, scale=c.scale)
    ms = statistics.median(timed(lambda: vkv.chunk_attn_segments(q, k, v, c.branches, scale=c.scale, out=res),
                                 20, st))
    fl = oracle.visited_flops_segments(1, 12, c.Lq, 128, c.branches)
    out["wan13b_dense"] = {"ms": ms, "tflops": fl / ms / 1e9}
    # standalone merge on the Wan-1.3B partials
    mo = vkv.lse_merge(res["o"][0], res["lse"][0], res["o"][1], res["lse"][1])
    ms = statistics.median(timed(lambda: vkv.lse_merge(res["o"][0], res["lse"][0], res["o"][1], res["lse"][1],
                                                       out=mo), 50, st, flush))
    nbytes = 3 * res["o"][0].numel() * 2 + 3 * res["lse"][0].numel() * 4
    out["lse_merge_wan13b"] = {"ms": ms, "gbs": nbytes / ms / 1e6, "bytes": nbytes,
                               "frac_hbm": nbytes / ms / 1e6 / peaks["hbm_gbs"]}
    del q, k, v, res, mo
    # standalone merge at the headline size (40 heads): inputs larger than L2
    oa, la, ob, lb = (t.to(dev) for t in W.make_merge_inputs(5, 1, 4680, 40, 128))
    mo = vkv.lse_merge(oa, la, ob, lb)
    ms = statistics.median(timed(lambda: vkv.lse_merge(oa, la, ob, lb, out=mo), 50, st, flush))
    nbytes = 3 * oa.numel() * 2 + 3 * la.numel() * 4
    out["lse_merge_wan14b"] = {"ms": ms, "gbs": nbytes / ms / 1e6, "bytes": nbytes,
                               "frac_hbm": nbytes / ms / 1e6 / peaks["hbm_gbs"]}
    del oa, la, ob, lb, mo
    # block-sparse: persistent + top-K window blocks
    c = W.cfg_sparse()
    q, k, v = c.q.to(dev), c.k.to(dev), c.v.to(dev)
    pers = torch.from_numpy(c.persist_idx).to(dev)
    kbar = vkv.block_pool(k, c.window_blk0, c.n_win_blk)  # window block means, cached as blocks enter
    sp = {}
    for frac in W.SPARSE_TOPK_FRACTIONS:
        K = W.topk_for_fraction(frac, c.n_win_blk)
        ws = torch.empty(vkv.vkv_block_select_workspace_size(1, 12, c.Lq, c.n_win_blk, 64, 128),
                         dtype=torch.uint8, device=dev)
        idx, _, order = vkv.block_select(q, k, c.window_blk0, c.n_win_blk, K, workspace=ws, order=True)
        ms_sel = statistics.median(timed(lambda: vkv.block_select(q, k, c.window_blk0, c.n_win_blk, K,
                                                                  workspace=ws, out_idx=idx, out_order=order),
                                         30, st, flush))
        o = vkv.chunk_attn_block_sparse(q, k, v, pers, idx, c.window_blk0, c.n_win_blk, scale=c.scale,
                                        qblk_order=order)
        ms_att = statistics.median(timed(lambda: vkv.chunk_attn_block_sparse(
            q, k, v, pers, idx, c.window_blk0, c.n_win_blk, scale=c.scale, out=o, qblk_order=order), 20, st))
        ms_nat = statistics.median(timed(lambda: vkv.chunk_attn_block_sparse(
            q, k, v, pers, idx, c.window_blk0, c.n_win_blk, scale=c.scale, out=o), 20, st))
        # selection inside the attention kernel (from the cached means; the query-block
        # order is a previous selection's) against the same two steps as separate launches
        fsel = torch.empty_like(idx)
        o_f = vkv.chunk_attn_block_sparse(q, k, v, pers, None, c.window_blk0, c.n_win_blk, scale=c.scale,
                                          qblk_order=order, kbar=kbar, topk=K, sel_out=fsel)
        ms_fused = statistics.median(timed(lambda: vkv.chunk_attn_block_sparse(
            q, k, v, pers, None, c.window_blk0, c.n_win_blk, scale=c.scale, out=o_f, qblk_order=order, kbar=kbar,
            topk=K, sel_out=fsel), 20, st))
        ms_two = statistics.median(timed(lambda: (
            vkv.block_select(q, k, c.window_blk0, c.n_win_blk, K, workspace=ws, out_idx=idx, kbar=kbar),
            vkv.chunk_attn_block_sparse(q, k, v, pers, idx, c.window_blk0, c.n_win_blk, scale=c.scale, out=o,
                                        qblk_order=order, split=False)), 20, st))
        fl = oracle.visited_flops_sparse(1, 12, c.Lq, 128, 64, c.persist_idx.shape[1], K)
        sel_bytes = (c.Lq + c.n_win_blk * 64) * 12 * 128 * 2
        sp[f"K{K}"] = {"attn_ms": ms_att, "attn_tflops": fl / ms_att / 1e9, "attn_ms_natural_order": ms_nat,
                       "select_ms": ms_sel, "select_gbs": sel_bytes / ms_sel / 1e6,
                       "chunk_ms": ms_sel + ms_att, "visited_frac": (32 + K) / (32 + c.n_win_blk),
                       "fused_select": {"ms": ms_fused, "tflops": fl / ms_fused / 1e9,
                                        "two_launch_ms": ms_two}}
    # representatives of the window blocks cached as blocks enter the cache: selection then
    # pools only the query blocks (14.2 MB read instead of 42.5 MB)
    K = W.topk_for_fraction(W.SPARSE_TOPK_FRACTIONS[0], c.n_win_blk)
    ms_pool = statistics.median(timed(lambda: vkv.block_pool(k, c.window_blk0, c.n_win_blk, out=kbar), 30, st,
                                      flush))
    idx, _, order = vkv.block_select(q, k, c.window_blk0, c.n_win_blk, K, workspace=ws, order=True, kbar=kbar)
    ms_cached = statistics.median(timed(lambda: vkv.block_select(q, k, c.window_blk0, c.n_win_blk, K, workspace=ws,
                                                                 out_idx=idx, out_order=order, kbar=kbar),
                                        30, st, flush))
    # persistent-memory update: the oldest window frame (24 blocks) leaves the window
    pidx, _ = vkv.persist_update(q, k, pers, c.window_blk0, 24)
    pws = torch.empty(vkv.vkv_persist_update_workspace_size(1, 12, c.Lq, pers.shape[1], 24, 64, 128),
                      dtype=torch.uint8, device=dev)
    ms_pu = statistics.median(timed(lambda: vkv.persist_update(q, k, pers, c.window_blk0, 24, out_idx=pidx,
                                                               workspace=pws), 30, st, flush))
    pu_bytes = (c.Lq + (pers.shape[1] + 24) * 64) * 12 * 128 * 2
    sp["persist_update"] = {"ms": ms_pu, "gbs": pu_bytes / ms_pu / 1e6, "candidates": pers.shape[1] + 24}
    q_bytes = c.Lq * 12 * 128 * 2
    sp["select_cached_representatives"] = {"K": K, "select_ms": ms_cached, "q_read_gbs": q_bytes / ms_cached / 1e6,
                                           "window_pool_ms": ms_pool}
    full = sp[f"K{c.n_win_blk}"]["attn_ms"]
    ks = [kk for kk in sp if kk.startswith("K")]
    for kk in ks:
        sp[kk]["time_frac_of_K_all"] = sp[kk]["attn_ms"] / full
    xs = np.array([sp[kk]["visited_frac"] for kk in ks])
    ys = np.array([sp[kk]["time_frac_of_K_all"] for kk in ks])
    slope, icpt = np.polyfit(xs, ys, 1)
    r2 = 1.0 - float(((ys - (slope * xs + icpt)) ** 2).sum()) / float(((ys - ys.mean()) ** 2).sum())
    sp["scaling_fit"] = {"slope": float(slope), "intercept": float(icpt), "r2": r2,
                         "target": "t(K)/t(144) = visited fraction: slope 1, intercept 0"}
    out["sparse"] = sp
    del q, k, v
    # head-aware compaction of a dense cache into the ragged one (config-4 shape and policies)
    ft, hist, cur, recent = 1560, 60, 3, 2
    rules = [(vkv.HEAD_ANCHOR, 8)] * 4 + [(vkv.HEAD_WAVE, p) for p in (2, 3, 4, 5)] + [(vkv.HEAD_VEIL, 8)] * 4
    g = torch.Generator(device=dev).manual_seed(12)
    kd = torch.randn((1, (hist + cur) * ft, 12, 128), generator=g, device=dev).to(torch.bfloat16)
    vd = torch.randn((1, (hist + cur) * ft, 12, 128), generator=g, device=dev).to(torch.bfloat16)
    kc, vc, cuc, cuh = vkv.compact_cache(kd, vd, rules, ft, hist, cur, recent)
    a = vkv.vkv_compact_args()
    a.B, a.H, a.d, a.frame_tokens, a.hist_frames, a.cur_frames, a.recent_frames = 1, 12, 128, ft, hist, cur, recent
    a.k_src, a.v_src = vkv.tensor_desc(kd), vkv.tensor_desc(vd)
    rr = (vkv.vkv_head_rule * 12)(*[vkv.vkv_head_rule(int(pp), int(x)) for pp, x in rules])
    a.rules = ctypes.cast(rr, ctypes.POINTER(vkv.vkv_head_rule))
    a.k_out, a.v_out, a.out_rows, a.cu_seqlens = kc.data_ptr(), vc.data_ptr(), kc.shape[0], cuc.data_ptr()
    ms = statistics.median(timed(lambda: vkv.vkv_compact_cache(a, st.cuda_stream), 30, st, flush))
    rows = int(cuh[-1])
    merged_rows = 4 * 4 * ft  # four veil heads, four merged pairs each
    nbytes = 2 * (rows + merged_rows) * 128 * 2 + 2 * rows * 128 * 2
    out["compaction_cfg4"] = {"ms": ms, "gbs": nbytes / ms / 1e6, "bytes": nbytes,
                              "frac_hbm": nbytes / ms / 1e6 / peaks["hbm_gbs"]}
    del kd, vd, kc, vc
    # ragged per-head cache
    c = W.cfg_ragged()
    q, k, v = c.q.to(dev), c.k.to(dev), c.v.to(dev)
    cu = torch.from_numpy(c.cu_seqlens).to(dev)
    o = vkv.chunk_attn_ragged(q, k, v, cu, c.cu_seqlens, scale=c.scale)
    ms = statistics.median(timed(lambda: vkv.chunk_attn_ragged(q, k, v, cu, c.cu_seqlens, scale=c.scale, out=o),
                                 20, st))
    fl = oracle.visited_flops_ragged(1, 12, c.Lq, 128, c.cu_seqlens)
    out["ragged"] = {"ms": ms, "tflops": fl / ms / 1e9}
    del q, k, v, o
    # latent (VideoMLA) attention: the Wan-1.3B 3-frame chunk over a 21-frame head-shared cache
    lat = {}
    for d_c in (192, 128):
        c = W.make_latent(d_c=d_c)
        q, kv = c.q.to(dev), c.kv.to(dev)
        o = vkv.latent_attn(q, kv, d_c, scale=c.scale)
        ms = statistics.median(timed(lambda: vkv.latent_attn(q, kv, d_c, scale=c.scale, out=o), 20, st, flush))
        fl = oracle.visited_flops_latent(c.B, c.H, c.Lq, c.Lkv, d_c, c.d_rope)
        lat[f"d_c{d_c}"] = {"ms": ms, "tflops": fl / ms / 1e9, "frac_bf16": fl / ms / 1e9 / peaks["bf16_tflops"],
                            "cache_bytes_per_layer": kv.numel() * 2,
                            "dense_cache_bytes_per_layer": 2 * c.H * 128 * c.Lkv * 2}
        del q, kv, o
    # a batch of 8 chunks, each over its own 21-frame latent cache (the batch size the
    # smaller cache makes room for)
    c = W.make_latent(B=8)
    q, kv = c.q.to(dev), c.kv.to(dev)
    o = vkv.latent_attn(q, kv, c.d_c, scale=c.scale)
    ms = statistics.median(timed(lambda: vkv.latent_attn(q, kv, c.d_c, scale=c.scale, out=o), 10, st, flush))
    fl = oracle.visited_flops_latent(c.B, c.H, c.Lq, c.Lkv, c.d_c, c.d_rope)
    lat["d_c192_batch8"] = {"ms": ms, "tflops": fl / ms / 1e9, "frac_bf16": fl / ms / 1e9 / peaks["bf16_tflops"],
                            "ms_per_chunk": ms / c.B}
    del q, kv, o
    out["latent_wan13b"] = lat
    return out


def run_ours(args):
    from kv_cache_attention_chunk_b200 import build, vkv
    rank, local, world = dist_setup()
    if local == 0:
        build.build()
    barrier()
    vkv.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    case = headline_case(rank)
    q, k, v = case.q.to(dev), case.k.to(dev), case.v.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    out = vkv.chunk_attn_segments(q, k, v, case.branches, scale=case.scale, err=err)
    stream = torch.cuda.current_stream(dev)

    def step():
        vkv.chunk_attn_segments(q, k, v, case.branches, scale=case.scale, err=err, out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    sampler = ClockSampler(vis.split(",")[local].strip() if vis else local)
    if rank == 0 or world == 1:
        sampler.start()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if (rank == 0 or world == 1) else None
    total_ms = e0.elapsed_time(e1)
    launch_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(total_ms, dev if world > 1 and torch.distributed.get_backend() == "nccl" else "cpu")
    ms_step = total_ms / args.steps
    fl = headline_flops()
    value = world * fl / (ms_step * 1e-3) / 1e12
    avg_launch = statistics.mean(launch_ms)
    achieved = fl / (avg_launch * 1e-3) / 1e12
    # our kernels per step: the attention kernel, and the piece combine kernel behind
    # it when the schedule cuts units along the key axis
    launches_per_step = 2 if headline_split(vkv, q, k, v, case.branches, case.scale) else 1
    peak = float(peaks["bf16_tflops"])
    peak_sus = float(peaks.get("bf16_tflops_sustained", 0.0)) or None

    # end to end through the C ABI with host buffers: every step uploads its inputs from pinned
    # host memory, runs the call and reads its outputs back.  Two device buffer sets pipeline the
    # steps as a serving loop would: step i+1's upload and step i-1's read-back (each on its own
    # stream, so the two copy directions overlap) run while step i's attention runs.
    hq, hk, hv = (t.cpu().pin_memory() for t in (case.q, case.k, case.v))

    def outs(o):
        return o["o"] + [o["o_merged"]] + o["lse"] + [o["lse_merged"]]

    hout = [t.cpu().pin_memory() for t in outs(out)]
    q2, k2, v2 = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    out2 = vkv.chunk_attn_segments(q, k, v, case.branches, scale=case.scale, err=err)
    sets = [(q, k, v, out), (q2, k2, v2, out2)]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        done_comp, done_down = [None, None], [None, None]
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(s_up)
        for i in range(n):
            qq, kk, vv, oo = sets[i % 2]
            if done_comp[i % 2] is not None:
                s_up.wait_event(done_comp[i % 2])  # step i-2 has read this buffer set
            with torch.cuda.stream(s_up):
                qq.copy_(hq, non_blocking=True)
                kk.copy_(hk, non_blocking=True)
                vv.copy_(hv, non_blocking=True)
            up = torch.cuda.Event()
            up.record(s_up)
            stream.wait_event(up)
            if done_down[i % 2] is not None:
                stream.wait_event(done_down[i % 2])  # step i-2's outputs are back on the host
            vkv.chunk_attn_segments(qq, kk, vv, case.branches, scale=case.scale, err=err, out=oo, stream=stream)
            cd = torch.cuda.Event()
            cd.record(stream)
            done_comp[i % 2] = cd
            s_down.wait_event(cd)
            with torch.cuda.stream(s_down):
                for h, d_ in zip(hout, outs(oo)):
                    h.copy_(d_, non_blocking=True)
            dd = torch.cuda.Event()
            dd.record(s_down)
            done_down[i % 2] = dd
        a1.record(s_down)
        return a0, a1

    e2e_steps = max(3, min(args.steps, 10))
    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    a0, a1 = e2e_run(e2e_steps)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1) / e2e_steps,
                            dev if world > 1 and torch.distributed.get_backend() == "nccl" else "cpu")
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = sum(t.numel() * t.element_size() for t in hout)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")

    if rank != 0:
        barrier()
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": headline_config(world),
        "chunk": {"ms": ms_step, "pct_of_bf16_peak": 100.0 * value / world / peak},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": recorded_traffic(),
                     "peak_source": f"{peak_src} bf16 dense (burst)", "kernel": headline_kernel_name(vkv, q, k, v, case),
                     "launch_ms_median": statistics.median(launch_ms),
                     "launch_ms_p10": float(np.percentile(launch_ms, 10)),
                     "launch_ms_p90": float(np.percentile(launch_ms, 90)),
                     # the timed steps run back to back for about a second under the power cap,
                     # the regime of the sustained GEMM figure; reported beside the burst fraction
                     "peak_sustained": peak_sus, "frac_of_sustained": achieved / peak_sus if peak_sus else None},
        "e2e": {"value": world * fl / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipeline": "two buffer sets; upload, call and read-back of consecutive steps overlap"},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks,
    }
    line["roofline"]["launch_mcycles_median"] = mcycles(line["roofline"]["launch_ms_median"], clocks)
    line["chunk"]["mcycles"] = mcycles(ms_step, clocks)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case)
    if world == 1 and not args.no_extras:
        del q, k, v, out, q2, k2, v2, out2, sets
        torch.cuda.empty_cache()
        line["modes"] = extras(dev, peaks)
    barrier()
    print(json.dumps(line), flush=True)
    return 0


def run_split(args):
    """ONE headline chunk split over the ranks (strong scaling): by head or by key range."""
    from kv_cache_attention_chunk_b200 import build, shard, vkv
    rank, local, world = dist_setup()
    if local == 0:
        build.build()
    barrier()
    vkv.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    case = headline_case(0)  # the same chunk on every rank
    fl = headline_flops()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    nccl = world > 1 and torch.distributed.get_backend() == "nccl"
    if args.split == "heads":
        h0, h1 = shard.head_range(case.H, world, rank)
        host = [t[:, :, h0:h1].contiguous() for t in (case.q, case.k, case.v)]
        branches, merged = case.branches, True
        part = f"heads {h0}..{h1 - 1}"
    else:
        parts = shard.key_parts(case.branches, world)
        kr, vr, seg = shard.compact_part(case.k, case.v, parts[rank])
        host = [case.q, kr, vr]
        branches, merged = [seg], False
        part = f"keys {sum(n for _, n in parts[rank])} of {sum(n for br in case.branches for _, n in br)}"
    q, k, v = (t.to(dev) for t in host)
    out = vkv.chunk_attn_segments(q, k, v, branches, scale=case.scale, merged=merged, err=err)
    per_attn = 2 if headline_split(vkv, q, k, v, branches, case.scale) else 1

    def step(q, k, v):
        res = vkv.chunk_attn_segments(q, k, v, branches, scale=case.scale, merged=merged, err=err, out=out,
                                      stream=stream)
        if args.split == "heads":
            o, l = res["o_merged"], res["lse_merged"]
            if args.gather:
                o = shard.gather_heads(o, case.H, rank, world)
            return o, l
        return shard.merge_to_rank0(res["o"][0], res["lse"][0], rank, world)

    launches_per_step = per_attn + ((world - 1) if (args.split == "keys" and rank == 0) else 0)
    for _ in range(args.warmup):
        step(q, k, v)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    sampler = ClockSampler(vis.split(",")[local].strip() if vis else local)
    if rank == 0:
        sampler.start()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step(q, k, v)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if rank == 0 else None
    ms_step = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev if nccl else "cpu")
    # end to end: this rank's inputs uploaded from pinned host memory every step, and the
    # result (rank 0's merged output, or each rank's own heads) read back
    hp = [t.pin_memory() for t in host]
    o_ref, l_ref = step(q, k, v)
    h_out = [o_ref.cpu().pin_memory(), l_ref.cpu().pin_memory()] if (rank == 0 or args.split == "heads") else []

    def e2e_step():
        for d_, h_ in zip((q, k, v), hp):
            d_.copy_(h_, non_blocking=True)
        o, l = step(q, k, v)
        if h_out:
            h_out[0].copy_(o, non_blocking=True)
            h_out[1].copy_(l, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    e2e_step()
    torch.cuda.synchronize()
    barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1) / e2e_steps, dev if nccl else "cpu")
    h2d = sum(t.numel() * t.element_size() for t in hp)
    d2h = sum(t.numel() * t.element_size() for t in h_out)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    if rank != 0:
        barrier()
        return 0
    value = fl / (ms_step * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "parallelism": f"{args.split} split of one chunk over {world} GPUs"
                   + (" + all-gather of the merged output" if args.gather and args.split == "heads" else "")
                   + (" + send/recv of partials to rank 0 and LSE merges" if args.split == "keys" else ""),
                   "rank0_part": part, "l2": "no flush: the inputs are larger than L2",
                   "flops_per_chunk": fl},
        "chunk": {"ms": ms_step, "mcycles": mcycles(ms_step, clocks), "pct_of_bf16_peak": 100.0 * value / world / peak},
        "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak, "unit": "TFLOP/s",
                     "frac": value / world / peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16 dense (burst), per GPU"},
        "e2e": {"value": fl / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "pipeline": "none (rank 0's bytes)"},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks,
    }
    barrier()
    print(json.dumps(line), flush=True)
    return 0


def run_profile(args):
    """Small fixed cases for ncu captures: warmup + steps launches of one kernel, no JSON contract."""
    from kv_cache_attention_chunk_b200 import build, vkv
    build.build()
    dev = torch.device("cuda", 0)
    st = torch.cuda.current_stream()
    if args.profile in ("wan13b", "wan14b"):
        c = W.cfg_wan13b() if args.profile == "wan13b" else headline_case(0)
        q, k, v = c.q.to(dev), c.k.to(dev), c.v.to(dev)
        out = vkv.chunk_attn_segments(q, k, v, c.branches, scale=c.scale)
        fn = lambda: vkv.chunk_attn_segments(q, k, v, c.branches, scale=c.scale, out=out)  # noqa: E731
    elif args.profile == "merge":
        oa, la, ob, lb = (t.to(dev) for t in W.make_merge_inputs(5, 1, 4680, 40, 128))
        o = vkv.lse_merge(oa, la, ob, lb)
        fn = lambda: vkv.lse_merge(oa, la, ob, lb, out=o)  # noqa: E731
    elif args.profile in ("select", "sparse9", "sparse144", "sparse9fs"):
        c = W.cfg_sparse()
        q, k, v = c.q.to(dev), c.k.to(dev), c.v.to(dev)
        K = 9 if args.profile != "sparse144" else 144
        idx, _, order = vkv.block_select(q, k, c.window_blk0, c.n_win_blk, K, order=True)
        if args.profile == "sparse9fs":
            # the selection inside the attention kernel, from cached window block means
            pers = torch.from_numpy(c.persist_idx).to(dev)
            kbar = vkv.block_pool(k, c.window_blk0, c.n_win_blk)
            o = vkv.chunk_attn_block_sparse(q, k, v, pers, None, c.window_blk0, c.n_win_blk, scale=c.scale,
                                            qblk_order=order, kbar=kbar, topk=K, sel_out=idx)
            fn = lambda: vkv.chunk_attn_block_sparse(q, k, v, pers, None, c.window_blk0,  # noqa: E731
                                                     c.n_win_blk, scale=c.scale, out=o, qblk_order=order,
                                                     kbar=kbar, topk=K, sel_out=idx)
        elif args.profile == "select":
            fn = lambda: vkv.block_select(q, k, c.window_blk0, c.n_win_blk, K, out_idx=idx,  # noqa: E731
                                          out_order=order)
        else:
            pers = torch.from_numpy(c.persist_idx).to(dev)
            o = vkv.chunk_attn_block_sparse(q, k, v, pers, idx, c.window_blk0, c.n_win_blk, scale=c.scale,
                                            qblk_order=order)
            fn = lambda: vkv.chunk_attn_block_sparse(q, k, v, pers, idx, c.window_blk0, c.n_win_blk,  # noqa: E731
                                                     scale=c.scale, out=o, qblk_order=order)
    elif args.profile == "ragged":
        c = W.cfg_ragged()
        q, k, v = c.q.to(dev), c.k.to(dev), c.v.to(dev)
        cu = torch.from_numpy(c.cu_seqlens).to(dev)
        o = vkv.chunk_attn_ragged(q, k, v, cu, c.cu_seqlens, scale=c.scale)
        fn = lambda: vkv.chunk_attn_ragged(q, k, v, cu, c.cu_seqlens, scale=c.scale, out=o)  # noqa: E731
    elif args.profile == "compaction":
        ft, hist, cur, recent = 1560, 60, 3, 2
        rules = [(vkv.HEAD_ANCHOR, 8)] * 4 + [(vkv.HEAD_WAVE, p) for p in (2, 3, 4, 5)] + [(vkv.HEAD_VEIL, 8)] * 4
        g = torch.Generator(device=dev).manual_seed(12)
        kd = torch.randn((1, (hist + cur) * ft, 12, 128), generator=g, device=dev).to(torch.bfloat16)
        vd = torch.randn((1, (hist + cur) * ft, 12, 128), generator=g, device=dev).to(torch.bfloat16)
        fn = lambda: vkv.compact_cache(kd, vd, rules, ft, hist, cur, recent)  # noqa: E731
    elif args.profile == "persist":
        c = W.cfg_sparse()
        q, k = c.q.to(dev), c.k.to(dev)
        pers = torch.from_numpy(c.persist_idx).to(dev)
        pidx, _ = vkv.persist_update(q, k, pers, c.window_blk0, 24)
        fn = lambda: vkv.persist_update(q, k, pers, c.window_blk0, 24, out_idx=pidx)  # noqa: E731
    elif args.profile == "latent":
        c = W.cfg_latent()
        q, kv = c.q.to(dev), c.kv.to(dev)
        o = vkv.latent_attn(q, kv, c.d_c, scale=c.scale)
        fn = lambda: vkv.latent_attn(q, kv, c.d_c, scale=c.scale, out=o)  # noqa: E731
    else:
        raise SystemExit(f"unknown profile case {args.profile}")
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    ts = timed(fn, args.steps, st)
    print(json.dumps({"profile": args.profile, "ms": ts}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile", default=None,
                    help="run one small case for an ncu capture: wan13b, wan14b, merge, select, sparse9, "
                         "sparse9fs, sparse144, ragged, latent, compaction, persist")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip the per-mode timings")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", choices=["none", "heads", "keys"], default="none",
                    help="split ONE chunk over the ranks (strong scaling) instead of a chunk per rank")
    ap.add_argument("--gather", action="store_true", help="--split heads: all-gather the merged output")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return run_profile(args)
    try:
        return run_split(args) if args.split != "none" else run_ours(args)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
