"""ctypes binding of libvkv (include/vkv.h): argument marshalling only.

Every computation runs in the library's sm_100a kernels; this module turns
torch tensors into the C structs, passes the current CUDA stream and raises
on a non-OK status.  There is no fallback: if libvkv.so is missing or no
sm_100 device is present the calls raise.

Raw entry points with the C names: ``vkv_chunk_attn``, ``vkv_block_select``,
``vkv_block_select_workspace_size``, ``vkv_lse_merge``, ``vkv_latent_attn``,
``vkv_status_string`` (and the other entry points of the header).
Convenience wrappers that allocate outputs with torch: ``chunk_attn_segments``,
``chunk_attn_block_sparse``, ``chunk_attn_ragged``, ``block_select``, ``lse_merge``,
``latent_attn`` and the others below.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
from ctypes import POINTER, c_float, c_int32, c_int64, c_size_t, c_void_p

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvkv.so")
LIB_TEST_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvkv_test.so")

MODE_SEGMENTS, MODE_BLOCK_SPARSE, MODE_RAGGED = 0, 1, 2
MAX_BRANCHES, MAX_SEGMENTS = 2, 8
DEVERR_TIMEOUT, DEVERR_BAD_INDEX, DEVERR_BAD_OFFSETS = 1, 2, 3
NOALLOC_SCRATCH_BYTES = 4 * 1024 * 1024  # VKV_NOALLOC_SCRATCH_BYTES in include/vkv.h
STATUS = {0: "VKV_OK", 1: "VKV_ERR_NULL", 2: "VKV_ERR_SHAPE", 3: "VKV_ERR_ALIGN", 4: "VKV_ERR_RANGE",
          5: "VKV_ERR_UNSUPPORTED", 6: "VKV_ERR_CUDA", 7: "VKV_ERR_WORKSPACE"}


class VkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({vkv_status_string(status)})")


class vkv_segment(ctypes.Structure):
    _fields_ = [("start", c_int32), ("len", c_int32)]


class vkv_tensor(ctypes.Structure):
    _fields_ = [("ptr", c_void_p), ("sb", c_int64), ("st", c_int64), ("sh", c_int64)]


class vkv_attn_args(ctypes.Structure):
    _fields_ = [
        ("mode", c_int32), ("B", c_int32), ("H", c_int32), ("Lq", c_int32), ("Lkv", c_int32),
        ("d", c_int32), ("scale", c_float),
        ("q", vkv_tensor), ("k", vkv_tensor), ("v", vkv_tensor),
        ("n_branches", c_int32),
        ("segs", POINTER(vkv_segment) * MAX_BRANCHES),
        ("n_segs", c_int32 * MAX_BRANCHES),
        ("block", c_int32),
        ("persist_idx", c_void_p), ("n_persist", c_int32),
        ("sel_idx", c_void_p), ("topk", c_int32), ("window_blk0", c_int32), ("n_win_blk", c_int32),
        ("cu_seqlens", c_void_p), ("cu_seqlens_host", POINTER(c_int32)),
        ("o", vkv_tensor * MAX_BRANCHES), ("lse", c_void_p * MAX_BRANCHES),
        ("o_merged", vkv_tensor), ("lse_merged", c_void_p),
        ("err_word", c_void_p),
        ("qblk_order", c_void_p),
        ("workspace", c_void_p), ("workspace_bytes", c_size_t),
        ("kbar", c_void_p), ("sel_out", c_void_p),
    ]


class vkv_select_args(ctypes.Structure):
    _fields_ = [
        ("B", c_int32), ("H", c_int32), ("d", c_int32), ("block", c_int32),
        ("Lq", c_int32), ("Lkv", c_int32), ("window_blk0", c_int32), ("n_win_blk", c_int32),
        ("topk", c_int32),
        ("q", vkv_tensor), ("k", vkv_tensor),
        ("out_idx", c_void_p), ("out_scores", c_void_p),
        ("workspace", c_void_p), ("workspace_bytes", c_size_t),
        ("err_word", c_void_p),
        ("out_order", c_void_p),
        ("kbar", c_void_p),
    ]


class vkv_head_rule(ctypes.Structure):
    _fields_ = [("policy", c_int32), ("param", c_int32)]


class vkv_compact_args(ctypes.Structure):
    _fields_ = [
        ("B", c_int32), ("H", c_int32), ("d", c_int32), ("frame_tokens", c_int32),
        ("hist_frames", c_int32), ("cur_frames", c_int32), ("recent_frames", c_int32),
        ("k_src", vkv_tensor), ("v_src", vkv_tensor),
        ("rules", POINTER(vkv_head_rule)),
        ("k_out", c_void_p), ("v_out", c_void_p), ("out_rows", c_int64),
        ("cu_seqlens", c_void_p), ("cu_seqlens_host", POINTER(c_int32)),
    ]


HEAD_FULL, HEAD_ANCHOR, HEAD_WAVE, HEAD_VEIL = 0, 1, 2, 3


class vkv_persist_args(ctypes.Structure):
    _fields_ = [
        ("B", c_int32), ("H", c_int32), ("d", c_int32), ("block", c_int32),
        ("Lq", c_int32), ("Lkv", c_int32),
        ("q", vkv_tensor), ("k", vkv_tensor),
        ("persist_idx", c_void_p), ("n_persist", c_int32),
        ("evict_blk0", c_int32), ("n_evict", c_int32),
        ("out_idx", c_void_p), ("out_scores", c_void_p),
        ("workspace", c_void_p), ("workspace_bytes", c_size_t),
        ("err_word", c_void_p),
    ]

class vkv_latent_args(ctypes.Structure):
    _fields_ = [
        ("B", c_int32), ("H", c_int32), ("Lq", c_int32), ("Lkv", c_int32),
        ("d_c", c_int32), ("d_rope", c_int32), ("scale", c_float),
        ("q", vkv_tensor), ("kv", vkv_tensor), ("kr", vkv_tensor), ("o", vkv_tensor),
        ("lse", c_void_p), ("err_word", c_void_p),
    ]

class vkv_schedule(ctypes.Structure):
    _fields_ = [
        ("n_ctas", c_int32), ("n_units", c_int32), ("n_pieces", c_int32), ("n_slots", c_int32),
        ("cta_begin", POINTER(c_int32)), ("cta_piece0", POINTER(c_int32)),
        ("units", POINTER(ctypes.c_uint32)), ("pieces", POINTER(ctypes.c_uint32)),
    ]


_lib = None
_test_lib = None


def lib() -> ctypes.CDLL:
    """Load libvkv.so (built in-tree by kv_cache_attention_chunk_b200.build); raise if absent."""
    global _lib
    if _lib is None:
        _lib = _load(LIB_PATH)
    return _lib


def test_lib() -> ctypes.CDLL:
    """Load the test build libvkv_test.so: the same library plus the test aids of
    include/vkv_test.h (vkv_debug_withhold_copy)."""
    global _test_lib
    if _test_lib is None:
        L = _load(LIB_TEST_PATH)
        L.vkv_debug_withhold_copy.argtypes = [c_int32]
        L.vkv_debug_withhold_copy.restype = c_int32
        L.vkv_debug_exp2_poly.argtypes = [c_void_p, c_void_p, c_int32, c_void_p]
        L.vkv_debug_exp2_poly.restype = c_int32
        _test_lib = L
    return _test_lib


@contextlib.contextmanager
def using_test_library():
    """Route the calls of this module through the test build while the block runs."""
    global _lib
    saved = lib()
    _lib = test_lib()
    try:
        yield _lib
    finally:
        _lib = saved


def _load(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m kv_cache_attention_chunk_b200.build`"
                           " (there is no fallback implementation)")
    L = ctypes.CDLL(path)
    L.vkv_chunk_attn.argtypes = [POINTER(vkv_attn_args), c_void_p]
    L.vkv_chunk_attn.restype = c_int32
    L.vkv_chunk_attn_workspace_size.argtypes = [POINTER(vkv_attn_args)]
    L.vkv_chunk_attn_workspace_size.restype = c_size_t
    L.vkv_debug_schedule.argtypes = [POINTER(vkv_attn_args), c_int32, c_int32, POINTER(vkv_schedule)]
    L.vkv_debug_schedule.restype = c_int32
    L.vkv_block_select.argtypes = [POINTER(vkv_select_args), c_void_p]
    L.vkv_block_select.restype = c_int32
    L.vkv_block_select_noalloc.argtypes = [POINTER(vkv_select_args), c_void_p]
    L.vkv_block_select_noalloc.restype = c_int32
    L.vkv_block_select_workspace_size.argtypes = [c_int32] * 6
    L.vkv_block_select_workspace_size.restype = c_size_t
    L.vkv_block_order.argtypes = [c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p]
    L.vkv_block_order.restype = c_int32
    L.vkv_lse_merge.argtypes = [vkv_tensor, c_void_p, vkv_tensor, c_void_p, vkv_tensor, c_void_p,
                                c_int32, c_int32, c_int32, c_int32, c_void_p]
    L.vkv_lse_merge.restype = c_int32
    L.vkv_status_string.argtypes = [c_int32]
    L.vkv_status_string.restype = ctypes.c_char_p
    L.vkv_version.argtypes = []
    L.vkv_version.restype = c_int32
    L.vkv_abi_sizeof.argtypes = [c_int32]
    L.vkv_abi_sizeof.restype = c_int32
    L.vkv_block_pool.argtypes = [vkv_tensor, c_int32, c_int32, c_int32, c_int32, c_int32, c_int32, c_void_p,
                                 c_void_p]
    L.vkv_block_pool.restype = c_int32
    L.vkv_compact_rows.argtypes = [POINTER(vkv_compact_args)]
    L.vkv_compact_rows.restype = c_int64
    L.vkv_compact_cache.argtypes = [POINTER(vkv_compact_args), c_void_p]
    L.vkv_compact_cache.restype = c_int32
    L.vkv_persist_update_workspace_size.argtypes = [c_int32] * 7
    L.vkv_persist_update_workspace_size.restype = c_size_t
    L.vkv_persist_update.argtypes = [POINTER(vkv_persist_args), c_void_p]
    L.vkv_persist_update.restype = c_int32
    L.vkv_latent_attn.argtypes = [POINTER(vkv_latent_args), c_void_p]
    L.vkv_latent_attn.restype = c_int32
    for i, st in enumerate((vkv_attn_args, vkv_select_args, vkv_tensor, vkv_segment, vkv_compact_args,
                            vkv_head_rule, vkv_persist_args, vkv_latent_args, vkv_schedule)):
        if L.vkv_abi_sizeof(i) != ctypes.sizeof(st):
            raise RuntimeError(f"ABI mismatch for {st.__name__}: C {L.vkv_abi_sizeof(i)} B, "
                               f"binding {ctypes.sizeof(st)} B")
    return L


# ---------------------------------------------------------------------------
# raw entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def vkv_status_string(status: int) -> str:
    return lib().vkv_status_string(int(status)).decode()


def vkv_chunk_attn(args: vkv_attn_args, stream: int | None) -> int:
    return int(lib().vkv_chunk_attn(ctypes.byref(args), c_void_p(stream or 0)))


def vkv_chunk_attn_workspace_size(args: vkv_attn_args) -> int:
    return int(lib().vkv_chunk_attn_workspace_size(ctypes.byref(args)))


def vkv_debug_schedule(args: vkv_attn_args, n_sm: int, split: int, out: vkv_schedule) -> int:
    return int(lib().vkv_debug_schedule(ctypes.byref(args), int(n_sm), int(split), ctypes.byref(out)))


def attn_schedule(args: vkv_attn_args, n_sm: int, split: bool) -> dict:
    """The work schedule of vkv_chunk_attn for these arguments on `n_sm` SMs (host only):
    numpy arrays cta_begin, cta_piece0, units (uint32 codes), pieces ([n, 2] uint32) and n_slots."""
    cb = np.zeros(n_sm + 1, np.int32)
    cp = np.zeros(n_sm + 1, np.int32)
    un = np.zeros(6144, np.uint32)
    pc = np.zeros(2 * 384, np.uint32)
    out = vkv_schedule(0, 0, 0, 0, cb.ctypes.data_as(POINTER(c_int32)), cp.ctypes.data_as(POINTER(c_int32)),
                       un.ctypes.data_as(POINTER(ctypes.c_uint32)), pc.ctypes.data_as(POINTER(ctypes.c_uint32)))
    _check(vkv_debug_schedule(args, n_sm, 1 if split else 0, out), "vkv_debug_schedule")
    g = out.n_ctas
    return {"cta_begin": cb[:g + 1].copy(), "cta_piece0": cp[:g + 1].copy(), "units": un[:out.n_units].copy(),
            "pieces": pc[:2 * out.n_pieces].reshape(-1, 2).copy(), "n_slots": out.n_slots}


def vkv_block_select(args: vkv_select_args, stream: int | None) -> int:
    return int(lib().vkv_block_select(ctypes.byref(args), c_void_p(stream or 0)))


def vkv_block_select_noalloc(args: vkv_select_args, stream: int | None) -> int:
    """vkv_block_select with the library's own fixed scratch array (no workspace argument)."""
    return int(lib().vkv_block_select_noalloc(ctypes.byref(args), c_void_p(stream or 0)))


def vkv_block_order(sel_idx, out_order, BH, n_qblk, topk, stream: int | None) -> int:
    return int(lib().vkv_block_order(c_void_p(sel_idx), c_void_p(out_order), int(BH), int(n_qblk), int(topk),
                                     c_void_p(stream or 0)))


def block_order(sel_idx, out=None, stream=None):
    """Query-block order [B*H, nQblk] grouping similar selections, from a selection
    sel_idx (device int32 [B*H, nQblk, topk], e.g. the sel_out of chunk_attn_block_sparse
    with kbar), for a later call's qblk_order."""
    sel_idx = sel_idx.contiguous()
    BH, n_qblk, topk = sel_idx.shape
    order = out if out is not None else torch.empty((BH, n_qblk), dtype=torch.int32, device=sel_idx.device)
    _check(vkv_block_order(sel_idx.data_ptr(), order.data_ptr(), BH, n_qblk, topk, _stream(stream)),
           "vkv_block_order")
    return order


def vkv_block_pool(x: vkv_tensor, B, L, H, d, blk0, n_blk, out, stream: int | None) -> int:
    return int(lib().vkv_block_pool(x, B, L, H, d, blk0, n_blk, c_void_p(out), c_void_p(stream or 0)))


def vkv_persist_update_workspace_size(B, H, Lq, n_persist, n_evict, block, d) -> int:
    return int(lib().vkv_persist_update_workspace_size(B, H, Lq, n_persist, n_evict, block, d))


def vkv_persist_update(args: vkv_persist_args, stream: int | None) -> int:
    return int(lib().vkv_persist_update(ctypes.byref(args), c_void_p(stream or 0)))


def vkv_latent_attn(args: vkv_latent_args, stream: int | None) -> int:
    return int(lib().vkv_latent_attn(ctypes.byref(args), c_void_p(stream or 0)))


def vkv_debug_withhold_copy(n_calls: int) -> int:
    """Test aid of the test build (include/vkv_test.h): the next n_calls attention
    launches of libvkv_test.so withhold their first cache-tile copy."""
    return int(test_lib().vkv_debug_withhold_copy(int(n_calls)))


def vkv_compact_rows(args: vkv_compact_args) -> int:
    return int(lib().vkv_compact_rows(ctypes.byref(args)))


def vkv_compact_cache(args: vkv_compact_args, stream: int | None) -> int:
    return int(lib().vkv_compact_cache(ctypes.byref(args), c_void_p(stream or 0)))


def vkv_block_select_workspace_size(B, H, Lq, n_win_blk, block, d) -> int:
    return int(lib().vkv_block_select_workspace_size(B, H, Lq, n_win_blk, block, d))


def vkv_lse_merge(o_a: vkv_tensor, lse_a, o_b: vkv_tensor, lse_b, o_out: vkv_tensor, lse_out,
                  B, H, Lq, d, stream: int | None) -> int:
    return int(lib().vkv_lse_merge(o_a, c_void_p(lse_a), o_b, c_void_p(lse_b), o_out, c_void_p(lse_out),
                                   B, H, Lq, d, c_void_p(stream or 0)))


# ---------------------------------------------------------------------------
# torch helpers
# ---------------------------------------------------------------------------
def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def tensor_desc(x: torch.Tensor) -> vkv_tensor:
    """[B, L, H, d] bf16 with a contiguous last axis -> vkv_tensor."""
    if x.dim() != 4 or x.dtype != torch.bfloat16 or x.stride(3) != 1:
        raise ValueError("expected a bf16 [B, L, H, d] tensor with contiguous d")
    return vkv_tensor(x.data_ptr(), x.stride(0), x.stride(1), x.stride(2))


def flat_desc(x: torch.Tensor) -> vkv_tensor:
    """[rows, d] bf16 with contiguous d -> vkv_tensor (row stride in st)."""
    if x.dim() != 2 or x.dtype != torch.bfloat16 or x.stride(1) != 1:
        raise ValueError("expected a bf16 [rows, d] tensor with contiguous d")
    return vkv_tensor(x.data_ptr(), 0, x.stride(0), 0)


def _check(status: int, what: str):
    if status != 0:
        raise VkvError(status, what)


def _base_args(mode, q, Lkv, d, scale, k_desc, v_desc, err):
    B, Lq, H, dq = q.shape
    if dq != d:
        raise ValueError("head dimension mismatch")
    a = vkv_attn_args()
    a.mode = mode
    a.B, a.H, a.Lq, a.Lkv, a.d = B, H, Lq, Lkv, d
    a.scale = float(scale if scale is not None else 1.0 / np.sqrt(d))
    a.q = tensor_desc(q)
    a.k = k_desc
    a.v = v_desc
    a.block = 64
    a.err_word = err.data_ptr() if err is not None else None
    return a


_attn_ws: dict = {}  # (device index, stream handle) -> uint8 device buffer, grown on demand


def _attn_workspace(a: vkv_attn_args, q: torch.Tensor, stream_handle: int, split: bool, workspace):
    """Point the call at a key-axis split workspace: the caller's, or one kept per
    (device, stream) by this module; none when split is False or the schedule
    splits nothing.  Returns the buffer (kept alive by the caller until launch)."""
    if workspace is not None:
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel() * workspace.element_size()
        return workspace
    if not split:
        return None
    need = vkv_chunk_attn_workspace_size(a)
    if need == 0:
        return None
    key = (q.device.index, stream_handle)
    buf = _attn_ws.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.empty(need, dtype=torch.uint8, device=q.device)
        _attn_ws[key] = buf
    a.workspace = buf.data_ptr()
    a.workspace_bytes = buf.numel()
    return buf


def _new_out(q):
    B, Lq, H, d = q.shape
    return (torch.empty((B, Lq, H, d), dtype=torch.bfloat16, device=q.device),
            torch.empty((B, H, Lq), dtype=torch.float32, device=q.device))


def segments_args(q, k, v, branches, scale=None, err=None) -> vkv_attn_args:
    """vkv_attn_args of a SEGMENTS call, inputs filled in, outputs left empty (the
    segment arrays are kept alive by the returned struct)."""
    d = q.shape[3]
    a = _base_args(MODE_SEGMENTS, q, k.shape[1], d, scale, tensor_desc(k), tensor_desc(v), err)
    a.n_branches = len(branches)
    keep = []
    for i, br in enumerate(branches):
        arr = (vkv_segment * max(1, len(br)))(*[vkv_segment(int(s), int(n)) for s, n in br])
        keep.append(arr)
        a.segs[i] = ctypes.cast(arr, POINTER(vkv_segment))
        a.n_segs[i] = len(br)
    a._keep_segs = keep
    return a


def chunk_attn_segments(q, k, v, branches, scale=None, merged=True, err=None, stream=None, out=None,
                        split=True, workspace=None):
    """Dual-branch (or single-branch) chunk attention over token segments.

    branches: list (length 1 or 2) of lists of (start, len) cache-row segments.
    split: let the schedule cut units along the key axis (a workspace kept by this
    module; `workspace`, a device uint8 tensor, overrides it).
    Returns dict(o=[...], lse=[...], o_merged, lse_merged).
    """
    nb = len(branches)
    a = segments_args(q, k, v, branches, scale, err)
    res = out if out is not None else {}
    if out is None:
        res["o"], res["lse"] = [], []
        for _ in range(nb):
            o, l = _new_out(q)
            res["o"].append(o)
            res["lse"].append(l)
        res["o_merged"], res["lse_merged"] = _new_out(q) if (merged and nb == 2) else (None, None)
    for i in range(nb):
        a.o[i] = tensor_desc(res["o"][i])
        a.lse[i] = res["lse"][i].data_ptr()
    if res.get("o_merged") is not None:
        a.o_merged = tensor_desc(res["o_merged"])
        a.lse_merged = res["lse_merged"].data_ptr()
    sh = _stream(stream)
    ws = _attn_workspace(a, q, sh, split, workspace)  # noqa: F841 (alive until the launch)
    _check(vkv_chunk_attn(a, sh), "vkv_chunk_attn")
    return res


def chunk_attn_block_sparse(q, k, v, persist_idx, sel_idx, window_blk0, n_win_blk, scale=None,
                            err=None, stream=None, out=None, qblk_order=None, split=True, workspace=None,
                            kbar=None, topk=None, sel_out=None):
    """Persistent blocks + selected window blocks (device int32 index tensors).

    qblk_order (optional device int32 [B*H, nQblk]): query-block permutation that
    groups blocks with similar selections into the same units (from block_select).
    split / workspace: key-axis pieces, as in chunk_attn_segments.

    kbar (optional device fp32 [B*H, n_win_blk, d], from block_pool): the kernel
    selects the top-`topk` window blocks itself (sel_idx may then be None); the
    selection is written to sel_out (device int32 [B*H, nQblk, topk]) when given.
    """
    d = q.shape[3]
    a = _base_args(MODE_BLOCK_SPARSE, q, k.shape[1], d, scale, tensor_desc(k), tensor_desc(v), err)
    persist_idx = persist_idx.contiguous()
    a.persist_idx = persist_idx.data_ptr() if persist_idx.numel() else None
    a.n_persist = persist_idx.shape[-1]
    if kbar is not None:
        if topk is None:
            topk = sel_out.shape[-1] if sel_out is not None else sel_idx.shape[-1]
        if not (kbar.dtype == torch.float32 and kbar.is_contiguous()):
            raise ValueError("kbar must be a contiguous float32 tensor [B*H, n_win_blk, d]")
        a.kbar = kbar.data_ptr()
        if sel_out is not None:
            if not (sel_out.dtype == torch.int32 and sel_out.is_contiguous()):
                raise ValueError("sel_out must be a contiguous int32 tensor [B*H, nQblk, topk]")
            a.sel_out = sel_out.data_ptr()
        a.topk = int(topk)
    else:
        sel_idx = sel_idx.contiguous()
        a.sel_idx = sel_idx.data_ptr() if sel_idx.numel() else None
        a.topk = sel_idx.shape[-1]
    a.window_blk0 = int(window_blk0)
    a.n_win_blk = int(n_win_blk)
    if qblk_order is not None:
        qblk_order = qblk_order.contiguous()
        a.qblk_order = qblk_order.data_ptr()
    o, l = out if out is not None else _new_out(q)
    a.o[0] = tensor_desc(o)
    a.lse[0] = l.data_ptr()
    sh = _stream(stream)
    ws = _attn_workspace(a, q, sh, split, workspace)  # noqa: F841 (alive until the launch)
    _check(vkv_chunk_attn(a, sh), "vkv_chunk_attn")
    return o, l


def chunk_attn_ragged(q, k_flat, v_flat, cu_seqlens, cu_seqlens_host=None, scale=None, err=None,
                      stream=None, out=None, split=True, workspace=None):
    """Ragged per-(batch, head) caches stored flattened with boundary offsets.

    With cu_seqlens_host the schedule knows each sequence's length and may cut
    long sequences' units along the key axis (split / workspace as in
    chunk_attn_segments)."""
    d = q.shape[3]
    a = _base_args(MODE_RAGGED, q, k_flat.shape[0], d, scale, flat_desc(k_flat), flat_desc(v_flat), err)
    a.cu_seqlens = cu_seqlens.data_ptr()
    host = None
    if cu_seqlens_host is not None:
        host = np.ascontiguousarray(np.asarray(cu_seqlens_host, dtype=np.int32))
        a.cu_seqlens_host = host.ctypes.data_as(POINTER(c_int32))
    o, l = out if out is not None else _new_out(q)
    a.o[0] = tensor_desc(o)
    a.lse[0] = l.data_ptr()
    sh = _stream(stream)
    ws = _attn_workspace(a, q, sh, split, workspace)  # noqa: F841 (alive until the launch)
    _check(vkv_chunk_attn(a, sh), "vkv_chunk_attn")
    return o, l


def block_select(q, k, window_blk0, n_win_blk, topk, workspace=None, scores=False, err=None, stream=None,
                 out_idx=None, order=False, out_order=None, kbar=None):
    """Top-K window blocks per 64-query block; returns (idx [B*H, nQblk, topk], scores or None).

    With order=True (or an out_order tensor) also returns the query-block order
    [B*H, nQblk] that groups blocks with similar selections: (idx, scores, order).
    kbar (optional device fp32 [B*H, n_win_blk, d], from block_pool) supplies the
    window blocks' representatives, so only the query blocks are pooled.
    """
    B, Lq, H, d = q.shape
    n_qblk = -(-Lq // 64)
    a = vkv_select_args()
    a.B, a.H, a.d, a.block = B, H, d, 64
    a.Lq, a.Lkv = Lq, k.shape[1]
    a.window_blk0, a.n_win_blk, a.topk = int(window_blk0), int(n_win_blk), int(topk)
    a.q = tensor_desc(q)
    a.k = tensor_desc(k)
    idx = out_idx if out_idx is not None else torch.empty((B * H, n_qblk, topk), dtype=torch.int32,
                                                          device=q.device)
    a.out_idx = idx.data_ptr()
    sc = None
    if scores:
        sc = torch.empty((B * H, n_qblk, n_win_blk), dtype=torch.float32, device=q.device)
        a.out_scores = sc.data_ptr()
    need = vkv_block_select_workspace_size(B, H, Lq, n_win_blk, 64, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    a.workspace = workspace.data_ptr()
    a.workspace_bytes = workspace.numel() * workspace.element_size()
    a.err_word = err.data_ptr() if err is not None else None
    if kbar is not None:
        kbar = kbar.contiguous()
        a.kbar = kbar.data_ptr()
    if order and out_order is None:
        out_order = torch.empty((B * H, n_qblk), dtype=torch.int32, device=q.device)
    if out_order is not None:
        a.out_order = out_order.data_ptr()
    _check(vkv_block_select(a, _stream(stream)), "vkv_block_select")
    if out_order is not None:
        return idx, sc, out_order
    return idx, sc


def block_pool(x, blk0, n_blk, stream=None, out=None):
    """fp32 mean of each 64-row block [blk0, blk0 + n_blk) of x [B, L, H, d] -> [B*H, n_blk, d]."""
    B, L, H, d = x.shape
    o = out if out is not None else torch.empty((B * H, n_blk, d), dtype=torch.float32, device=x.device)
    _check(vkv_block_pool(tensor_desc(x), B, L, H, d, int(blk0), int(n_blk), o.data_ptr(), _stream(stream)),
           "vkv_block_pool")
    return o


def lse_merge(o_a, lse_a, o_b, lse_b, stream=None, out=None):
    B, Lq, H, d = o_a.shape
    o, l = out if out is not None else _new_out(o_a)
    _check(vkv_lse_merge(tensor_desc(o_a), lse_a.data_ptr(), tensor_desc(o_b), lse_b.data_ptr(),
                         tensor_desc(o), l.data_ptr(), B, H, Lq, d, _stream(stream)), "vkv_lse_merge")
    return o, l


def compact_cache(k, v, rules, frame_tokens, hist_frames, cur_frames, recent_frames, stream=None):
    """Head-aware compaction of a dense cache into a flattened ragged cache.

    k, v: device bf16 [B, L, H, d] with L = (hist_frames + cur_frames) * frame_tokens;
    rules: one (policy, param) per head (HEAD_FULL / HEAD_ANCHOR / HEAD_WAVE / HEAD_VEIL).
    Returns (k_flat [rows, d], v_flat, cu_seqlens on the device, cu_seqlens on the host).
    """
    B, L, H, d = k.shape
    a = vkv_compact_args()
    a.B, a.H, a.d = B, H, d
    a.frame_tokens, a.hist_frames, a.cur_frames, a.recent_frames = (int(frame_tokens), int(hist_frames),
                                                                     int(cur_frames), int(recent_frames))
    a.k_src = tensor_desc(k)
    a.v_src = tensor_desc(v)
    rr = (vkv_head_rule * H)(*[vkv_head_rule(int(p), int(x)) for p, x in rules])
    a.rules = ctypes.cast(rr, POINTER(vkv_head_rule))
    rows = vkv_compact_rows(a)
    if rows < 0:
        raise VkvError(-rows, "vkv_compact_rows")
    k_out = torch.empty((rows, d), dtype=k.dtype, device=k.device)
    v_out = torch.empty((rows, d), dtype=v.dtype, device=v.device)
    cu_dev = torch.empty(B * H + 1, dtype=torch.int32, device=k.device)
    cu_host = np.zeros(B * H + 1, dtype=np.int32)
    a.k_out, a.v_out, a.out_rows = k_out.data_ptr(), v_out.data_ptr(), rows
    a.cu_seqlens = cu_dev.data_ptr()
    a.cu_seqlens_host = cu_host.ctypes.data_as(POINTER(c_int32))
    _check(vkv_compact_cache(a, _stream(stream)), "vkv_compact_cache")
    return k_out, v_out, cu_dev, cu_host


def persist_update(q, k, persist_idx, evict_blk0, n_evict, scores=False, err=None, stream=None, out_idx=None,
                   workspace=None):
    """Top-C of (persistent blocks + evicted window blocks) by <mean query, block mean>.

    q [B, Lq, H, d], k [B, Lkv, H, d] device bf16; persist_idx device int32 [B*H, C].
    Returns (new persistent ids [B*H, C] ascending, candidate scores [B*H, C + n_evict] or None).
    """
    B, Lq, H, d = q.shape
    persist_idx = persist_idx.contiguous()
    C = persist_idx.shape[-1]
    a = vkv_persist_args()
    a.B, a.H, a.d, a.block, a.Lq, a.Lkv = B, H, d, 64, Lq, k.shape[1]
    a.q, a.k = tensor_desc(q), tensor_desc(k)
    a.persist_idx, a.n_persist = persist_idx.data_ptr(), C
    a.evict_blk0, a.n_evict = int(evict_blk0), int(n_evict)
    idx = out_idx if out_idx is not None else torch.empty((B * H, C), dtype=torch.int32, device=q.device)
    a.out_idx = idx.data_ptr()
    sc = None
    if scores:
        sc = torch.empty((B * H, C + int(n_evict)), dtype=torch.float32, device=q.device)
        a.out_scores = sc.data_ptr()
    need = vkv_persist_update_workspace_size(B, H, Lq, C, int(n_evict), 64, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel()
    a.err_word = err.data_ptr() if err is not None else None
    _check(vkv_persist_update(a, _stream(stream)), "vkv_persist_update")
    return idx, sc


def latent_desc(x: torch.Tensor) -> vkv_tensor:
    """[B, L, w] bf16 cache rows with contiguous w -> vkv_tensor (sh unused)."""
    if x.dim() != 3 or x.dtype != torch.bfloat16 or x.stride(2) != 1:
        raise ValueError("expected a bf16 [B, L, w] tensor with contiguous w")
    return vkv_tensor(x.data_ptr(), x.stride(0), x.stride(1), 0)


def latent_attn(q, kv, d_c, scale=None, kr=None, err=None, stream=None, out=None, lse=True):
    """Latent attention over a head-shared cache (vkv_latent_attn).

    q [B, Lq, H, d_c + d_rope] absorbed queries; kv [B, Lkv, d_c (+ d_rope)] cached rows
    [c ; k_R]; kr optional [B, Lkv, d_rope] when the rotary keys are stored apart.
    Returns (latent output [B, Lq, H, d_c] bf16, LSE [B, H, Lq] fp32 or None).
    """
    B, Lq, H, dq = q.shape
    d_rope = dq - d_c
    a = vkv_latent_args()
    a.B, a.H, a.Lq, a.Lkv, a.d_c, a.d_rope = B, H, Lq, kv.shape[1], d_c, d_rope
    a.scale = float(scale if scale is not None else 1.0 / np.sqrt(dq))
    a.q = tensor_desc(q)
    if kv.shape[1] > 0:  # an empty cache is passed as a NULL pointer
        a.kv = latent_desc(kv)
        if kr is not None:
            a.kr = latent_desc(kr)
    if out is None:
        o = torch.empty((B, Lq, H, d_c), dtype=torch.bfloat16, device=q.device)
        l = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device) if lse else None
    else:
        o, l = out
    a.o = tensor_desc(o)
    a.lse = l.data_ptr() if l is not None else None
    a.err_word = err.data_ptr() if err is not None else None
    _check(vkv_latent_attn(a, _stream(stream)), "vkv_latent_attn")
    return o, l
