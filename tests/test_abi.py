"""The C-ABI library: loads without a GPU, exports what include/vkv.h declares,
struct layouts match the binding, and host-side validation rejects bad
arguments with the documented status before any device work.

No call here reaches a kernel: every request is invalid on purpose (the
library checks arguments before it looks for a device), or, for a valid
request on a machine without a GPU, it must return VKV_ERR_CUDA.
"""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from kv_cache_attention_chunk_b200 import build, vkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()
    vkv.lib()


def declared_functions(header="vkv.h"):
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(vkv_\w+)\s*\(", src)))


def test_exports_every_declared_function():
    names = declared_functions()
    assert {"vkv_chunk_attn", "vkv_block_select", "vkv_lse_merge"} <= set(names)
    L = vkv.lib()
    for n in names:
        assert hasattr(L, n), f"{n} declared in vkv.h but not exported"


def test_test_aids_only_in_the_test_build():
    """include/vkv_test.h is exported by libvkv_test.so (which also exports all of
    vkv.h) and by no means by the production libvkv.so."""
    aids = declared_functions("vkv_test.h")
    assert aids == ["vkv_debug_exp2_poly", "vkv_debug_withhold_copy"]
    T_ = vkv.test_lib()
    for n in aids + declared_functions():
        assert hasattr(T_, n), f"{n} not exported by the test build"
    prod = ctypes.CDLL(vkv.LIB_PATH)
    for n in aids:
        assert not hasattr(prod, n), f"{n} is a test aid but the production library exports it"
    headers = sorted(f for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h"))
    assert headers == ["vkv.h", "vkv_test.h"]


def test_struct_layouts_match_binding():
    L = vkv.lib()
    for i, st in enumerate((vkv.vkv_attn_args, vkv.vkv_select_args, vkv.vkv_tensor, vkv.vkv_segment)):
        assert L.vkv_abi_sizeof(i) == ctypes.sizeof(st)
    assert L.vkv_abi_sizeof(99) == -1


def test_status_strings_and_version():
    for s in range(8):
        assert len(vkv.vkv_status_string(s)) >= 2
    assert vkv.lib().vkv_version() >= 100


def T(ptr=FAKE, sb=0, st=1024, sh=128):
    return vkv.vkv_tensor(ptr, sb, st, sh)


def seg_args(**kw):
    a = vkv.vkv_attn_args()
    a.mode = vkv.MODE_SEGMENTS
    a.B, a.H, a.Lq, a.Lkv, a.d = 1, 8, 256, 1024, 128
    a.scale = 0.088
    a.q = T(sb=256 * 1024)
    a.k = T(sb=1024 * 1024)
    a.v = T(sb=1024 * 1024)
    a.n_branches = 2
    segs0 = (vkv.vkv_segment * 2)(vkv.vkv_segment(0, 128), vkv.vkv_segment(768, 256))
    segs1 = (vkv.vkv_segment * 1)(vkv.vkv_segment(128, 640))
    a._keep = (segs0, segs1)
    a.segs[0] = ctypes.cast(segs0, ctypes.POINTER(vkv.vkv_segment))
    a.segs[1] = ctypes.cast(segs1, ctypes.POINTER(vkv.vkv_segment))
    a.n_segs[0], a.n_segs[1] = 2, 1
    for i in range(2):
        a.o[i] = T(sb=256 * 1024)
        a.lse[i] = FAKE
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def call(a):
    return vkv.vkv_chunk_attn(a, None)


def test_valid_request_without_gpu_reports_cuda_error():
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert call(seg_args()) == 6  # VKV_ERR_CUDA


@pytest.mark.parametrize("field,value,status", [
    ("d", 96, 5), ("d", 256, 5), ("mode", 7, 5),
    ("B", 0, 2), ("H", -1, 2), ("Lq", 0, 2), ("scale", 0.0, 2), ("scale", float("nan"), 2),
    ("n_branches", 3, 2), ("n_branches", 0, 2),
])
def test_bad_sizes(field, value, status):
    assert call(seg_args(**{field: value})) == status


def test_null_and_alignment():
    assert vkv.lib().vkv_chunk_attn(None, None) == 1
    assert call(seg_args(q=T(ptr=0))) == 1
    assert call(seg_args(q=T(ptr=FAKE + 2, sb=256 * 1024))) == 3
    assert call(seg_args(k=T(st=1028, sb=1024 * 1024))) == 3  # stride not a multiple of 8
    a = seg_args()
    a.lse[1] = None
    assert call(a) == 1
    a = seg_args()
    a.o[0] = T(ptr=FAKE + 8, sb=256 * 1024)
    assert call(a) == 3


def test_segments_out_of_range():
    a = seg_args()
    bad = (vkv.vkv_segment * 1)(vkv.vkv_segment(1000, 100))  # runs past Lkv = 1024
    a._bad = bad
    a.segs[1] = ctypes.cast(bad, ctypes.POINTER(vkv.vkv_segment))
    assert call(a) == 4
    bad2 = (vkv.vkv_segment * 1)(vkv.vkv_segment(-1, 10))
    a._bad2 = bad2
    a.segs[1] = ctypes.cast(bad2, ctypes.POINTER(vkv.vkv_segment))
    assert call(a) == 4
    a = seg_args()
    a.n_segs[0] = 9  # more than VKV_MAX_SEGMENTS
    assert call(a) == 2


def sparse_args(**kw):
    a = seg_args()
    a.mode = vkv.MODE_BLOCK_SPARSE
    a.Lkv = 64 * 64
    a.k = T(sb=4096 * 1024)
    a.v = T(sb=4096 * 1024)
    a.block = 64
    a.persist_idx, a.n_persist = FAKE, 8
    a.sel_idx, a.topk, a.window_blk0, a.n_win_blk = FAKE, 4, 32, 32
    for k, v in kw.items():
        setattr(a, k, v)
    return a


def test_sparse_validation():
    assert call(sparse_args(block=32)) == 5
    assert call(sparse_args(topk=40)) == 2            # topk > window
    assert call(sparse_args(window_blk0=40)) == 4     # window past the cache
    assert call(sparse_args(n_persist=280, topk=8)) == 5  # block list too long
    assert call(sparse_args(sel_idx=None)) == 1
    if not torch.cuda.is_available():
        assert call(sparse_args()) == 6


def test_sparse_selection_in_kernel_validation():
    # window block means given: sel_idx is not read, the selection limits apply
    assert call(sparse_args(kbar=FAKE + 4)) == 3                      # means not 16-byte aligned
    assert call(sparse_args(kbar=FAKE, topk=0)) == 2                  # nothing to select
    a = sparse_args(kbar=FAKE, Lkv=1024 * 64, window_blk0=8, n_win_blk=513, n_persist=8)
    a.k = T(sb=1024 * 64 * 1024)
    a.v = T(sb=1024 * 64 * 1024)
    assert call(a) == 2                                               # window beyond 512 blocks
    a.n_win_blk = 512
    if not torch.cuda.is_available():
        assert call(a) == 6                                           # accepted up to the device call
        assert call(sparse_args(kbar=FAKE, sel_idx=None)) == 6
    # the selection runs on whole units: the schedule cuts no pieces where it otherwise would
    a = sparse_args(topk=144, H=2, Lq=256, n_win_blk=144, window_blk0=0, Lkv=64 * 200, n_persist=32)
    a.k = T(sb=64 * 200 * 1024)
    a.v = T(sb=64 * 200 * 1024)
    assert vkv.attn_schedule(a, 148, True)["pieces"].shape[0] > 0
    a.kbar = FAKE
    sch = vkv.attn_schedule(a, 148, True)
    assert sch["pieces"].shape[0] == 0 and sch["n_slots"] == 0


def ragged_args(cu_host):
    a = seg_args()
    a.mode = vkv.MODE_RAGGED
    a.H = 3
    a.Lkv = 1000
    a.k = vkv.vkv_tensor(FAKE, 0, 128, 0)
    a.v = vkv.vkv_tensor(FAKE, 0, 128, 0)
    a.cu_seqlens = FAKE
    arr = np.ascontiguousarray(np.asarray(cu_host, dtype=np.int32))
    a._arr = arr
    a.cu_seqlens_host = arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    a.q = T(sb=256 * 3 * 128, st=3 * 128)
    a.o[0] = T(sb=256 * 3 * 128, st=3 * 128)
    return a


def test_ragged_host_offsets_checked():
    assert call(ragged_args([0, 10, 5, 20])) == 4      # decreasing
    assert call(ragged_args([0, 10, 20, 1001])) == 4   # past the flat cache
    assert call(ragged_args([-1, 10, 20, 30])) == 4
    a = ragged_args([0, 10, 20, 30])
    a.k = vkv.vkv_tensor(FAKE, 0, 100, 0)  # row stride not a multiple of 8
    assert call(a) == 3
    if not torch.cuda.is_available():
        assert call(ragged_args([0, 10, 20, 30])) == 6


def test_block_order_validation():
    assert vkv.vkv_block_order(0, FAKE, 12, 72, 9, None) == 1
    assert vkv.vkv_block_order(FAKE, 0, 12, 72, 9, None) == 1
    assert vkv.vkv_block_order(FAKE, FAKE, 0, 72, 9, None) == 2
    assert vkv.vkv_block_order(FAKE, FAKE, 12, 0, 9, None) == 2
    assert vkv.vkv_block_order(FAKE, FAKE, 12, 72, 0, None) == 2
    assert vkv.vkv_block_order(FAKE, FAKE, 12, 4097, 9, None) == 5
    if not torch.cuda.is_available():
        assert vkv.vkv_block_order(FAKE, FAKE, 12, 72, 9, None) == 6


def test_block_select_validation_and_workspace_size():
    ws = vkv.vkv_block_select_workspace_size(1, 12, 4608, 144, 64, 128)
    assert ws == 12 * 144 * 128 * 4  # the window block means (query blocks pool in shared memory)
    assert ws % 256 == 0
    assert vkv.vkv_block_select_workspace_size(0, 12, 4608, 144, 64, 128) == 0
    s = vkv.vkv_select_args()
    s.B, s.H, s.d, s.block, s.Lq, s.Lkv = 1, 12, 128, 64, 4608, 864 * 64
    s.window_blk0, s.n_win_blk, s.topk = 720, 144, 9
    s.q, s.k = T(sb=0), T(sb=0)
    s.out_idx = FAKE
    s.workspace, s.workspace_bytes = FAKE, ws - 256
    assert vkv.vkv_block_select(s, None) == 7
    s.workspace_bytes = ws
    s.topk = 0
    assert vkv.vkv_block_select(s, None) == 2
    s.topk = 9
    s.window_blk0 = 730
    assert vkv.vkv_block_select(s, None) == 4
    s.window_blk0 = 720
    s.block = 32
    assert vkv.vkv_block_select(s, None) == 5
    s.block = 64
    if not torch.cuda.is_available():
        assert vkv.vkv_block_select(s, None) == 6


def test_lse_merge_validation():
    t = T(sb=0)
    assert vkv.vkv_lse_merge(t, FAKE, t, FAKE, t, None, 1, 2, 3, 128, None) == 1
    assert vkv.vkv_lse_merge(t, FAKE, t, FAKE, t, FAKE, 1, 2, 3, 12, None) == 5
    assert vkv.vkv_lse_merge(t, FAKE + 2, t, FAKE, t, FAKE, 1, 2, 3, 128, None) == 3
    if not torch.cuda.is_available():
        assert vkv.vkv_lse_merge(t, FAKE, t, FAKE, t, FAKE, 1, 2, 3, 128, None) == 6


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(vkv, "_lib", None)
    monkeypatch.setattr(vkv, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        vkv.lib()


def test_compact_rows_of_the_pyramid_policies():
    """Host planning of the head-aware compaction: per-head frame lists of the config-4 readings."""
    from kv_cache_attention_chunk_b200 import vkv
    a = vkv.vkv_compact_args()
    a.B, a.H, a.d, a.frame_tokens, a.hist_frames, a.cur_frames, a.recent_frames = 1, 12, 128, 1560, 60, 3, 2
    rules = [(vkv.HEAD_ANCHOR, 8)] * 4 + [(vkv.HEAD_WAVE, p) for p in (2, 3, 4, 5)] + [(vkv.HEAD_VEIL, 8)] * 4
    rr = (vkv.vkv_head_rule * 12)(*[vkv.vkv_head_rule(p, x) for p, x in rules])
    a.rules = ctypes.cast(rr, ctypes.POINTER(vkv.vkv_head_rule))
    assert vkv.vkv_compact_rows(a) == 299520
    a.B = 2
    assert vkv.vkv_compact_rows(a) == 2 * 299520
    rr[9] = vkv.vkv_head_rule(vkv.HEAD_VEIL, 3)  # odd merge count
    assert vkv.vkv_compact_rows(a) == -2  # -VKV_ERR_SHAPE


def test_compact_cache_rejects_small_output_without_a_gpu():
    from kv_cache_attention_chunk_b200 import vkv
    a = vkv.vkv_compact_args()
    a.B, a.H, a.d, a.frame_tokens, a.hist_frames, a.cur_frames, a.recent_frames = 1, 1, 64, 16, 4, 1, 1
    rr = (vkv.vkv_head_rule * 1)(vkv.vkv_head_rule(vkv.HEAD_FULL, 0))
    a.rules = ctypes.cast(rr, ctypes.POINTER(vkv.vkv_head_rule))
    assert vkv.vkv_compact_rows(a) == 5 * 16
    a.k_src = vkv.vkv_tensor(64, 64, 64, 64)
    a.v_src = vkv.vkv_tensor(64, 64, 64, 64)
    a.k_out, a.v_out, a.cu_seqlens = 64, 64, 64
    a.out_rows = 79
    assert vkv.vkv_compact_cache(a, None) == 4  # VKV_ERR_RANGE: checked before any device work


def latent_args(**kw):
    a = vkv.vkv_latent_args()
    a.B, a.H, a.Lq, a.Lkv, a.d_c, a.d_rope, a.scale = 1, 12, 4680, 32760, 192, 32, 0.088
    a.q = T(sb=4680 * 12 * 224, st=12 * 224, sh=224)
    a.kv = T(sb=32760 * 224, st=224, sh=0)
    a.o = T(sb=4680 * 12 * 192, st=12 * 192, sh=192)
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("field,value,status", [
    ("d_c", 64, 5), ("d_c", 256, 5), ("d_rope", 64, 5), ("d_rope", 0, 5),
    ("B", 0, 2), ("H", 0, 2), ("Lq", 0, 2), ("Lkv", -1, 2), ("scale", 0.0, 2), ("scale", float("inf"), 2),
])
def test_latent_bad_sizes(field, value, status):
    assert vkv.vkv_latent_attn(latent_args(**{field: value}), None) == status


def test_latent_null_and_alignment():
    assert vkv.lib().vkv_latent_attn(None, None) == 1
    assert vkv.vkv_latent_attn(latent_args(q=T(ptr=0)), None) == 1
    assert vkv.vkv_latent_attn(latent_args(kv=T(ptr=0, st=224)), None) == 1
    assert vkv.vkv_latent_attn(latent_args(q=T(ptr=FAKE + 2, sb=4680 * 12 * 224, st=12 * 224, sh=224)), None) == 3
    assert vkv.vkv_latent_attn(latent_args(kv=T(st=228, sb=32760 * 228)), None) == 3
    assert vkv.vkv_latent_attn(latent_args(kr=T(ptr=FAKE + 4, st=32, sb=32760 * 32)), None) == 3
    # an empty cache needs no cache pointer
    if not torch.cuda.is_available():
        assert vkv.vkv_latent_attn(latent_args(Lkv=0, kv=T(ptr=0)), None) == 6
        assert vkv.vkv_latent_attn(latent_args(), None) == 6


def test_withhold_copy_arming():
    assert vkv.vkv_debug_withhold_copy(-1) == 2
    assert vkv.vkv_debug_withhold_copy(1) == 0
    assert vkv.vkv_debug_withhold_copy(0) == 0
