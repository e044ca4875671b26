"""The FMA-pipe exp2 of the attention softmax (vkv_attn_kernel.cuh, exp2_poly2).

Part of the softmax's exponentials are computed as 2^x = 2^r * q(f), r = round(x),
f = x - r in [-1/2, 1/2], q a cubic fitted to 2^f by relative-error minimax
(csrc/fit_exp2_poly.py).  CPU: the fit reproduces the constants in the kernel
source, its error bound holds, and the whole algorithm evaluated in fp32 stays
within 1e-4 relative of 2^x.  GPU (test build): the device function itself
against 2^x in fp64.
"""
import importlib.util
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "kv_cache_attention_chunk_b200", "csrc")
REL_BOUND = 1.0e-4  # the fit's 7.5e-5, with fp32 evaluation rounding


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2_poly", os.path.join(CSRC, "fit_exp2_poly.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_fit_reproduces_kernel_constants():
    m = _fit_module()
    c = m.coefficients()  # c0..c3
    text = open(os.path.join(CSRC, "vkv_attn_kernel.cuh")).read()
    text = text[text.index("void exp2_poly2("):]
    src = [float(x) for x in re.findall(r"pack2f\(([0-9.]+)f, [0-9.]+f\)", text)]
    used = [v for v in src if v != 12582912.0][:4]  # c3, c2, c1, c0 in Horner order
    assert np.array_equal(np.float32(used[::-1]), np.float32(c))
    exact, horner = m.errors(c)
    assert exact < 7.6e-5 and horner < 7.6e-5


def _device_algorithm(x):
    """The kernel's steps in fp32 (numpy; the kernel fuses the multiply-adds)."""
    c = np.float32(_fit_module().coefficients())
    f32 = np.float32
    xc = np.maximum(x.astype(f32), f32(-126.0))
    magic = f32(12582912.0)  # 1.5 * 2^23: adding it rounds to an integer in the low mantissa bits
    t = (xc + magic).astype(f32)
    fr = (xc - (t - magic)).astype(f32)
    q = ((c[3] * fr + c[2]) * fr + c[1]).astype(f32)
    q = (q * fr + c[0]).astype(f32)
    e = (t.view(np.uint32) * np.uint32(8388608) + q.view(np.uint32)).view(np.float32)
    return e


def test_algorithm_relative_error_and_masked_arguments():
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-125.0, 8.0, 400001), rng.uniform(-125.0, 8.0, 200000),
                        np.arange(-125, 9).astype(np.float64) + 0.5]).astype(np.float32)
    e = _device_algorithm(x).astype(np.float64)
    rel = np.abs(e / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= REL_BOUND
    masked = _device_algorithm(np.array([-np.inf, -1000.0, -127.0], dtype=np.float32))
    assert np.all(masked >= 0) and np.all(masked <= 2.0 ** -125)


def test_planted_wrong_coefficient_is_caught():
    """A coefficient off in its fourth digit breaks the bound (the check can fail)."""
    m = _fit_module()
    c = m.coefficients()
    c[2] *= 1.001
    assert m.errors(c)[0] > REL_BOUND


@pytest.mark.gpu
def test_device_exp2_poly_against_fp64():
    from kv_cache_attention_chunk_b200 import build, vkv
    build.build()
    L = vkv.test_lib()
    rng = np.random.default_rng(11)
    x = np.concatenate([np.linspace(-125.0, 8.0, 1 << 20), rng.uniform(-125.0, 8.0, 1 << 18)]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    assert L.vkv_debug_exp2_poly(xd.data_ptr(), yd.data_ptr(), xd.numel(), None) == 0
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= REL_BOUND, rel.max()
    m = torch.tensor([-np.inf, -1000.0, -127.0], dtype=torch.float32, device="cuda")
    ym = torch.empty_like(m)
    assert L.vkv_debug_exp2_poly(m.data_ptr(), ym.data_ptr(), 3, None) == 0
    torch.cuda.synchronize()
    assert bool((ym >= 0).all()) and bool((ym <= 2.0 ** -125).all())
