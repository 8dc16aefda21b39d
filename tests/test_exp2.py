"""The FMA-pipe base-2 exponential of the forward kernel's softmax, pinned on its own.

The d=64 softmax evaluates one exponential pair in four on the FMA and integer pipes instead
of the special-function unit: a range reduction in the style of Cody and Waite (n = floor(x)
by an add of 1.5 * 2^23 rounded toward minus infinity, f = x - n in [0, 1)), a cubic for 2^f
whose coefficients were fitted for minimum relative error on [0, 1), and n added to the
exponent field.  Its stated bound is a relative error of at most 7.5e-5 for x in (-126, 8]
(the softmax's arguments are at most 8 in log2 units: the reference maximum lags the row
maximum by at most 2^8); at x <= -126 the result is at most 2^-126, which the fp16/bf16
rounding of P and the flushed row sum discard.

The CPU tests read the coefficients out of the kernel source, restate the steps in fp32
numpy and check the bound against 2^x in fp64; planted mistakes (a round-to-nearest
reduction, reversed coefficients, a wrong exponent shift) must break it.  The GPU tests run
the kernel's own device function through the attn_debug_exp2 test hook and check it
against the exact value and against CUDA's exp2f."""
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KERNEL = os.path.join(ROOT, "exact_attention_sdpa_b200", "csrc", "attn_fwd_kernel.cuh")
BOUND = 7.5e-5


def kernel_coefficients():
    """c0..c3 of ex2_emu2 as written in the kernel source (fp32)."""
    src = open(KERNEL).read()
    body = src[src.index("void ex2_emu2("):]
    body = body[:body.index("\n}\n")]
    vals = dict(re.findall(r"\b(c[0-3]) = ([0-9.eE+-]+)f", body))
    assert sorted(vals) == ["c0", "c1", "c2", "c3"], vals
    return [np.float32(float(vals[f"c{i}"])) for i in range(4)]


def _fma32(a, b, c):
    """fp32 fused multiply-add: the fp64 product of two fp32 values is exact."""
    return (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)


def emulate(x, coeffs, round_down=True, shift_bits=23):
    """The kernel's steps in fp32 numpy."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    xf = x.astype(np.float64)
    n = np.floor(xf) if round_down else np.rint(xf)
    t = (n + 12582912.0).astype(np.float32)                    # 1.5 * 2^23 + n, exact
    r = (t.astype(np.float64) - 12582912.0).astype(np.float32)
    f = (x - r).astype(np.float32)
    c0, c1, c2, c3 = coeffs
    p = _fma32(f, np.full_like(f, c3), c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(shift_bits))
    return bits.view(np.float32)


def grid():
    rng = np.random.default_rng(0)
    dense = np.linspace(-125.999, 8.0, 2_000_001)
    near_int = (np.arange(-125, 9)[:, None] + np.array([-1e-6, 0.0, 1e-6, 0.5])[None, :]).ravel()
    rand = rng.uniform(-125.999, 8.0, 500_000)
    x = np.concatenate([dense, near_int, rand]).astype(np.float32)
    return x[(x > -126.0) & (x <= 8.0)]


def max_rel_err(y, x):
    ref = np.exp2(x.astype(np.float64))
    return float((np.abs(y.astype(np.float64) - ref) / ref).max())


def test_cubic_meets_the_stated_bound():
    x = grid()
    err = max_rel_err(emulate(x, kernel_coefficients()), x)
    assert err <= BOUND, err
    # the bound is tight for these coefficients (a fit, not a loose claim)
    assert err > 0.5 * BOUND, err


def test_clamped_range_stays_tiny():
    x = np.array([-126.0, -127.5, -200.0, -1e4, -np.inf], np.float32)
    y = emulate(x, kernel_coefficients())
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -126)


@pytest.mark.parametrize("mistake", ["round_nearest", "reversed", "shift22", "dropped_cubic"])
def test_planted_mistakes_break_the_bound(mistake):
    c = kernel_coefficients()
    x = grid()[::7]
    if mistake == "round_nearest":
        y = emulate(x, c, round_down=False)
    elif mistake == "reversed":
        y = emulate(x, c[::-1])
    elif mistake == "shift22":
        y = emulate(x, c, shift_bits=22)
    else:
        y = emulate(x, [c[0], c[1], c[2], np.float32(0.0)])
    assert not max_rel_err(y, x) <= BOUND          # (a NaN from a broken exponent field fails too)


@pytest.mark.gpu
def test_device_fma_pipe_exp2_against_exact_and_exp2f():
    from exact_attention_sdpa_b200._native import EXP2_CUDA_EXP2F, EXP2_FMA_PIPE, debug_exp2
    x = grid()
    xd = torch.from_numpy(x).cuda()
    y = debug_exp2(xd, EXP2_FMA_PIPE).cpu().numpy()
    ref_cuda = debug_exp2(xd, EXP2_CUDA_EXP2F).cpu().numpy()
    torch.cuda.synchronize()
    # the kernel's output is the fp32 result of the cubic: its own bound plus one fp32 rounding
    assert max_rel_err(y, x) <= BOUND + 2.0 ** -23
    rel_cuda = np.abs(y.astype(np.float64) - ref_cuda) / ref_cuda.astype(np.float64)
    assert float(rel_cuda.max()) <= BOUND + 2.0 ** -22
    # the device result agrees with the fp32 restatement to an ulp or two (fused vs emulated FMA)
    ye = emulate(x, kernel_coefficients())
    assert float((np.abs(y.astype(np.float64) - ye) / ye).max()) <= 2.0 ** -21
    lo = torch.tensor([-126.0, -127.5, -200.0, -1e4, float("-inf"), -126.0], device="cuda")
    ylo = debug_exp2(lo, EXP2_FMA_PIPE).cpu().numpy()
    assert np.all(ylo >= 0) and np.all(ylo <= 2.0 ** -126)


@pytest.mark.gpu
def test_device_mufu_exp2_against_exact():
    from exact_attention_sdpa_b200._native import EXP2_MUFU, debug_exp2
    x = grid()
    y = debug_exp2(torch.from_numpy(x).cuda(), EXP2_MUFU).cpu().numpy()
    assert max_rel_err(y, x) <= 2.0 ** -20
