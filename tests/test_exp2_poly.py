"""The FMA-pipe 2^x polynomial of the encoder's softmax (exp2_poly2 in csrc/ptx.cuh).

2^x = 2^n * 2^f with n = round(x), f in [-1/2, 1/2], and 2^f from a degree-3
polynomial chosen to minimise the maximum RELATIVE error on [-1/2, 1/2] (a
minimax fit, computed with the Remez exchange algorithm). These tests

* regenerate the four coefficients from that definition (Remez exchange in
  float64, then rounded to float32) and require the constants compiled into the
  kernels to be exactly those float32 values;
* emulate the kernel's float32 evaluation (range reduction by the 1.5 * 2^23
  shift, Horner with fused multiply-adds, exponent-field insertion, clamp at
  -125) and bound its relative error against float64 2^x over [-125, 8];
* on a GPU, run the device routine itself over the same sweep.

The bound, 7.48e-5 relative (about 630 float32 ulp), is 26 times smaller than
the 2^-9 relative rounding of the bf16 P the result is packed into.
"""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "online_softmax_attention_flash_b200", "csrc", "ptx.cuh")
POLY_BOUND = 7.5e-5        # minimax relative error of the fit (7.478e-5) plus float32 rounding
SWEEP = (-125.0, 8.0)


def remez_relative(deg=3, a=-0.5, b=0.5, iters=40, grid=200001):
    """Minimax polynomial for 2^x on [a, b] in the relative sense (Remez exchange).

    Solve p(x_i) - 2^x_i = (-1)^i E 2^x_i on deg + 2 reference points, move the
    reference to the extrema of the relative error between its sign changes, repeat.
    Returns (coefficients c0..c_deg in float64, max relative error).
    """
    n = deg + 2
    k = np.arange(n)
    x = (a + b) / 2 - (b - a) / 2 * np.cos(np.pi * k / (n - 1))   # Chebyshev extrema
    t = np.linspace(a, b, grid)
    for _ in range(iters):
        A = np.empty((n, n))
        A[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)[None, :]
        A[:, deg + 1] = (-1.0) ** k * np.exp2(x)
        c = np.linalg.solve(A, np.exp2(x))[:deg + 1]
        err = np.polyval(c[::-1], t) / np.exp2(t) - 1.0
        segs = np.split(np.arange(grid), np.flatnonzero(np.diff(np.sign(err)) != 0) + 1)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        assert len(ext) == n, "equioscillation lost"
        x = t[ext]
    return c, float(np.max(np.abs(err)))


def kernel_constants():
    src = open(PTX, encoding="utf-8").read()
    body = src[src.index("exp2_poly2"):]
    vals = {m.group(1): np.float32(m.group(2))
            for m in re.finditer(r"kC([0-3])\s*=\s*([-0-9.eE+]+)f", body)}
    shift = np.float32(re.search(r"kShift\s*=\s*([0-9.eE+]+)f", body).group(1))
    return [vals[str(i)] for i in range(4)], shift


def fma32(a, b, c):
    """float32 fused multiply-add: the float64 result (a*b is exact there) rounded once."""
    return (np.float64(a) * np.float64(b) + np.float64(c)).astype(np.float32)


def exp2_poly_emulated(x):
    """The kernel's float32 arithmetic, step by step."""
    (c0, c1, c2, c3), shift = kernel_constants()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    j = (x + shift).astype(np.float32)                 # round-to-nearest of x in the low bits
    n = (j - shift).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = fma32(c3, f, c2)
    p = fma32(p, f, c1)
    p = fma32(p, f, c0)
    bits = p.view(np.int32) + (j.view(np.int32) << 23)
    return bits.view(np.float32)


def test_coefficients_are_the_remez_minimax_fit():
    c, emax = remez_relative()
    assert abs(emax - 7.478e-5) < 1e-7
    got, shift = kernel_constants()
    assert shift == np.float32(1.5 * 2 ** 23)
    assert [np.float32(v) for v in c] == got, (c, got)


def test_emulated_relative_error_over_the_softmax_range():
    x = np.linspace(*SWEEP, 2_000_001).astype(np.float32)
    y = exp2_poly_emulated(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= POLY_BOUND, rel.max()
    # far below the bf16 rounding of P (2^-9 relative)
    assert rel.max() < 2.0 ** -9 / 20


def test_a_wrong_coefficient_breaks_the_bound():
    # pin sanity: the emulation is sensitive to the constants it reads
    (c0, c1, c2, c3), shift = kernel_constants()
    x = np.linspace(-0.5, 0.5, 10001).astype(np.float32)
    f = x.astype(np.float64)
    p = ((np.float64(c3) * 1.01 * f + c2) * f + c1) * f + c0
    assert np.max(np.abs(p / np.exp2(f) - 1.0)) > POLY_BOUND


@pytest.fixture(scope="module")
def probe_lib(tmp_path_factory):
    from online_softmax_attention_flash_b200 import build as b
    out = str(tmp_path_factory.mktemp("probe") / "libexp2_probe.so")
    src = os.path.join(ROOT, "tests", "kernels", "exp2_probe.cu")
    subprocess.run([b.nvcc_path(), *b.ARCH_FLAGS, "-O3", "-std=c++17", "-shared", "-Xcompiler",
                    "-fPIC", "-I", b.CSRC, "-o", out, src], check=True)
    lib = ctypes.CDLL(out)
    lib.exp2_probe.restype = ctypes.c_int
    lib.exp2_probe.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p]
    return lib


@pytest.mark.gpu
def test_device_polynomial_and_mufu_against_float64(probe_lib):
    import torch
    x = torch.linspace(*SWEEP, 4_000_001, dtype=torch.float32)
    xd = x.cuda()
    yp = torch.empty_like(xd)
    ym = torch.empty_like(xd)
    s = torch.cuda.current_stream()
    assert probe_lib.exp2_probe(xd.data_ptr(), yp.data_ptr(), ym.data_ptr(), x.numel(),
                                s.cuda_stream) == 0
    torch.cuda.synchronize()
    ref = np.exp2(x.double().numpy())
    rel_poly = np.abs(yp.cpu().double().numpy() / ref - 1.0)
    rel_mufu = np.abs(ym.cpu().double().numpy() / ref - 1.0)
    assert rel_poly.max() <= POLY_BOUND, rel_poly.max()
    # the device result is the float32 emulation above (within one ulp: the emulated fused
    # multiply-add rounds through float64, which can differ in rare double-rounding cases)
    dev_bits = yp.cpu().numpy().view(np.int32).astype(np.int64)
    emu_bits = exp2_poly_emulated(x.numpy()).view(np.int32).astype(np.int64)
    assert np.max(np.abs(dev_bits - emu_bits)) <= 1
    # MUFU ex2.approx.ftz: a few ulp (context for the polynomial's ~630 ulp)
    assert rel_mufu.max() <= 2.0 ** -21, rel_mufu.max()
