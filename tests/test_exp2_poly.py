"""The FMA-pipe exponential used next to the MUFU one in the softmax
(exp2_poly in gad_ptx.cuh): its coefficients are the degree-4 polynomial that
interpolates 2^f at the five Chebyshev nodes of [-1/2, 1/2], and with fp32
Horner steps it stays within 4e-6 relative error of 2^x, far below the fp16
rounding (2^-11) the softmax weights get next.  Host-side check of the
constants and of the exponent-field arithmetic, emulated in numpy float32."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _coefficients():
    src = open(os.path.join(ROOT, "paged_fp8_gated_b200", "csrc", "gad_ptx.cuh")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("return")]
    hexes = re.findall(r"(0x[0-9a-f.]+p[-+]\d+)f", body)
    # fmaf(c4, f, c3), fmaf(p, f, c2), fmaf(p, f, c1), fmaf(p, f, 1.0f)
    consts = [float.fromhex(h) for h in hexes if h not in ("0x1.8p+23",)]
    c4, c3, c2, c1 = consts
    return np.float32([1.0, c1, c2, c3, c4])


def _emulate(x, c):
    x = np.maximum(np.float32(x), np.float32(-125.0))
    t = (x + np.float32(1.5 * 2 ** 23)).astype(np.float32)
    f = (x - (t - np.float32(1.5 * 2 ** 23)).astype(np.float32)).astype(np.float32)
    p = np.float32(c[4])
    for k in (3, 2, 1, 0):
        p = (p * f + c[k]).astype(np.float32)   # fp32 product then sum: at least as far off as a fused step
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.astype(np.int32).view(np.float32)


def test_coefficients_are_the_chebyshev_interpolant():
    c = _coefficients()
    n = 4
    k = np.arange(n + 1)
    nodes = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * (n + 1)))
    want = np.linalg.solve(np.vander(nodes, n + 1, increasing=True), 2.0 ** nodes)
    assert np.array_equal(c, want.astype(np.float32))


def test_relative_error_over_the_softmax_range():
    c = _coefficients()
    x = np.concatenate([np.linspace(-120.0, 8.0, 400001), -np.arange(0, 120) - 0.5,
                        np.float32([0.0, -1.0, 1.0, 7.5])]).astype(np.float32)
    got = _emulate(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.all(np.abs(got / want - 1.0) < 5e-6)
    # below the clamp: a tiny positive weight, 0 after the fp16 rounding
    tiny = _emulate(np.float32([-200.0, -np.inf]), c)
    assert np.all(tiny == np.float32(2.0 ** -125))
    assert np.all(tiny.astype(np.float16) == 0)
