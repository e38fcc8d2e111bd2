"""Pins of the oracle for the opt-in native block-scaled MMA forward (4-bit weight codes times
MXFP8 activations): the activation quantiser against a brute-force nearest-value search and
numpy's frexp, and the forward against the plain layer oracle where the quantisation is exact
and against the element-wise error bound where it is not (CPU only)."""
import math

import numpy as np
import pytest

from oracle import oracle as O
from bit_quantized_base_b200 import synth

E4M3 = np.array([O.decode_e4m3(c) for c in range(0x7F)], np.float64)


def _nearest_e4m3(a):
    """Brute force: the code of the nearest E4M3 magnitude to a >= 0 (saturating at 448), an
    exact tie going to the even code."""
    a = min(a, 448.0)
    d = np.abs(E4M3 - a)
    best = np.flatnonzero(d == d.min())
    even = best[best % 2 == 0]
    return int(even[0] if len(even) else best[0])


def test_mxfp8_quantize_brute_force():
    rng = np.random.default_rng(41)
    M, K = 6, 256
    x = rng.standard_normal((M, K)) * np.exp2(rng.integers(-20, 20, size=(M, 1)))
    x[2, 32:64] = 0.0                                   # zero block
    x[3, :32] = 0.0
    x[3, 0] = 1.0                                       # scale 2^-8: q = 256 x
    x[3, 1:9] = [0.5 * (E4M3[c] + E4M3[c + 1]) / 256.0 for c in (0x30, 0x31, 0x40, 0x41, 0x07, 0x08, 0x7C, 0x7D)]
    codes, e = O.mxfp8_quantize(x)
    amax = np.abs(x.reshape(M, K // 32, 32)).max(axis=2)
    for i in range(M):
        for b in range(K // 32):
            if amax[i, b] == 0:
                assert e[i, b] == 0
                continue
            _, p = math.frexp(amax[i, b])              # amax = m 2^p, m in [0.5, 1)
            assert e[i, b] == min(max(p - 1 - 8 + 127, 0), 254)
    for i in range(M):
        for k in range(K):
            sc = math.ldexp(1.0, int(e[i, k // 32]) - 127)
            q = x[i, k] / sc
            want = _nearest_e4m3(abs(q))
            if want != 0 and q < 0:
                want |= 0x80
            assert codes[i, k] == want, (i, k, x[i, k])
    # the planted midpoints: each tie goes to the even code of its pair
    assert [int(c) for c in codes[3, 1:9]] == [0x30, 0x32, 0x40, 0x42, 0x08, 0x08, 0x7C, 0x7E]


def _codes_no_top_mantissa(rng, M, K):
    """Random E4M3 codes (either sign, no NaN) whose mantissa field is at most 6 (1.75): the
    shared-exponent rule maps a block's largest magnitude into [256, 512) and the grid tops out
    at 448 = 1.75 x 2^8, so a block led by a mantissa of 1.875 would saturate when requantised."""
    c = rng.integers(0, 0x7F, size=(M, K)).astype(np.uint8)
    c = np.where((c & 7) == 7, c - 1, c).astype(np.uint8)
    return c | (rng.integers(0, 2, size=(M, K)) << 7).astype(np.uint8)


def test_mxfp8_round_trip_of_representable_values():
    rng = np.random.default_rng(42)
    M, K = 8, 128
    codes = _codes_no_top_mantissa(rng, M, K)
    e = rng.integers(100, 150, size=(M, K // 32)).astype(np.uint8)
    v = O.mxfp8_dequant(codes, e)
    c2, e2 = O.mxfp8_quantize(v)
    assert np.array_equal(O.mxfp8_dequant(c2, e2), v)   # values (a -0 comes back as +0)


def _rep_activations(rng, M, K):
    """bf16 bit patterns of activations that MXFP8 represents exactly (E4M3 values, 4
    significant bits, times powers of two: exact in bf16 as well)."""
    codes = _codes_no_top_mantissa(rng, M, K)
    e = rng.integers(118, 126, size=(M, K // 32)).astype(np.uint8)
    x = O.mxfp8_dequant(codes, e).astype(np.float32)
    return synth.to_bf16_bits(x)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_w4a8_forward_equals_layer_when_exact(fmt):
    # activations on the MXFP8 grid and, for NVFP4, a power-of-two tensor scale: every product
    # is exact, so the W4A8 forward equals the plain layer oracle up to fp64 summation order
    rng = np.random.default_rng(43)
    M, N, K, r, s = 24, 48, 256, 8, 2.0
    p = synth.small_layer(fmt, M, N, K, r, s=s, seed=9, random_codes=True)
    X = _rep_activations(rng, M, K)
    ts = 0.5 if fmt == "nvfp4" else 1.0
    y8 = O.layer_w4a8_forward(fmt, M, N, K, r, s, p["codes"], p["scales"], ts, X, p["A"], p["B"])
    y = O.layer(fmt, M, N, K, r, s, p["codes"], p["scales"], ts, X, p["A"], p["B"], want=("Y",))["Y"]
    assert np.allclose(y8, y, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_w4a8_forward_error_bound():
    # generic bf16 activations: |Y8 - Y| <= sum_k |x - deq8(q(x))| |w| element-wise, with Y the
    # same forward on the unquantised X; the per-element quantisation error is within half an
    # E4M3 step of its block, or is the clipping of a magnitude above 448 x the block scale (the
    # shared exponent puts the block maximum in [256, 512) x scale)
    rng = np.random.default_rng(44)
    M, N, K, r, s = 16, 32, 192, 8, 2.0
    p = synth.small_layer("mxfp4", M, N, K, r, s=s, seed=10, random_codes=True)
    X = p["X"]
    y8 = O.layer_w4a8_forward("mxfp4", M, N, K, r, s, p["codes"], p["scales"], 1.0, X, p["A"], p["B"])
    y = O.layer("mxfp4", M, N, K, r, s, p["codes"], p["scales"], 1.0, X, p["A"], p["B"], want=("Y",))["Y"]
    Xf = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    qc, qe = O.mxfp8_quantize(Xf)
    dx = np.abs(Xf - O.mxfp8_dequant(qc, qe))
    sc = np.repeat(np.exp2(qe.astype(np.float64) - 127.0), 32, axis=1)
    clip = np.abs(Xf) - 448.0 * sc
    assert np.all(dx <= np.maximum(np.maximum(np.abs(Xf) * 2.0 ** -4, sc * 2.0 ** -10), clip) * (1 + 1e-12))
    assert (clip > 0).any()                              # the clipping case is exercised
    Wd = (O.dequant("mxfp4", N, K, p["codes"], p["scales"]).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bound = dx @ np.abs(Wd).T
    assert np.all(np.abs(y8 - y) <= bound * (1 + 1e-9) + 1e-12 * np.abs(y).max())
    assert np.abs(y8 - y).max() > 0                      # the quantisation is visible
