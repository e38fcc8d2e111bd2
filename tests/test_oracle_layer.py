"""Pins of the oracle's layer forward/backward (CPU only).

* Gradients against central finite differences of L = <G, Y>: L is linear in each of X, A and B
  separately, so with steps h that keep every perturbed input exactly representable in bf16 the
  central difference IS the derivative (up to fp64 rounding).  A dropped scale, a wrong sign or a
  transposed operand in dX / dA / dB fails here.
* The step-0 table of "Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §2 "Initialization
  matters" (golden/lora_init_gradients.txt): B = 0 -> dA = 0, dB != 0; A = 0 -> dB = 0, dA != 0;
  and B = 0 makes Y the frozen base output exactly.
* Special cases that reduce to a library matmul: B = 0 (Y = X deq(W)^T), all-zero weight codes
  (Y = s X A^T B^T), compared with numpy's BLAS in fp64 on the oracle's own decoded weight.
* Linearity of the LoRA term in s.
"""
import numpy as np
import pytest

from conftest import read_golden
from oracle import oracle as O
from bit_quantized_base_b200 import synth


def _f(h):
    return synth.bf16_bits_to_f32(h).astype(np.float64)


def _dyadic_bf16(rng, shape, lo=-4, hi=4, denom=16):
    """Values k/denom with small integer k: exact in bf16, and so are k/denom +- 1/denom."""
    return synth.to_bf16_bits(rng.integers(lo, hi + 1, size=shape).astype(np.float32) / denom)


def _problem(fmt, M, N, K, r, seed):
    rng = np.random.default_rng(seed)
    codes, scales, ts = synth.random_stored_weight(fmt, N, K, rng)
    ts = 1.0 if ts is None else float(ts)
    X = _dyadic_bf16(rng, (M, K))
    A = _dyadic_bf16(rng, (r, K))
    B = _dyadic_bf16(rng, (N, r))
    G = synth.to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    return codes, scales, ts, X, A, B, G


def _loss(fmt, M, N, K, r, s, codes, scales, ts, X, A, B, G):
    Y = O.layer(fmt, M, N, K, r, s, codes, scales, ts, X, A, B, None, want=("Y",))["Y"]
    return float(np.sum(Y * _f(G)))


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4", "nvfp4"])
def test_gradients_match_central_differences(fmt):
    M, N, K, r, s = 5, 16, 64, 4, 1.75
    codes, scales, ts, X, A, B, G = _problem(fmt, M, N, K, r, seed=11)
    out = O.layer(fmt, M, N, K, r, s, codes, scales, ts, X, A, B, G)
    h = 1.0 / 16

    def fd(name, idx):
        arrs = {"X": X, "A": A, "B": B}
        plus, minus = {k: v.copy() for k, v in arrs.items()}, {k: v.copy() for k, v in arrs.items()}
        v = _f(arrs[name][idx])
        plus[name][idx] = synth.to_bf16_bits(np.array([v + h], np.float32))[0]
        minus[name][idx] = synth.to_bf16_bits(np.array([v - h], np.float32))[0]
        assert _f(plus[name][idx]) == v + h and _f(minus[name][idx]) == v - h
        lp = _loss(fmt, M, N, K, r, s, codes, scales, ts, plus["X"], plus["A"], plus["B"], G)
        lm = _loss(fmt, M, N, K, r, s, codes, scales, ts, minus["X"], minus["A"], minus["B"], G)
        return (lp - lm) / (2 * h)

    rng = np.random.default_rng(5)
    for _ in range(6):
        j, k = int(rng.integers(r)), int(rng.integers(K))
        assert np.isclose(fd("A", (j, k)), out["dA"][j, k], rtol=1e-9, atol=1e-9)
        n, j = int(rng.integers(N)), int(rng.integers(r))
        assert np.isclose(fd("B", (n, j)), out["dB"][n, j], rtol=1e-9, atol=1e-9)
        m, k = int(rng.integers(M)), int(rng.integers(K))
        assert np.isclose(fd("X", (m, k)), out["dX"][m, k], rtol=1e-9, atol=1e-9)


def test_step0_initialisation_table():
    M, N, K, r, s = 6, 32, 128, 8, 2.0
    codes, scales, ts, X, A, B, G = _problem("nf4", M, N, K, r, seed=3)
    zeroB = np.zeros_like(B)
    zeroA = np.zeros_like(A)
    expect = {row[0]: (row[1], row[2]) for row in read_golden("lora_init_gradients.txt")}
    o1 = O.layer("nf4", M, N, K, r, s, codes, scales, ts, X, A, zeroB, G)
    o2 = O.layer("nf4", M, N, K, r, s, codes, scales, ts, X, zeroA, B, G)
    for out, key in ((o1, "A_random_B_zero"), (o2, "A_zero_B_random")):
        dA_zero = bool(np.all(out["dA"] == 0.0))
        dB_zero = bool(np.all(out["dB"] == 0.0))
        assert dA_zero == (expect[key][0] == "zero"), key
        assert dB_zero == (expect[key][1] == "zero"), key
    # B = 0: the forward pass is exactly the frozen base output
    Wd = _f(O.dequant("nf4", N, K, codes, scales))
    base = _f(X) @ Wd.T
    np.testing.assert_allclose(o1["Y"], base, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4", "nvfp4"])
def test_b_zero_reduces_to_dense_matmul(fmt):
    M, N, K, r = 9, 48, 192, 16
    p = synth.small_layer(fmt, M, N, K, r, seed=4)
    B0 = np.zeros_like(p["B"])
    out = O.layer(fmt, M, N, K, r, p["s"], p["codes"], p["scales"], p["tensor_scale"], p["X"],
                  p["A"], B0, p["dY"])
    Wd = _f(O.dequant(fmt, N, K, p["codes"], p["scales"], p["tensor_scale"]))
    np.testing.assert_allclose(out["Y"], _f(p["X"]) @ Wd.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(out["dX"], _f(p["dY"]) @ Wd, rtol=1e-12, atol=1e-12)
    assert np.all(out["dA"] == 0.0)


def test_zero_weight_reduces_to_lora_chain():
    M, N, K, r, s = 7, 32, 128, 8, 0.5
    p = synth.small_layer("mxfp4", M, N, K, r, seed=8)
    codes = np.zeros_like(p["codes"])                 # every element code 0 -> +0
    out = O.layer("mxfp4", M, N, K, r, s, codes, p["scales"], 1.0, p["X"], p["A"], p["B"], p["dY"])
    X, A, B, G = _f(p["X"]), _f(p["A"]), _f(p["B"]), _f(p["dY"])
    np.testing.assert_allclose(out["Y"], s * (X @ A.T) @ B.T, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(out["dX"], s * (G @ B) @ A, rtol=1e-11, atol=1e-13)


def test_lora_term_linear_in_scale():
    M, N, K, r = 4, 32, 128, 8
    p = synth.small_layer("nf4", M, N, K, r, seed=9)
    args = (p["codes"], p["scales"], 1.0, p["X"], p["A"], p["B"], p["dY"])
    y0 = O.layer("nf4", M, N, K, r, 0.0, *args)
    y1 = O.layer("nf4", M, N, K, r, 1.0, *args)
    y3 = O.layer("nf4", M, N, K, r, 3.0, *args)
    for name in ("Y", "dX"):
        np.testing.assert_allclose(y3[name] - y0[name], 3.0 * (y1[name] - y0[name]),
                                   rtol=1e-9, atol=1e-12)
    for name in ("dA", "dB"):
        np.testing.assert_allclose(y3[name], 3.0 * y1[name], rtol=1e-12, atol=0)


def test_row_sampling_matches_full():
    M, N, K, r = 12, 32, 128, 8
    p = synth.small_layer("nvfp4", M, N, K, r, seed=12)
    args = ("nvfp4", M, N, K, r, p["s"], p["codes"], p["scales"], p["tensor_scale"], p["X"],
            p["A"], p["B"], p["dY"])
    full = O.layer(*args)
    rows = np.array([11, 0, 5], np.int64)
    part = O.layer(*args, rows=rows)
    np.testing.assert_array_equal(part["Y"], full["Y"][rows])
    np.testing.assert_array_equal(part["dX"], full["dX"][rows])
    for k in ("dA", "dB", "T", "U"):
        np.testing.assert_array_equal(part[k], full[k])


def test_lora_shapes_pin_parameter_count():
    (r, d_in, d_out, params), = read_golden("lora_param_count.txt")
    r, d_in, d_out = int(r), int(d_in), int(d_out)
    # the layer takes A [r, d_in] and B [d_out, r]
    assert r * d_in + d_out * r == int(params)


def test_empty_batch():
    p = synth.small_layer("nf4", 3, 16, 64, 8, seed=1)
    out = O.layer("nf4", 0, 16, 64, 8, 2.0, p["codes"], p["scales"], 1.0, p["X"][:0], p["A"],
                  p["B"], p["dY"][:0])
    assert out["Y"].shape == (0, 16) and np.all(out["dA"] == 0) and np.all(out["dB"] == 0)
