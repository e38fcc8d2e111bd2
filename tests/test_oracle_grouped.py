"""Pins of the oracle's grouped (MoE) layer, oracle.grouped_layer (CPU only).

The grouped layer is the single layer applied to each expert e on the rows [off[e], off[e+1]) of
the packed activations, with that expert's own stored weight, adapters and NVFP4 tensor scale
("Quantized weights, full precision", "LoRA operations and quantization": LoRA on the experts of
an MoE model).  What can go wrong is bookkeeping: which rows an expert takes, and which expert's
weight, scale or adapter it uses.  The pins fix both without re-calling the single layer on a
slice:

* Experts that all share one weight and one adapter pair are one layer over all the rows: the
  concatenated Y, dX, T, U rows equal the single layer's, and the per-expert dA, dB add up to
  the single layer's.  Inputs are small dyadic values, so every fp64 sum is exact and the checks
  are equalities.
* Experts whose weights differ by known powers of two (MXFP4 scale bytes shifted by e, or NVFP4
  tensor scales 2^e) give each expert's rows exactly 2^e times the shared-weight answer; adapters
  scaled per expert scale T, U, the LoRA output and the gradients by their own known factors.  A
  row sliced into the wrong expert, or a weight, scale or adapter taken from another expert,
  changes a power of two and fails.
* An expert with no rows returns empty outputs and dA = dB = 0.

Planted mistakes (an offset moved by one row, two experts' weights or tensor scales swapped, the
adapters of the next expert, dY sliced one row late) each fail one of these pins.
"""
import numpy as np
import pytest

from oracle import oracle as O
from bit_quantized_base_b200 import synth

COUNTS = [3, 0, 5, 2]          # expert 1 has no rows
N, K, R, S = 16, 128, 4, 2.0


def _f(h):
    return synth.bf16_bits_to_f32(h).astype(np.float64)


def _dyadic(rng, shape, lo=-4, hi=4, denom=16):
    return synth.to_bf16_bits(rng.integers(lo, hi + 1, size=shape).astype(np.float32) / denom)


def _scaled_bits(h, p):
    """bf16 bit patterns times 2^p (exact for the small dyadic values used here)."""
    return synth.to_bf16_bits(_f(h).astype(np.float32) * np.float32(2.0 ** p))


def _offsets(counts):
    off = np.zeros(len(counts) + 1, np.int64)
    off[1:] = np.cumsum(counts)
    return off


def _shared_problem(fmt, seed):
    rng = np.random.default_rng(seed)
    codes, scales, ts = synth.random_stored_weight(fmt, N, K, rng)
    ts = 1.0 if ts is None else float(ts)
    off = _offsets(COUNTS)
    M = int(off[-1])
    X = _dyadic(rng, (M, K))
    dY = _dyadic(rng, (M, N))
    A = _dyadic(rng, (R, K))
    B = _dyadic(rng, (N, R))
    return codes, scales, ts, off, X, dY, A, B


def _stack(a, E):
    return np.stack([a] * E)


def _rows(res, key):
    return np.concatenate([r[key] for r in res], axis=0)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4", "nvfp4"])
def test_shared_experts_are_one_layer(fmt):
    codes, scales, ts, off, X, dY, A, B = _shared_problem(fmt, seed=21)
    E, M = len(COUNTS), int(off[-1])
    tss = np.full(E, ts, np.float32) if fmt == "nvfp4" else None
    res = O.grouped_layer(fmt, off, N, K, R, S, _stack(codes, E), _stack(scales, E), tss, X,
                          _stack(A, E), _stack(B, E), dY)
    one = O.layer(fmt, M, N, K, R, S, codes, scales, ts, X, A, B, dY)
    for key in ("Y", "dX", "T", "U"):
        np.testing.assert_array_equal(_rows(res, key), one[key])
    np.testing.assert_array_equal(sum(r["dA"] for r in res), one["dA"])
    np.testing.assert_array_equal(sum(r["dB"] for r in res), one["dB"])
    assert res[1]["Y"].shape == (0, N) and res[1]["dX"].shape == (0, K)
    assert np.all(res[1]["dA"] == 0) and np.all(res[1]["dB"] == 0)


def test_each_expert_uses_its_own_weight():
    # MXFP4: adding e to every E8M0 scale byte multiplies expert e's decoded weight by 2^e exactly
    codes, scales, _, off, X, dY, A, B = _shared_problem("mxfp4", seed=22)
    E, M = len(COUNTS), int(off[-1])
    scales = np.minimum(scales, 120).astype(np.uint8)
    sc_e = np.stack([(scales.astype(np.int32) + e).astype(np.uint8) for e in range(E)])
    B0 = np.zeros_like(B)                                   # base term only in Y and dX
    res = O.grouped_layer("mxfp4", off, N, K, R, S, _stack(codes, E), sc_e, None, X,
                          _stack(A, E), _stack(B0, E), dY)
    one = O.layer("mxfp4", M, N, K, R, S, codes, scales, 1.0, X, A, B0, dY)
    for e in range(E):
        m0, m1 = int(off[e]), int(off[e + 1])
        np.testing.assert_array_equal(res[e]["Y"], 2.0 ** e * one["Y"][m0:m1])
        np.testing.assert_array_equal(res[e]["dX"], 2.0 ** e * one["dX"][m0:m1])


def test_each_expert_uses_its_own_tensor_scale():
    codes, scales, _, off, X, dY, A, B = _shared_problem("nvfp4", seed=23)
    E, M = len(COUNTS), int(off[-1])
    tss = np.array([2.0 ** e for e in range(E)], np.float32)
    B0 = np.zeros_like(B)
    res = O.grouped_layer("nvfp4", off, N, K, R, S, _stack(codes, E), _stack(scales, E), tss, X,
                          _stack(A, E), _stack(B0, E), dY)
    one = O.layer("nvfp4", M, N, K, R, S, codes, scales, 1.0, X, A, B0, dY)
    for e in range(E):
        m0, m1 = int(off[e]), int(off[e + 1])
        np.testing.assert_array_equal(res[e]["Y"], tss[e] * one["Y"][m0:m1])
        np.testing.assert_array_equal(res[e]["dX"], tss[e] * one["dX"][m0:m1])
    # with B = 0, dB = s dY^T T does not see the tensor scale: the experts' dB add up to one layer's
    np.testing.assert_array_equal(sum(r["dB"] for r in res), one["dB"])


def test_each_expert_uses_its_own_adapters():
    # all-zero codes: Y = s T B^T, dX = s U A.  Expert e: A_e = 2^e A, B_e = 2^(2e) B, so
    # T_e = 2^e T, U_e = 2^(2e) U, Y_e = 2^(3e) Y, dX_e = 2^(3e) dX on its rows, and
    # dA_e = 2^(2e) (dA restricted to its rows), dB_e = 2^e (dB restricted to its rows).
    codes, scales, _, off, X, dY, A, B = _shared_problem("mxfp4", seed=24)
    codes = np.zeros_like(codes)
    E, M = len(COUNTS), int(off[-1])
    A_e = np.stack([_scaled_bits(A, e) for e in range(E)])
    B_e = np.stack([_scaled_bits(B, 2 * e) for e in range(E)])
    res = O.grouped_layer("mxfp4", off, N, K, R, S, _stack(codes, E), _stack(scales, E), None, X,
                          A_e, B_e, dY)
    one = O.layer("mxfp4", M, N, K, R, S, codes, scales, 1.0, X, A, B, dY)
    dA_sum = np.zeros_like(one["dA"])
    dB_sum = np.zeros_like(one["dB"])
    for e in range(E):
        m0, m1 = int(off[e]), int(off[e + 1])
        np.testing.assert_array_equal(res[e]["T"], 2.0 ** e * one["T"][m0:m1])
        np.testing.assert_array_equal(res[e]["U"], 2.0 ** (2 * e) * one["U"][m0:m1])
        np.testing.assert_array_equal(res[e]["Y"], 2.0 ** (3 * e) * one["Y"][m0:m1])
        np.testing.assert_array_equal(res[e]["dX"], 2.0 ** (3 * e) * one["dX"][m0:m1])
        dA_sum += res[e]["dA"] / 2.0 ** (2 * e)
        dB_sum += res[e]["dB"] / 2.0 ** e
    np.testing.assert_array_equal(dA_sum, one["dA"])
    np.testing.assert_array_equal(dB_sum, one["dB"])


def test_empty_expert_and_empty_batch():
    codes, scales, _, _, X, dY, A, B = _shared_problem("nf4", seed=25)
    off = np.zeros(4, np.int64)                             # three experts, no rows at all
    res = O.grouped_layer("nf4", off, N, K, R, S, _stack(codes, 3), _stack(scales, 3), None,
                          X[:0], _stack(A, 3), _stack(B, 3), dY[:0])
    for r in res:
        assert r["Y"].shape == (0, N) and r["dX"].shape == (0, K)
        assert np.all(r["dA"] == 0) and np.all(r["dB"] == 0)


# ------------------------------------------------------------------------- planted mistakes
_orig = O.grouped_layer


def _offset_moved(fmt, offsets, *a, **k):
    off = np.array(offsets, np.int64).copy()
    off[3] -= 1                                             # expert 2 ends one row early
    return _orig(fmt, off, *a, **k)


def _weights_swapped(fmt, offsets, N_, K_, r, s, codes, scales, tss, X, A, B, dY=None, **k):
    codes, scales = codes.copy(), scales.copy()
    codes[[0, 2]], scales[[0, 2]] = codes[[2, 0]], scales[[2, 0]]
    return _orig(fmt, offsets, N_, K_, r, s, codes, scales, tss, X, A, B, dY, **k)


def _tensor_scales_swapped(fmt, offsets, N_, K_, r, s, codes, scales, tss, X, A, B, dY=None, **k):
    if tss is not None:
        tss = np.array(tss).copy()
        tss[[2, 3]] = tss[[3, 2]]
    return _orig(fmt, offsets, N_, K_, r, s, codes, scales, tss, X, A, B, dY, **k)


def _next_experts_adapters(fmt, offsets, N_, K_, r, s, codes, scales, tss, X, A, B, dY=None, **k):
    A, B = np.roll(A, -1, axis=0), np.roll(B, -1, axis=0)
    return _orig(fmt, offsets, N_, K_, r, s, codes, scales, tss, X, A, B, dY, **k)


def _dy_one_row_late(fmt, offsets, N_, K_, r, s, codes, scales, tss, X, A, B, dY=None, **k):
    if dY is not None:
        dY = np.concatenate([dY[1:], dY[:1]], axis=0)
    return _orig(fmt, offsets, N_, K_, r, s, codes, scales, tss, X, A, B, dY, **k)


PINS = [lambda: test_shared_experts_are_one_layer("nvfp4"),
        test_each_expert_uses_its_own_weight,
        test_each_expert_uses_its_own_tensor_scale,
        test_each_expert_uses_its_own_adapters]

MUTANTS = [_offset_moved, _weights_swapped, _tensor_scales_swapped, _next_experts_adapters,
           _dy_one_row_late]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m.__name__ for m in MUTANTS])
def test_pins_catch_planted_grouping_mistake(monkeypatch, mutant):
    for pin in PINS:
        pin()
    monkeypatch.setattr(O, "grouped_layer", mutant)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin caught {mutant.__name__}"
