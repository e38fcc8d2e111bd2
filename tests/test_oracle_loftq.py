"""Pins of the oracle's LoftQ initialisation (CPU only).

"Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §4: alternate Q = quantise(W - s B A) and
s B A = best rank-r approximation of W - Q.  Pinned by the page's worked 3x3 example (integer
rounding for the quantiser), by Eckart-Young (the error of each SVD step equals the energy of the
discarded singular values, computed here by an independent eigen-solver on R R^T), and by a
planted case whose answer is known in closed form: a weight that is an NF4 grid point plus a
rank-2 matrix too small to move any code, which LoftQ recovers exactly after one iteration."""
import os

import numpy as np
import pytest

from oracle import oracle as O
from loftq_cases import planted

GOLD = os.path.join(os.path.dirname(__file__), "golden", "loftq_3x3.txt")


def _golden():
    lines = [l.split("#")[0].strip() for l in open(GOLD)]
    lines = [l for l in lines if l]
    out, i = {}, 0
    while i < len(lines):
        head = lines[i].split()
        if len(head) == 2:
            out[head[0]] = float(head[1])
            i += 1
        elif head[0] in ("u", "v"):
            out[head[0]] = np.array([float(x) for x in lines[i + 1].split()])
            i += 2
        else:
            out[head[0]] = np.array([[float(x) for x in lines[i + j].split()] for j in (1, 2, 3)])
            i += 4
    return out


@pytest.mark.parametrize("s", [1.0, 2.0])
def test_loftq_worked_example(s):
    g = _golden()
    res = O.loftq(g["W"], r=1, s=s, iters=1, quant=np.rint)
    assert np.array_equal(np.rint(g["W"]), g["Q0"])
    assert np.allclose(g["W"] - g["Q0"], g["R0"], atol=1e-12)
    assert np.allclose(np.outer(g["u"], g["v"]), g["R0"], atol=1e-12)     # R0 is rank 1
    assert abs(res["errs"][0] - g["err_qlora"]) < 1e-12
    assert abs(res["errs"][1] - g["err_loftq_1"]) < 1e-12
    assert np.allclose(s * res["B"] @ res["A"], g["R0"], atol=1e-12)
    # B = U sqrt(sigma / s), A = sqrt(sigma / s) V^T: both factors carry half of sigma
    assert np.allclose(np.linalg.norm(res["B"]), np.linalg.norm(res["A"]), atol=1e-12)
    more = O.loftq(g["W"], r=1, s=s, iters=5, quant=np.rint)
    assert all(abs(e - g["err_loftq_more"]) < 1e-12 for e in more["errs"][1:])
    assert np.array_equal(more["Q"], g["Q0"])


def test_loftq_svd_step_is_eckart_young():
    # each iteration's error is the energy of R_t's discarded spectrum; the spectrum here comes
    # from numpy's symmetric eigen-solver on R R^T, not from the SVD the oracle uses
    rng = np.random.default_rng(3)
    N, K, r = 40, 96, 5
    W = rng.standard_normal((N, K)) * 0.7
    res = O.loftq(W, r=r, s=0.5, iters=1, quant=lambda v: np.round(v * 2) / 2)
    R = W - np.round(W * 2) / 2
    lam = np.sort(np.linalg.eigvalsh(R @ R.T))[::-1]
    assert abs(res["errs"][1] - np.sqrt(lam[r:].sum())) < 1e-9
    assert np.allclose(res["sigma"] ** 2, lam[:r], rtol=1e-9)
    assert res["errs"][1] < res["errs"][0]


def test_loftq_planted_nf4_is_recovered():
    N, K, rank = 32, 256, 2
    W, packed, a, Df, L = planted(N, K, rank, 7)
    res = O.loftq(W, r=rank, s=2.0, iters=3, fmt="nf4")
    codes, scales, _, _ = res["stored"]
    assert np.array_equal(codes, packed) and np.array_equal(scales, a)
    assert np.array_equal(res["Q"], Df)
    assert abs(res["errs"][0] - np.linalg.norm(W.astype(np.float64) - Df)) < 1e-12
    # what is left is W's own fp32 rounding of D + L: L is a rank-2 candidate, so the best rank-2
    # fit leaves at most ||(W - D) - L||, and that is below 1e-4 of the start
    resid = np.linalg.norm(W.astype(np.float64) - Df - L)
    assert res["errs"][1] <= resid * (1 + 1e-9) and resid < 1e-4 * res["errs"][0]
    assert np.allclose(2.0 * res["B"] @ res["A"], L, rtol=0, atol=1e-4 * np.abs(L).max())
    # a rank below the planted one cannot recover it: the error stays at the dropped factor
    low = O.loftq(W, r=rank - 1, s=2.0, iters=1, fmt="nf4")
    assert low["errs"][1] > 1e-3 * low["errs"][0]


def test_loftq_planted_mxfp4_is_recovered():
    # the same construction on the MXFP4 grid: every 32-block holds +6 (code 7) in column 0 at
    # scale 2^(e-127), so its exponent stays e; the other codes lie in +-{0.5 .. 4} and L, zero on
    # column 0, stays below a quarter of the smallest step (0.5 x scale): quantising W gives D back
    rng = np.random.default_rng(8)
    N, K, rank = 16, 256, 3
    mag = rng.integers(1, 7, size=(N, K))                   # E2M1 magnitude codes 1..6
    sign = rng.integers(0, 2, size=(N, K)) << 3
    codes = (mag | sign).astype(np.uint8)
    codes[:, ::32] = 7
    e = rng.integers(118, 124, size=(N, K // 32)).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    D = (O.dequant("mxfp4", N, K, packed, e).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    V = rng.standard_normal((K, rank))
    V[::32] = 0.0
    L = rng.standard_normal((N, rank)) @ V.T
    L *= 0.1 * np.exp2(float(e.min()) - 127) / np.abs(L).max()  # < 0.125 x the smallest scale
    W = (D + L).astype(np.float32)
    res = O.loftq(W, r=rank, s=1.0, iters=2, fmt="mxfp4")
    c, sc, _, _ = res["stored"]
    assert np.array_equal(c, packed) and np.array_equal(sc, e)
    resid = np.linalg.norm(W.astype(np.float64) - D - L)
    assert res["errs"][1] <= resid * (1 + 1e-9) and res["errs"][2] <= resid * (1 + 1e-9)
    assert np.allclose(res["B"] @ res["A"], L, rtol=0, atol=1e-4 * np.abs(L).max())


def test_loftq_alternation_is_monotone_with_an_exact_projection():
    # with rounding to a fixed grid as the quantiser, each sub-problem is solved exactly (rounding
    # is the nearest grid point element by element; the truncated SVD is the best rank-r fit), so
    # the objective ||W - Q - s B A|| can only fall from one iteration to the next -- and on a
    # generic weight the requantisation of iteration 2 strictly lowers it
    rng = np.random.default_rng(21)
    W = rng.standard_normal((30, 50))
    grid = lambda v: np.round(v * 2.0) / 2.0
    res = O.loftq(W, r=4, s=1.5, iters=6, quant=grid)
    e = res["errs"]
    assert all(e[t + 1] <= e[t] * (1 + 1e-12) for t in range(len(e) - 1))
    assert e[2] < e[1] * (1 - 1e-6)
    # the returned Q is the quantisation of W - s B A with the factors before the last SVD: it
    # is a grid point, and the final factors are the best rank-r fit of W - Q
    assert np.array_equal(res["Q"], grid(res["Q"]))
    S = np.linalg.svd(W - res["Q"], compute_uv=False)
    assert abs(e[-1] - np.sqrt((S[4:] ** 2).sum())) < 1e-9
