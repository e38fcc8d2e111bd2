"""GPU LoftQ initialisation against the oracle and against planted answers.

"Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §4: alternate Q = quantise(W - s B A) and
s B A = the rank-r truncated SVD of W - Q.  The GPU's SVD is randomized subspace iteration in
fp32, the oracle's an exact fp64 SVD, so:
  - what is unique is compared exactly or to fp32 precision: the first quantisation (bit-exact),
    errs[0], and -- on a planted weight whose residual has rank <= l, where the truncated SVD is
    exact for both -- the recovered codes (bit-exact), the error (~0) and s B A (to bf16);
  - on a generic weight, where the top-r subspace is barely separated from the rest of the
    spectrum, the errors (1 %) and singular values (2 %, Ritz values as lower bounds) are
    compared within stated tolerances and the rest is checked for validity (errors below the
    plain QLoRA start, reproducible bits)."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from loftq_cases import planted

pytestmark = pytest.mark.gpu


def _Q():
    from bit_quantized_base_b200 import qlora as Q
    return Q


def _wide(t):
    return t.float().cpu().numpy().astype(np.float64)


def _run(W, fmt, r, s, iters, power_iters=4, seed=0):
    Q = _Q()
    N, K = W.shape
    Wq = Q.empty_weight(fmt, N, K)
    Wd = torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda()
    A, B, errs, sig = Q.qlora_loftq(Wd, Wq, r, s, iters=iters, power_iters=power_iters, seed=seed)
    torch.cuda.synchronize()
    return Wq, A, B, errs.cpu().numpy().astype(np.float64), sig.cpu().numpy().astype(np.float64)


def _codes(Wq):
    return Wq.codes.cpu().numpy(), Wq.scales.cpu().numpy()


@pytest.mark.parametrize("N,K,rank,r", [(64, 512, 2, 2), (48, 704, 3, 8), (16, 128, 1, 4)])
def test_loftq_planted_recovered(N, K, rank, r):
    # a residual of rank <= l: the randomized SVD is exact, and LoftQ recovers W after one step
    W, packed, a, D, L = planted(N, K, rank, 11)
    s = 2.0
    Wq, A, B, errs, sig = _run(W, "nf4", r, s, iters=2)
    codes, scales = _codes(Wq)
    assert np.array_equal(codes, packed) and np.array_equal(scales.view(np.uint32), a.view(np.uint32))
    ref = O.loftq(W, r=r, s=s, iters=2, fmt="nf4")
    assert abs(errs[0] - ref["errs"][0]) <= 1e-6 * ref["errs"][0]
    assert errs[1] <= 1e-4 * errs[0] and errs[2] <= 1e-4 * errs[0]
    BA = s * _wide(B) @ _wide(A)
    assert np.abs(BA - L).max() <= 1e-2 * np.abs(L).max()
    assert np.allclose(sig[:rank], ref["sigma"][:rank], rtol=1e-4)
    assert np.all(sig[rank:] <= 1e-4 * sig[0])


@pytest.mark.parametrize("fmt", ["nf4", "nf4dq", "mxfp4", "nvfp4"])
def test_loftq_first_quantisation_bit_exact(fmt):
    # with one iteration Q is quantise(W): the encoder rules, bit for bit
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((96, 640)) * 0.02).astype(np.float32)
    Wq, _, _, errs, _ = _run(W, fmt, 8, 1.0, iters=1)
    c, sc, ts, s2 = O.encode(fmt, W)
    codes, scales = _codes(Wq)
    assert np.array_equal(codes, c)
    assert np.array_equal(scales.view(np.uint8), np.ascontiguousarray(sc).view(np.uint8))
    if fmt == "nvfp4":
        assert float(Wq.tensor_scale.cpu()[0]) == ts
    if fmt == "nf4dq":
        assert np.array_equal(Wq.scales2.cpu().numpy(), s2)
    ref = O.loftq(W, r=8, s=1.0, iters=1, fmt=fmt)
    assert abs(errs[0] - ref["errs"][0]) <= 1e-6 * ref["errs"][0]


def test_loftq_generic_against_oracle():
    # N(0, 0.02) weight: a flat residual spectrum; errors within 1 % of the exact-SVD oracle,
    # every error below the plain QLoRA start, and the run reproducible bitwise
    rng = np.random.default_rng(6)
    N, K, r, s, iters = 256, 512, 16, 2.0, 5
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    Wq, A, B, errs, sig = _run(W, "nf4", r, s, iters=iters, power_iters=6)
    ref = O.loftq(W, r=r, s=s, iters=iters, fmt="nf4")
    assert abs(errs[0] - ref["errs"][0]) <= 1e-6 * ref["errs"][0]
    for t in range(1, iters + 1):
        assert errs[t] < errs[0]
        assert abs(errs[t] - ref["errs"][t]) <= 1e-2 * ref["errs"][t], (t, errs, ref["errs"])
    # the last residuals differ (the quantisations after the first follow each side's own
    # factors), so their singular values agree only loosely ...
    assert np.allclose(sig, ref["sigma"], rtol=3e-2)
    # ... while the first residual is the same matrix on both sides (Q_1 is bit-exact): there the
    # Ritz values are lower bounds of the exact singular values, and on a flat spectrum converge
    # slowly at the subspace's edge (6 power iterations: a numpy model of the same iteration
    # leaves 1.1 % on the 16th), faster at the top
    _, _, _, _, sig1 = _run(W, "nf4", r, s, iters=1, power_iters=6)
    ref1 = O.loftq(W, r=r, s=s, iters=1, fmt="nf4")["sigma"]
    assert np.all(sig1 <= ref1 * (1 + 1e-5))
    assert np.all(sig1 >= ref1 * (1 - 2e-2))
    assert np.allclose(sig1[:4], ref1[:4], rtol=5e-3)
    # the returned factors are the ones the last error describes (bf16 rounding aside)
    codes, scales = _codes(Wq)
    deq = O.dequant("nf4", N, K, codes, scales)
    deq = (deq.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    e = np.linalg.norm(W.astype(np.float64) - deq - s * _wide(B) @ _wide(A))
    assert abs(e - errs[-1]) <= 2e-3 * errs[-1]
    # B and A carry sqrt(sigma / s) each: column norms of B equal row norms of A
    assert np.allclose(np.linalg.norm(_wide(B), axis=0), np.linalg.norm(_wide(A), axis=1), rtol=1e-2)
    Wq2, A2, B2, errs2, _ = _run(W, "nf4", r, s, iters=iters, power_iters=6)
    assert np.array_equal(errs, errs2)
    assert torch.equal(A, A2) and torch.equal(B, B2) and torch.equal(Wq.codes, Wq2.codes)


def test_loftq_full_size_planted():
    # the Llama-3-8B-shaped up-projection (N=14336, K=4096) at rank 64, planted rank 8
    N, K, rank, r, s = 14336, 4096, 8, 64, 2.0
    W, packed, a, D, L = planted(N, K, rank, 12)
    Wq, A, B, errs, sig = _run(W, "nf4", r, s, iters=2, power_iters=2)
    codes, scales = _codes(Wq)
    assert np.array_equal(codes, packed) and np.array_equal(scales.view(np.uint32), a.view(np.uint32))
    e0 = np.linalg.norm(W.astype(np.float64) - D)
    assert abs(errs[0] - e0) <= 1e-5 * e0
    assert errs[2] <= 1e-4 * errs[0]
    rows = np.r_[0:8, 7000:7008, N - 8:N]
    BA = s * _wide(B)[rows] @ _wide(A)
    assert np.abs(BA - L[rows]).max() <= 1e-2 * np.abs(L).max()
    assert np.all(sig[rank:] <= 1e-4 * sig[0])


def test_loftq_rejects_bad_arguments():
    Q = _Q()
    W = torch.zeros((32, 128), dtype=torch.float32, device="cuda")
    Wq = Q.empty_weight("nf4", 32, 128)
    with pytest.raises(RuntimeError):
        Q.qlora_loftq(W, Wq, 0, 1.0)                 # r = 0
    with pytest.raises(RuntimeError):
        Q.qlora_loftq(W, Wq, 97, 1.0)                # r above the subspace limit
    with pytest.raises(RuntimeError):
        Q.qlora_loftq(W, Wq, 4, -1.0)                # scale <= 0
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(RuntimeError):
        Q.qlora_loftq(W, Wq, 4, 1.0, work=small)     # short workspace
    assert Q.qlora_loftq_workspace_size(32, 128, 0) == 0
