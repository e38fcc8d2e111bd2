"""Seeded LoftQ inputs whose answer is known in closed form (shared by the oracle pins and the GPU
tests).  The planted weight is built with the oracle's decode of seeded codes; the answer a test
checks -- the seeded codes and absmax, and the seeded low-rank matrix -- is fixed by the seeds,
not computed by either side."""
import numpy as np

from oracle import oracle as O


def planted(N, K, rank, seed, scale=1.0 / 64):
    """W = D + L with D an NF4 grid point and L of rank `rank` too small to move any code.

    D: every 64-block's column 0 holds code 15 (level +1) with a bf16-exact absmax in
    [0.01, 0.04], the other codes lie in 1..14 (|level| <= 0.723).  L = U V^T with V zero on
    column 0 of every block and max |L| = 0.01 * scale, below every block's absmax times `scale`.
    With scale <= 1/64, W / absmax stays within a quarter of the smallest NF4 gap of D / absmax,
    so quantising W gives D back (codes and absmax), and W - D = L up to W's fp32 rounding.
    Returns (W fp32 [N,K], packed codes [N,K/2], absmax [N,K/64], D float64, L float64)."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(1, 15, size=(N, K), dtype=np.uint8)
    codes[:, ::64] = 15
    a = rng.uniform(0.01, 0.04, size=(N, K // 64)).astype(np.float32)
    a = ((a.view(np.uint32) + 0x8000) & 0xFFFF0000).view(np.float32)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    D = (O.dequant("nf4", N, K, packed, a).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    U = rng.standard_normal((N, rank))
    V = rng.standard_normal((K, rank))
    V[::64] = 0.0
    L = U @ V.T
    L *= (0.01 * scale) / np.abs(L).max()
    W = (D + L).astype(np.float32)
    return W, packed, a, D, L
