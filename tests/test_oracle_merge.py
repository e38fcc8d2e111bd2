"""Pins of the oracle's adapter merge (the value requantisation starts from) on the CPU.

"Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §2 "Deployment: keep or merge": merging adds
the scaled low-rank product to the dequantised base.  Each pin fixes the result by other
means than the oracle's own loop: an adapter of zero leaves the decode, an adapter built to cancel
the base gives exact zeros, and numpy's float64 matmul (a different summation order) agrees to one
fp32 ulp."""
import numpy as np
import pytest

from oracle import oracle as O
from bit_quantized_base_b200 import synth


def _bf16(x):
    x = np.asarray(x, np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _wide(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _weight(fmt, N, K, seed):
    d = synth.small_layer(fmt, 16, N, K, 8, seed=seed)
    return d["codes"], d["scales"], d.get("tensor_scale", 1.0), d.get("scales2")


@pytest.mark.parametrize("fmt", ["nf4", "nf4dq", "mxfp4", "nvfp4"])
def test_merge_zero_adapter_is_decode(fmt):
    N, K, r = 32, 256, 5
    codes, scales, ts, s2 = _weight(fmt, N, K, 3)
    A = _bf16(np.random.default_rng(1).standard_normal((r, K)))
    B = np.zeros((N, r), np.uint16)
    m = O.merge(fmt, N, K, codes, scales, ts, A, B, 2.0, scales2=s2)
    assert np.array_equal(m, _wide(O.dequant(fmt, N, K, codes, scales, ts, scales2=s2)).astype(np.float32))


def test_merge_cancelling_adapter_gives_zero():
    # every row of the MXFP4 weight decodes to the same row w (codes repeated, scale 2^0), and
    # B A = -w / s with B = 1, A = -w / 2 (exact in bf16): the merge is exactly 0 everywhere
    N, K, s = 16, 128, 2.0
    rng = np.random.default_rng(5)
    row = rng.integers(0, 256, size=K // 2, dtype=np.uint8)
    codes = np.tile(row, (N, 1))
    scales = np.full((N, K // 32), 127, np.uint8)
    w = _wide(O.dequant("mxfp4", N, K, codes, scales))
    assert np.all(w == w[0])
    A = _bf16((-w[0] / s)[None, :])
    assert np.array_equal(_wide(A)[0], -w[0] / s)
    B = _bf16(np.ones((N, 1)))
    m = O.merge("mxfp4", N, K, codes, scales, 1.0, A, B, s)
    assert np.all(m == 0.0)
    # the same adapter with the opposite sign doubles the weight, exactly
    m2 = O.merge("mxfp4", N, K, codes, scales, 1.0, A, _bf16(-np.ones((N, 1))), s)
    assert np.array_equal(m2.astype(np.float64), 2.0 * w)


@pytest.mark.parametrize("fmt", ["nf4", "nvfp4"])
def test_merge_matches_float64_matmul(fmt):
    N, K, r, s = 48, 192, 7, 0.375
    codes, scales, ts, s2 = _weight(fmt, N, K, 9)
    rng = np.random.default_rng(2)
    A = _bf16(rng.standard_normal((r, K)) * 0.05)
    B = _bf16(rng.standard_normal((N, r)) * 0.05)
    m = O.merge(fmt, N, K, codes, scales, ts, A, B, s, scales2=s2).astype(np.float64)
    want = _wide(O.dequant(fmt, N, K, codes, scales, ts, scales2=s2)) + s * (_wide(B) @ _wide(A))
    ulp = np.spacing(np.abs(want).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(m - want) <= ulp)
    # the adapter is visible: a transposed or dropped term would move most elements by far more
    assert np.mean(np.abs(m - _wide(O.dequant(fmt, N, K, codes, scales, ts, scales2=s2))) > 0) > 0.9
