"""GPU parity of the short-batch kernels (batches of at most 64 rows; C ABI through the binding).

* Bit-exact decode: the short-batch decoders exported on their own (qlora_debug_dequant modes 2
  and 3) on weights whose scales reach every edge case, against the oracle's decode (NVFP4 times
  2^-8, the factor those kernels carry); and the whole forward and dX kernels driven with windows
  of the identity (X rows = rows of I, B = 0 gives Y = rows of deq(W)^T; dY rows = rows of I, A = 0
  gives dX = rows of deq(W)), on shapes where the tiles split between CTAs, so every output bit
  must equal a decoded weight after the partial reduction and the NVFP4 tensor scale.
* Tolerance parity of Y, T, dX, dA, dB at 1..64 rows with ragged tails in every dimension.
* Determinism, and the per-tile arrival counters left at zero after every launch.
"""
import numpy as np
import pytest
import torch

from bit_quantized_base_b200 import synth
from oracle import oracle as O
from gpu_util import GpuLayer, assert_close, bits, to_f64
from test_gpu_layer import FMTS, _edge_weight, _fold_signed_zero

pytestmark = pytest.mark.gpu


def _times_2_pow(b, p):
    """bf16 bit patterns times 2^p (exact for the normal values here; NaN, inf and zero kept)."""
    f = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64) * (2.0 ** p)
    out = (f.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    nan = (b & 0x7FFF) > 0x7F80
    out[nan] = b[nan]
    return out


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("mode", [2, 3], ids=["regs", "smem"])
def test_short_decoder_bit_exact(fmt, mode):
    from bit_quantized_base_b200 import qlora as Q
    N, K = 272, 448
    codes, scales, ts = _edge_weight(fmt, N, K, seed=31 + mode)
    W = Q.weight_from_numpy(fmt, codes, scales, ts)
    out = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
    Q.qlora_debug_dequant(W, mode, out)
    torch.cuda.synchronize()
    got = bits(out)
    ref = O.dequant(fmt, N, K, codes, scales, ts, with_tensor_scale=False)
    if fmt == "nvfp4":
        ref = _times_2_pow(ref, -8)
    gnan = (got & 0x7FFF) > 0x7F80
    rnan = (ref & 0x7FFF) > 0x7F80
    assert np.array_equal(gnan, rnan), "NaN positions differ"
    mism = (got != ref) & ~rnan
    assert not mism.any(), f"{mism.sum()} decoded elements differ, first at {np.argwhere(mism)[0]}"


@pytest.mark.parametrize("fmt", FMTS)
def test_short_forward_identity_is_bit_exact(fmt):
    # 272 x 320: 3 tiles of 128 weight rows (the last ragged) x 6 steps, cut into ranges of 2
    # steps, so every tile is split between 3 CTAs and reduced from partials
    N, K, M, r = 272, 320, 64, 16
    rng = np.random.default_rng(5)
    codes, scales, _ = synth.random_stored_weight(fmt, N, K, rng)
    ts = 0.0123 if fmt == "nvfp4" else 1.0
    ref = _fold_signed_zero(O.dequant(fmt, N, K, codes, scales, ts, with_tensor_scale=True).T)
    eye = np.eye(K, dtype=np.float32)
    for k0 in range(0, K, M):
        p = dict(fmt=fmt, M=M, N=N, K=K, r=r, s=2.0, codes=codes, scales=scales, tensor_scale=ts,
                 X=synth.to_bf16_bits(eye[k0:k0 + M]),
                 A=synth.to_bf16_bits(rng.standard_normal((r, K)).astype(np.float32)),
                 B=np.zeros((N, r), np.uint16), dY=np.zeros((M, N), np.uint16))
        g = GpuLayer(p)
        Y, _ = g.fwd()
        torch.cuda.synchronize()
        assert g.status() == 0
        got = bits(Y)
        assert np.array_equal(got, ref[k0:k0 + M]), f"rows {k0}+: {(got != ref[k0:k0 + M]).sum()} differ"


@pytest.mark.parametrize("fmt", FMTS)
def test_short_dx_identity_is_bit_exact(fmt):
    # contraction over N = 208 (3 full steps of 64 weight rows and a ragged one of 16), output
    # tiles of 256 columns over K = 384 (one full, one of 128)
    N, K, M, r = 208, 384, 64, 8
    rng = np.random.default_rng(6)
    codes, scales, _ = synth.random_stored_weight(fmt, N, K, rng)
    ts = 3.5 if fmt == "nvfp4" else 1.0
    ref = _fold_signed_zero(O.dequant(fmt, N, K, codes, scales, ts, with_tensor_scale=True))
    eye = np.eye(N, dtype=np.float32)
    for n0 in range(0, N, M):
        rows = min(M, N - n0)
        p = dict(fmt=fmt, M=rows, N=N, K=K, r=r, s=2.0, codes=codes, scales=scales, tensor_scale=ts,
                 X=np.zeros((rows, K), np.uint16), A=np.zeros((r, K), np.uint16),
                 B=synth.to_bf16_bits(rng.standard_normal((N, r)).astype(np.float32)),
                 dY=synth.to_bf16_bits(eye[n0:n0 + rows]))
        g = GpuLayer(p)
        dX, _, _ = g.bwd()
        torch.cuda.synchronize()
        assert g.status() == 0
        got = bits(dX)
        assert np.array_equal(got, ref[n0:n0 + rows]), f"rows {n0}+: {(got != ref[n0:n0 + rows]).sum()} differ"


SHORT_CASES = [
    # fmt, M, N, K, r
    ("nf4", 1, 144, 256, 16),
    ("mxfp4", 3, 272, 320, 8),
    ("nvfp4", 16, 400, 512, 64),
    ("nf4", 33, 528, 704, 32),
    ("mxfp4", 48, 1040, 1216, 16),
    ("nvfp4", 64, 2064, 960, 8),
    ("nf4", 64, 4096, 2048, 64),
    ("nvfp4", 7, 16, 4096, 16),      # one weight tile, a long contraction: every CTA on one tile
    ("mxfp4", 20, 12288, 64, 32),    # one contraction step per tile: no tile is split
]


@pytest.mark.parametrize("fmt,M,N,K,r", SHORT_CASES)
def test_short_layer_parity(fmt, M, N, K, r):
    p = synth.small_layer(fmt, M, N, K, r, s=2.0, seed=M * 11 + N + K + r)
    g = GpuLayer(p)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(T)
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = O.layer(fmt, M, N, K, r, p["s"], p["codes"], p["scales"], p["tensor_scale"], p["X"],
                  p["A"], p["B"], p["dY"])
    assert_close(to_f64(T), ref["T"], "T")
    assert_close(to_f64(Y), ref["Y"], "Y")
    assert_close(to_f64(dX), ref["dX"], "dX")
    assert_close(to_f64(dA), ref["dA"], "dA")
    assert_close(to_f64(dB), ref["dB"], "dB")
    # every launch leaves the arrival counters (workspace bytes 64..191: lora_down's multi-cluster
    # U; 256..8191: the short-batch kernels' tiles) at zero
    assert int(torch.count_nonzero(g.ws[64:192])) == 0
    assert int(torch.count_nonzero(g.ws[256:8192])) == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_short_deterministic_and_recompute(fmt):
    p = synth.small_layer(fmt, 24, 1040, 1216, 32, seed=77)
    g = GpuLayer(p)
    Y1, T1 = g.fwd()
    r1 = g.bwd(T1)
    Y2, T2 = g.fwd()
    r2 = g.bwd(None)              # T recomputed with the forward's plan
    torch.cuda.synchronize()
    assert g.status() == 0
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    assert torch.equal(T1.view(torch.int16), T2.view(torch.int16))
    for a, b in zip(r1, r2):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("fmt", FMTS)
def test_short_long_ranges_repeat_bitwise(fmt):
    # 16 rows over a 16384 x 2048 weight: the forward's 128 tiles x 9 steps and dX's 8 tiles x
    # 129 steps give each CTA 8 to 9 iterations, so every code slot and operand stage is refilled
    # many times; repeated launches must agree bit for bit and match the oracle
    M, N, K, r = 16, 16384, 2048, 16
    p = synth.small_layer(fmt, M, N, K, r, s=2.0, seed=404)
    g = GpuLayer(p)
    runs = []
    for _ in range(4):
        Y, T = g.fwd()
        dX, dA, dB = g.bwd(T)
        torch.cuda.synchronize()
        runs.append((bits(Y), bits(dX), bits(dA), bits(dB)))
    assert g.status() == 0
    for k, name in enumerate(("Y", "dX", "dA", "dB")):
        for rr in runs[1:]:
            assert np.array_equal(runs[0][k], rr[k]), f"{name} differs between launches"
    ref = O.layer(fmt, M, N, K, r, p["s"], p["codes"], p["scales"], p["tensor_scale"], p["X"],
                  p["A"], p["B"], p["dY"], want=("Y", "dX"))
    assert_close(to_f64(Y), ref["Y"], "Y")
    assert_close(to_f64(dX), ref["dX"], "dX")
