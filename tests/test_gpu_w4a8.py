"""GPU parity of the opt-in native block-scaled forward for MXFP4 weights (W4A8;
"Quantized weights, full precision", "LoRA operations and quantization"; "Fine-Tuning 4-Bit
Models", "Case 3"), through the C ABI.

* The MXFP8 activation quantiser is bit-exact against the oracle's rule (codes and scales) on
  random blocks and on blocks that reach its edge cases: all zeros, bf16 subnormals only, a block
  whose small elements round to zero under a large shared exponent (no signed zero), saturation
  at 448, the largest finite bf16.
* Y of the W4A8 forward against oracle.layer_w4a8_forward (the fp64 product of the quantised X and
  the exact E2M1 x E8M0 weight, plus s T B^T), T against the oracle's T, with the same tolerance
  as the bf16 path: both sides multiply the same quantised values exactly, so only fp32
  accumulation and the bf16 output and Zs roundings differ.  Ragged shapes in M and N (tiles of
  128 x 192), K in multiples of 128; repeated launches bitwise equal.
* The 28672 x 8192 MXFP4 gate-proj at M = 8192 on sampled rows.
"""
import numpy as np
import pytest
import torch

from bit_quantized_base_b200 import synth
from oracle import oracle as O
from gpu_util import assert_close, bits, to_f64

pytestmark = pytest.mark.gpu


def _wide(h):
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _quant_gpu(Xb):
    from bit_quantized_base_b200 import qlora as Q
    M, K = Xb.shape
    X = Q.bf16_from_bits(Xb)
    codes = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((M, K // 32), dtype=torch.uint8, device="cuda")
    Q.qlora_mxfp8_quantize(X, M, K, codes, scales)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def test_mxfp8_quantizer_bit_exact():
    rng = np.random.default_rng(8)
    M, K = 48, 1024
    x = (rng.standard_normal((M, K)) * np.exp2(rng.integers(-20, 20, size=(M, 1)))).astype(np.float32)
    Xb = synth.to_bf16_bits(x)
    Xb[0, 0:32] = 0                                           # all-zero block
    Xb[0, 32:64] = rng.integers(1, 0x80, size=32)             # positive bf16 subnormals only
    Xb[0, 64:96] = rng.integers(0x8001, 0x8080, size=32)      # negative subnormals
    Xb[1, 0:32] = synth.to_bf16_bits(np.float32(2.0 ** 60) * np.linspace(-1e-6, 1e-6, 32).astype(np.float32))
    Xb[1, 0] = 0x5D80                                          # 2^60: the rest of the block rounds to 0
    Xb[1, 32:64] = synth.to_bf16_bits(np.float32(1.99) * np.ones(32, np.float32))   # saturates at 448
    Xb[1, 64:96] = 0x7F7F                                      # the largest finite bf16
    Xb[1, 96:128] = 0xFF7F
    Xb[2, 0:32] = synth.to_bf16_bits(np.float32(-0.0) * np.ones(32, np.float32))
    codes, scales = _quant_gpu(Xb)
    rc, rs = O.mxfp8_quantize(_wide(Xb))
    assert np.array_equal(scales, rs), f"{(scales != rs).sum()} scales differ"
    d = codes != rc
    assert not d.any(), f"{d.sum()} codes differ, first at {np.argwhere(d)[0]}: " \
        f"{codes[tuple(np.argwhere(d)[0])]:#x} vs {rc[tuple(np.argwhere(d)[0])]:#x}"
    assert not np.any(codes == 0x80)                           # no signed zero


def _run_w4a8(p, T_out=True):
    from bit_quantized_base_b200 import qlora as Q
    M, N, K, r = p["M"], p["N"], p["K"], p["r"]
    W = Q.weight_from_numpy("mxfp4", p["codes"], p["scales"], None)
    X, A, B = (Q.bf16_from_bits(p[k]) for k in ("X", "A", "B"))
    ws = Q.alloc_workspace(Q.OP_FWD_W4A8, W, M, r)
    Q.qlora_workspace_init(ws)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((M, r), dtype=torch.bfloat16, device="cuda") if T_out else None
    Q.qlora_linear_fwd_w4a8(W, X, A, B, Y, T, M, r, p["s"], ws)
    return Q, W, X, A, B, Y, T, ws


CASES = [
    # M, N, K, r: one row; ragged tiles in M (128) and N (192); a single weight tile with a long
    # contraction; several tiles per CTA
    (1, 192, 128, 16),
    (100, 400, 256, 8),
    (130, 208, 384, 32),
    (257, 592, 512, 64),
    (64, 16, 1024, 16),
    (300, 1024, 2048, 16),
]


@pytest.mark.parametrize("M,N,K,r", CASES)
def test_w4a8_forward_parity(M, N, K, r):
    p = synth.small_layer("mxfp4", M, N, K, r, s=2.0, seed=M + N + K + r)
    Q, W, X, A, B, Y, T, ws = _run_w4a8(p)
    torch.cuda.synchronize()
    assert Q.qlora_get_device_status(ws) == 0
    ref = O.layer_w4a8_forward("mxfp4", M, N, K, r, p["s"], p["codes"], p["scales"], None, p["X"],
                               p["A"], p["B"])
    assert_close(to_f64(Y), ref, "Y")
    refT = O.layer("mxfp4", M, N, K, r, p["s"], p["codes"], p["scales"], 1.0, p["X"], p["A"],
                   p["B"], want=("T",))["T"]
    assert_close(to_f64(T), refT, "T")


def test_w4a8_forward_deterministic_and_differs_from_bf16_by_the_quantisation():
    from bit_quantized_base_b200 import qlora as Q
    M, N, K, r = 200, 592, 1024, 16
    p = synth.small_layer("mxfp4", M, N, K, r, s=2.0, seed=12)
    Q, W, X, A, B, Y1, T1, ws = _run_w4a8(p)
    Y2 = torch.empty_like(Y1)
    Q.qlora_linear_fwd_w4a8(W, X, A, B, Y2, None, M, r, p["s"], ws)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    # against the bf16 forward: the gap is the activation quantisation, a few percent, not more
    wsb = Q.alloc_workspace(Q.OP_FWD, W, M, r)
    Q.qlora_workspace_init(wsb)
    Yb = torch.empty_like(Y1)
    Q.qlora_linear_fwd(W, X, A, B, Yb, None, M, r, p["s"], wsb)
    torch.cuda.synchronize()
    a, b = to_f64(Y1), to_f64(Yb)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 1e-3 < rel < 0.08, rel


def test_w4a8_full_size_gate_proj_sampled_rows():
    p = synth.layer_inputs("llama3_70b_gate_mxfp4", 0)
    M, N, K, r = p["M"], p["N"], p["K"], p["r"]
    Q, W, X, A, B, Y, T, ws = _run_w4a8(p)
    torch.cuda.synchronize()
    assert Q.qlora_get_device_status(ws) == 0
    rows = np.unique(np.concatenate([[0, 1, 127, 128, M - 1], np.random.default_rng(3).integers(0, M, 11)]))
    ref = O.layer_w4a8_forward("mxfp4", len(rows), N, K, r, p["s"], p["codes"], p["scales"], None,
                               p["X"][rows], p["A"], p["B"])
    got = to_f64(Y[torch.from_numpy(rows).cuda()])
    assert_close(got, ref, "Y rows")
