"""GPU parity of the single-layer path (C ABI through the binding) against the fp64 oracle.

* Bit-exact decode: the kernels' dequant stage exported tile by tile (qlora_debug_dequant) and,
  stronger, the full fused GEMM driven with identity activations (X = I, B = 0 gives Y = deq(W)^T;
  dY = I, A = 0 gives dX = deq(W)) -- one exact product per output element, so every output bit
  must equal the oracle's decoded weight, including NVFP4's tensor scale applied in the epilogue.
* Tolerance parity of Y, T, dX, dA, dB on seeded problems that span several tiles with ragged
  tails in every dimension, all formats and ranks.
* Determinism, M = 0, and the bounded device wait.
"""
import numpy as np
import pytest
import torch

from bit_quantized_base_b200 import synth
from oracle import oracle as O
from gpu_util import GpuLayer, assert_close, bits, to_f64

pytestmark = pytest.mark.gpu


def _fold_signed_zero(b):
    """-0 (0x8000) -> +0: a GEMM output is a sum that includes +0 products, and IEEE addition
    of -0 and +0 is +0, so the identity GEMM cannot carry the sign of a zero weight (E2M1 code 8,
    or a negative level times a zero scale).  The decode itself keeps -0: see
    test_debug_dequant_bit_exact."""
    b = b.copy()
    b[b == 0x8000] = 0
    return b

FMTS = ["nf4", "mxfp4", "nvfp4"]


def _edge_weight(fmt, N, K, seed):
    """Random codes with scales that reach the decode's edge cases (subnormal products, overflow
    to inf, NaN scales, E4M3 subnormals and maximum)."""
    rng = np.random.default_rng(seed)
    if fmt == "nf4":
        pool = np.array([0.02, 1.0, 3.0e-39, 1e-41, 7.3e37, 2.5e38, 0.0, 1.234567e-5, 3.3e38],
                        np.float32)
    elif fmt == "mxfp4":
        pool = np.array([0, 1, 2, 60, 100, 126, 127, 128, 200, 252, 253, 254, 255])
    else:
        pool = np.array([0x00, 0x01, 0x07, 0x08, 0x30, 0x38, 0x40, 0x55, 0x7E, 0x7F, 0xB8, 0xFE])
    codes, scales, ts = synth.random_stored_weight(fmt, N, K, rng, scale_codes=pool)
    return codes, scales, (1.0 if ts is None else float(ts))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("transposed", [0, 1])
def test_debug_dequant_bit_exact(fmt, transposed):
    from bit_quantized_base_b200 import qlora as Q
    N, K = 272, 448          # ragged against both tilings (128 x 64 and 64 x 128)
    codes, scales, ts = _edge_weight(fmt, N, K, seed=17 + transposed)
    W = Q.weight_from_numpy(fmt, codes, scales, ts)
    out = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
    Q.qlora_debug_dequant(W, transposed, out)
    torch.cuda.synchronize()
    got = bits(out)
    ref = O.dequant(fmt, N, K, codes, scales, ts, with_tensor_scale=False)
    gnan = (got & 0x7FFF) > 0x7F80
    rnan = (ref & 0x7FFF) > 0x7F80
    assert np.array_equal(gnan, rnan), "NaN positions differ"
    mism = (got != ref) & ~rnan
    assert not mism.any(), f"{mism.sum()} decoded elements differ, first at {np.argwhere(mism)[0]}"


def _nf4dq_edge_weight(N, K, seed):
    """Random codes, every first-level E4M3 code (NaN and subnormals included) and second-level
    scales that make the absmax product overflow, underflow, vanish or go subnormal."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    c1 = rng.integers(0, 256, size=(N, K // 64), dtype=np.uint8)
    c1.reshape(-1)[:256] = np.arange(256, dtype=np.uint8)
    pool = np.array([1.0, 2.0 ** -20, 3.3e38, 0.0, 1.5, 7.1e-3, 1e-40, 4.2e35], np.float32)
    s2 = pool[rng.integers(0, len(pool), size=O.dq_groups(N, K))]
    return codes, c1, s2


@pytest.mark.parametrize("transposed", [0, 1])
def test_debug_dequant_nf4dq_bit_exact(transposed):
    from bit_quantized_base_b200 import qlora as Q
    N, K = 272, 448
    codes, c1, s2 = _nf4dq_edge_weight(N, K, seed=27 + transposed)
    W = Q.weight_from_numpy("nf4dq", codes, c1, None, scales2=s2)
    out = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
    Q.qlora_debug_dequant(W, transposed, out)
    torch.cuda.synchronize()
    got = bits(out)
    ref = O.dequant("nf4dq", N, K, codes, c1, scales2=s2)
    gnan = (got & 0x7FFF) > 0x7F80
    rnan = (ref & 0x7FFF) > 0x7F80
    assert np.array_equal(gnan, rnan), "NaN positions differ"
    mism = (got != ref) & ~rnan
    assert not mism.any(), f"{mism.sum()} decoded elements differ, first at {np.argwhere(mism)[0]}"


@pytest.mark.parametrize("dx", [False, True])
def test_fused_nf4dq_identity_is_bit_exact(dx):
    # X = I (forward) or dY = I (dX) with a zero LoRA term: every output is one decoded weight
    N, K = 208, 384
    rng = np.random.default_rng(8 + dx)
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    c1 = rng.integers(0x18, 0x70, size=(N, K // 64), dtype=np.uint8)
    s2 = rng.uniform(1e-4, 1e-2, size=O.dq_groups(N, K)).astype(np.float32)
    r = 8
    if not dx:
        M = K
        p = dict(fmt="nf4dq", M=M, N=N, K=K, r=r, s=2.0, codes=codes, scales=c1, tensor_scale=1.0,
                 scales2=s2, X=synth.to_bf16_bits(np.eye(K, dtype=np.float32)),
                 A=synth.to_bf16_bits(rng.standard_normal((r, K)).astype(np.float32)),
                 B=np.zeros((N, r), np.uint16), dY=np.zeros((M, N), np.uint16))
    else:
        M = N
        p = dict(fmt="nf4dq", M=M, N=N, K=K, r=r, s=2.0, codes=codes, scales=c1, tensor_scale=1.0,
                 scales2=s2, X=np.zeros((M, K), np.uint16), A=np.zeros((r, K), np.uint16),
                 B=synth.to_bf16_bits(rng.standard_normal((N, r)).astype(np.float32)),
                 dY=synth.to_bf16_bits(np.eye(N, dtype=np.float32)))
    g = GpuLayer(p)
    if not dx:
        out, _ = g.fwd()
    else:
        out, _, _ = g.bwd()
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = _fold_signed_zero(O.dequant("nf4dq", N, K, codes, c1, scales2=s2))
    if not dx:
        ref = ref.T
    assert np.array_equal(bits(out), ref), f"{(bits(out) != ref).sum()} elements differ"


@pytest.mark.parametrize("fmt", FMTS)
def test_fused_forward_identity_is_bit_exact(fmt):
    from bit_quantized_base_b200 import qlora as Q
    N, K = 272, 320
    rng = np.random.default_rng(5)
    codes, scales, ts = synth.random_stored_weight(fmt, N, K, rng)
    ts = 0.0123 if fmt == "nvfp4" else 1.0
    M = K
    p = dict(fmt=fmt, M=M, N=N, K=K, r=16, s=2.0, codes=codes, scales=scales, tensor_scale=ts,
             X=synth.to_bf16_bits(np.eye(K, dtype=np.float32)),
             A=synth.to_bf16_bits(rng.standard_normal((16, K)).astype(np.float32)),
             B=np.zeros((N, 16), np.uint16), dY=np.zeros((M, N), np.uint16))
    g = GpuLayer(p)
    Y, _ = g.fwd()
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = _fold_signed_zero(O.dequant(fmt, N, K, codes, scales, ts, with_tensor_scale=True).T)
    got = bits(Y)                                                            # [K, N] = deq(W)^T
    assert np.array_equal(got, ref), f"{(got != ref).sum()} elements differ"


@pytest.mark.parametrize("fmt", FMTS)
def test_fused_dx_identity_is_bit_exact(fmt):
    N, K = 208, 384
    rng = np.random.default_rng(6)
    codes, scales, _ = synth.random_stored_weight(fmt, N, K, rng)
    ts = 3.5 if fmt == "nvfp4" else 1.0
    M = N
    p = dict(fmt=fmt, M=M, N=N, K=K, r=8, s=2.0, codes=codes, scales=scales, tensor_scale=ts,
             X=np.zeros((M, K), np.uint16), A=np.zeros((8, K), np.uint16),
             B=synth.to_bf16_bits(rng.standard_normal((N, 8)).astype(np.float32)),
             dY=synth.to_bf16_bits(np.eye(N, dtype=np.float32)))
    g = GpuLayer(p)
    dX, dA, dB = g.bwd()
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = _fold_signed_zero(O.dequant(fmt, N, K, codes, scales, ts, with_tensor_scale=True))
    assert np.array_equal(bits(dX), ref), f"{(bits(dX) != ref).sum()} elements differ"


CASES = [
    # fmt, M, N, K, r
    ("nf4", 1, 128, 256, 16),
    ("nf4", 7, 272, 320, 8),
    ("nf4", 300, 400, 512, 64),
    ("mxfp4", 129, 384, 192, 32),
    ("mxfp4", 255, 144, 640, 16),
    ("nvfp4", 256, 256, 256, 16),
    ("nvfp4", 513, 528, 448, 64),
    # short batches (weight-streaming kernels): many output tiles, ranges that split tiles
    ("nf4", 16, 1024, 2048, 16),
    ("mxfp4", 64, 2048, 1024, 64),
    ("nvfp4", 200, 768, 4096, 8),
    ("nf4", 128, 4096, 512, 32),
    ("mxfp4", 2, 16, 64, 8),
    ("nvfp4", 96, 528, 704, 32),
    # 76 pair tiles on 74 pairs: the last wave's tiles run split in two 256-row tiles (fwd, dX)
    ("nf4", 1000, 9728, 128, 8),
    ("mxfp4", 1024, 128, 9728, 16),
    # NF4 with double-quantised absmax (tiled kernels at every batch size); K/64 = 5 or 19
    # blocks per row, so second-level groups of 256 straddle rows
    ("nf4dq", 5, 272, 320, 8),
    ("nf4dq", 300, 400, 1216, 64),
    ("nf4dq", 700, 1040, 576, 16),
]


@pytest.mark.parametrize("fmt,M,N,K,r", CASES)
def test_layer_parity(fmt, M, N, K, r):
    p = synth.small_layer(fmt, M, N, K, r, s=2.0, seed=M * 7 + N + K + r)
    g = GpuLayer(p)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(T)
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = O.layer(fmt, M, N, K, r, p["s"], p["codes"], p["scales"], p["tensor_scale"], p["X"],
                  p["A"], p["B"], p["dY"], scales2=p.get("scales2"))
    assert_close(to_f64(T), ref["T"], "T")
    assert_close(to_f64(Y), ref["Y"], "Y")
    assert_close(to_f64(dX), ref["dX"], "dX")
    assert_close(to_f64(dA), ref["dA"], "dA")
    assert_close(to_f64(dB), ref["dB"], "dB")


@pytest.mark.parametrize("fmt,M", [("nf4", 16), ("mxfp4", 64), ("nvfp4", 200)])
def test_workspace_without_partials_runs_the_tiled_kernels(fmt, M):
    # a workspace holding only the header, Zs, T, U and lora_down's cluster sums -- what one sized
    # for more than 256 rows offers a short batch -- has no room for the short-batch or streaming
    # kernels' split partials: the calls run the tiled kernels and still match the oracle
    from bit_quantized_base_b200 import qlora as Q
    N, K, r = 2064, 1216, 16
    p = synth.small_layer(fmt, M, N, K, r, s=2.0, seed=M + 5)
    g = GpuLayer(p)
    z = -(-M * r * 2 // 256) * 256
    need = 8192 + 3 * z + 8 * 128 * r * 4
    assert Q.qlora_workspace_size(Q.OP_BWD, g.W, M, r) > need
    g.ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    Q.qlora_workspace_init(g.ws)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(T)
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = O.layer(fmt, M, N, K, r, p["s"], p["codes"], p["scales"], p["tensor_scale"], p["X"],
                  p["A"], p["B"], p["dY"])
    for name, got in (("T", T), ("Y", Y), ("dX", dX), ("dA", dA), ("dB", dB)):
        assert_close(to_f64(got), ref[name], name)


def test_backward_recomputes_T_and_skips_dx():
    p = synth.small_layer("mxfp4", 200, 256, 384, 16, seed=3)
    g = GpuLayer(p)
    dX, dA, dB = g.bwd(T=None, want_dx=False)
    torch.cuda.synchronize()
    ref = O.layer("mxfp4", 200, 256, 384, 16, p["s"], p["codes"], p["scales"], 1.0, p["X"],
                  p["A"], p["B"], p["dY"], want=("dA", "dB"))
    assert dX is None
    assert_close(to_f64(dA), ref["dA"], "dA")
    assert_close(to_f64(dB), ref["dB"], "dB")


@pytest.mark.parametrize("M", [200, 1000])   # streaming and pair paths
def test_backward_recompute_matches_saved_T(M):
    # T recomputed in the backward pass uses the forward's plan: same T, bit for bit, so the
    # gradients equal those computed from the saved T
    p = synth.small_layer("nf4", M, 768, 1024, 32, seed=4)
    g = GpuLayer(p)
    Y, T = g.fwd()
    saved = g.bwd(T)
    recomputed = g.bwd(None)
    torch.cuda.synchronize()
    for a, b in zip(saved, recomputed):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_deterministic_reruns():
    p = synth.small_layer("nf4", 1000, 512, 1024, 32, seed=9)
    g = GpuLayer(p)
    Y1, T1 = g.fwd()
    r1 = g.bwd(T1)
    Y2, T2 = g.fwd()
    r2 = g.bwd(T2)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    for a, b in zip(r1, r2):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_pair_ticket_from_any_start():
    # The pair kernel draws pair ranks from a ticket in the workspace header (32-bit word 1) that
    # wraps at the pair count: npairs draws from any start below it are a permutation of the
    # ranks, so results do not depend on where the ticket stands, and every launch leaves it
    # where it found it.
    p = synth.small_layer("mxfp4", 1300, 2048, 1024, 16, seed=21)   # pair path
    g = GpuLayer(p)
    Y0, T0 = g.fwd()
    r0 = g.bwd(T0)
    torch.cuda.synchronize()
    ticket = g.ws[4:8].view(torch.int32)
    assert int(ticket.item()) == 0
    ticket.fill_(3)
    Y1, T1 = g.fwd()
    r1 = g.bwd(T1)
    torch.cuda.synchronize()
    assert g.status() == 0
    assert int(ticket.item()) == 3
    assert torch.equal(Y0.view(torch.int16), Y1.view(torch.int16))
    for a, b in zip(r0, r1):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("fmt", FMTS)
def test_decode_rate_measurement(fmt):
    # the benchmark's decode ceiling: a positive rate of the order of the ALU's width
    from bit_quantized_base_b200 import qlora as Q
    v = Q.qlora_debug_decode_rate(fmt, 200)
    assert 2.0 < v < 200.0, v


def test_step0_init_on_gpu():
    # B = 0 -> dA == 0 exactly and Y equals the base product ("Initialization matters")
    p = synth.small_layer("nf4", 64, 128, 256, 16, seed=2)
    p["B"] = np.zeros_like(p["B"])
    g = GpuLayer(p)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(T)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA.float()) == 0
    assert torch.count_nonzero(dB.float()) > 0


def test_empty_batch_zeroes_gradients():
    from bit_quantized_base_b200 import qlora as Q
    p = synth.small_layer("nvfp4", 4, 128, 256, 16, seed=1)
    g = GpuLayer(p)
    dA = torch.full((16, 256), 1.0, dtype=torch.bfloat16, device="cuda")
    dB = torch.full((128, 16), 1.0, dtype=torch.bfloat16, device="cuda")
    Q.qlora_linear_bwd(g.W, g.X, g.A, g.B, None, g.dY, None, dA, dB, 0, 16, 2.0, g.ws)
    Q.qlora_linear_fwd(g.W, g.X, g.A, g.B, g.X, None, 0, 16, 2.0, g.ws)   # M = 0: no-op
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA.float()) == 0 and torch.count_nonzero(dB.float()) == 0


def test_bounded_wait_reports_timeout():
    from bit_quantized_base_b200 import qlora as Q
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    Q.qlora_workspace_init(ws)
    assert Q.qlora_get_device_status(ws) == 0
    Q.qlora_debug_wait_timeout(ws, 2000)        # ~2 ms: nothing arrives, the wait gives up
    assert Q.qlora_get_device_status(ws) == 5   # QLORA_ERR_DEVICE_TIMEOUT, context still usable
    Q.qlora_workspace_init(ws)
    assert Q.qlora_get_device_status(ws) == 0
    x = torch.ones(16, device="cuda")
    assert float(x.sum()) == 16.0
