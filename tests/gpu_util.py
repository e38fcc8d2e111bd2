"""Shared helpers of the GPU parity tests: upload seeded inputs, run the library through its C ABI
(the Python binding), and compare against the oracle with the stated tolerance."""
import os

import numpy as np
import torch

from bit_quantized_base_b200 import synth

# Output tolerance for bf16 outputs against the fp64 oracle: relative Frobenius error and
# max-abs error relative to the largest reference magnitude.  With QLORA_PRINT_ERRORS=1 every
# comparison prints its two errors (run pytest with -s to see them).
REL_FRO = 4e-3
MAX_ABS_REL = 2e-2


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def assert_close(got, ref, name, rel_fro=REL_FRO, max_abs_rel=MAX_ABS_REL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    nref = np.linalg.norm(ref)
    err = np.linalg.norm(got - ref)
    mx = np.abs(ref).max() if ref.size else 0.0
    if nref == 0.0:
        assert err == 0.0, f"{name}: expected exact zeros, |err|={err}"
        return
    if os.environ.get("QLORA_PRINT_ERRORS"):
        print(f"[parity] {os.environ.get('PYTEST_CURRENT_TEST', '').split(' ')[0]} {name}: "
              f"rel_fro={err / nref:.3e} max_abs_rel={np.abs(got - ref).max() / mx:.3e}")
    assert err / nref <= rel_fro, f"{name}: rel Frobenius error {err / nref:.3e} > {rel_fro}"
    assert np.abs(got - ref).max() <= max_abs_rel * mx, \
        f"{name}: max abs error {np.abs(got - ref).max():.3e} > {max_abs_rel} * {mx:.3e}"


class GpuLayer:
    """Device copies of one layer problem (dict from synth.small_layer / layer_inputs)."""

    def __init__(self, p, device="cuda"):
        from bit_quantized_base_b200 import qlora as Q
        self.Q = Q
        self.p = p
        self.W = Q.weight_from_numpy(p["fmt"], p["codes"], p["scales"], p["tensor_scale"], device,
                                     scales2=p.get("scales2"))
        self.X = Q.bf16_from_bits(p["X"], device)
        self.A = Q.bf16_from_bits(p["A"], device)
        self.B = Q.bf16_from_bits(p["B"], device)
        self.dY = Q.bf16_from_bits(p["dY"], device)
        M, N, K, r = p["M"], p["N"], p["K"], p["r"]
        self.M, self.N, self.K, self.r = M, N, K, r
        self.ws = Q.alloc_workspace(Q.OP_BWD, self.W, M, r)
        Q.qlora_workspace_init(self.ws)

    def fwd(self):
        Q, M, N, r = self.Q, self.M, self.N, self.r
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        T = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        Q.qlora_linear_fwd(self.W, self.X, self.A, self.B, Y, T, M, r, self.p["s"], self.ws)
        return Y, T

    def bwd(self, T=None, want_dx=True):
        Q, M, N, K, r = self.Q, self.M, self.N, self.K, self.r
        dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda") if want_dx else None
        dA = torch.full((r, K), float("nan"), dtype=torch.bfloat16, device="cuda")
        dB = torch.full((N, r), float("nan"), dtype=torch.bfloat16, device="cuda")
        Q.qlora_linear_bwd(self.W, self.X, self.A, self.B, T, self.dY, dX, dA, dB, M, r,
                           self.p["s"], self.ws)
        return dX, dA, dB

    def status(self):
        return self.Q.qlora_get_device_status(self.ws)
