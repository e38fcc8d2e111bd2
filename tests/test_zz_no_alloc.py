"""qlora_linear_fwd_noalloc: the forward pass for callers that cannot allocate device memory where
they run the layer (runtimes that allocate everything up front and forbid allocation on the step
path, or C callers with no allocator).  Instead of a caller workspace it uses a fixed scratch array
inside the library.  This file checks, through the C ABI, that two calls in a row give the same
outputs as the workspace entry point -- bit for bit above 256 rows, where both run the same tiled
kernels, and within the parity tolerance of the other tests below, where the workspace entry point
streams the weight instead -- that the calls leave the device allocator's count unchanged, that
the scratch's status word reads QLORA_OK afterwards, and that a size beyond the fixed scratch is
refused.  It is collected last on purpose and runs the same alone or after every other test."""
import pytest
import torch

from bit_quantized_base_b200 import synth
from gpu_util import GpuLayer, assert_close, to_f64

pytestmark = pytest.mark.gpu


def _reference_forward(g):
    return g.fwd()          # qlora_linear_fwd with a caller-allocated workspace


@pytest.mark.parametrize("first,second", [
    (("nf4", 300, 400, 512, 64), ("mxfp4", 129, 384, 192, 16)),
    (("nvfp4", 513, 528, 448, 32), ("nf4", 7, 272, 320, 8)),
])
def test_noalloc_forward_matches_workspace_forward_twice(first, second):
    from bit_quantized_base_b200 import qlora as Q
    for keep_t, (fmt, M, N, K, r) in zip((True, False), (first, second)):
        p = synth.small_layer(fmt, M, N, K, r, s=2.0, seed=M + N + K + r)
        g = GpuLayer(p)
        Y_ref, T_ref = _reference_forward(g)
        Y = torch.empty_like(Y_ref)
        T = torch.empty_like(T_ref) if keep_t else None
        torch.cuda.synchronize()
        before = torch.cuda.memory_allocated()
        Q.qlora_linear_fwd_noalloc(g.W, g.X, g.A, g.B, Y, T, M, r, p["s"])
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        assert Q.qlora_linear_fwd_noalloc_status() == 0
        if M > 256:
            assert torch.equal(Y, Y_ref), f"Y {fmt} not bitwise equal"
            if keep_t:
                assert torch.equal(T, T_ref), f"T {fmt} not bitwise equal"
        else:
            assert_close(to_f64(Y), to_f64(Y_ref), f"Y {fmt}")
            if keep_t:
                assert_close(to_f64(T), to_f64(T_ref), f"T {fmt}")


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from bit_quantized_base_b200 import qlora as Q
    p = synth.small_layer("nf4", 16, 128, 256, 64, seed=4)
    g = GpuLayer(p)
    M_big = 1_048_448 // 64 + 1            # M * r one row beyond the limit without T_save
    with pytest.raises(Q.QLoraError) as e:
        Q.qlora_linear_fwd_noalloc(g.W, g.X, g.A, g.B, g.X, None, M_big, 64, 2.0)
    assert e.value.status == 3              # QLORA_ERR_WORKSPACE
