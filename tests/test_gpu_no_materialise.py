"""The dequantised weight is never materialised: a full forward + backward of the Llama-3-8B-shaped
NF4 up-projection (M=4096, N=14336, K=4096, r=64) through the C ABI raises neither PyTorch's
peak allocation nor the device's used memory by anything near one bf16 copy of the weight
(N*K*2 bytes), and the caller-provided workspace is itself far smaller than that copy.
("Training LLMs on a Budget", "The setup"; "Quantized weights, full precision", 4-bit base
weight storage with on-the-fly dequantization.)"""
import pytest
import torch

from bit_quantized_base_b200 import synth
from gpu_util import GpuLayer

pytestmark = pytest.mark.gpu


def test_full_size_step_allocates_no_weight_copy():
    p = synth.layer_inputs("llama3_8b_up_nf4", 0)
    N, K, M = p["N"], p["K"], p["M"]
    copy_bytes = N * K * 2
    g = GpuLayer(p)
    assert g.ws.numel() < copy_bytes // 4, f"workspace {g.ws.numel()} B"
    Y, T = g.fwd()                       # first call: library state (streams, events) set up
    g.bwd(T)
    torch.cuda.synchronize()
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((M, p["r"]), dtype=torch.bfloat16, device="cuda")
    dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((p["r"], K), dtype=torch.bfloat16, device="cuda")
    dB = torch.empty((N, p["r"]), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    base = torch.cuda.memory_allocated()
    torch.cuda.reset_peak_memory_stats()
    Q = g.Q
    for _ in range(2):
        Q.qlora_linear_fwd(g.W, g.X, g.A, g.B, Y, T, M, p["r"], p["s"], g.ws)
        Q.qlora_linear_bwd(g.W, g.X, g.A, g.B, T, g.dY, dX, dA, dB, M, p["r"], p["s"], g.ws)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert g.status() == 0
    assert torch.cuda.max_memory_allocated() - base < copy_bytes // 16
    assert free0 - free1 < copy_bytes // 16, f"device memory fell by {free0 - free1} B"
