"""GPU parity of the grouped (mixture-of-experts) entry points against the oracle applied per
expert ("Quantized weights, full precision: The math behind 75% cheaper fine-tuning", "LoRA
operations and quantization": LoRA on the experts of an MoE model).  Ragged expert sizes, experts
with no rows, per-expert NVFP4 tensor scales, and offsets that the device rejects."""
import numpy as np
import pytest
import torch

from bit_quantized_base_b200 import synth
from gpu_util import assert_close, to_f64

pytestmark = pytest.mark.gpu


class GpuGrouped:
    def __init__(self, p):
        from bit_quantized_base_b200 import qlora as Q
        self.Q, self.p = Q, p
        self.W = Q.weight_from_numpy(p["fmt"], p["codes"], p["scales"], p["tensor_scale"],
                                     scales2=p.get("scales2"))
        self.X = Q.bf16_from_bits(p["X"])
        self.A = Q.bf16_from_bits(p["A"])
        self.B = Q.bf16_from_bits(p["B"])
        self.dY = Q.bf16_from_bits(p["dY"])
        self.off = torch.from_numpy(p["offsets"].astype(np.int32)).cuda()
        self.E, self.M, self.N, self.K, self.r = p["E"], p["M"], p["N"], p["K"], p["r"]
        self.ws = Q.alloc_workspace(Q.OP_GROUPED_BWD, self.W, max(self.M, 1), self.r, self.E)
        Q.qlora_workspace_init(self.ws)

    def fwd(self, save_t=True):
        Q = self.Q
        Y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device="cuda")
        T = torch.empty((self.M, self.r), dtype=torch.bfloat16, device="cuda") if save_t else None
        Q.qlora_grouped_fwd(self.W, self.E, self.off, self.M, self.X, self.A, self.B, Y, T, self.r,
                            self.p["s"], self.ws)
        return Y, T

    def bwd(self, T=None, want_dx=True):
        Q, E, M, N, K, r = self.Q, self.E, self.M, self.N, self.K, self.r
        dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda") if want_dx else None
        dA = torch.full((E, r, K), float("nan"), dtype=torch.bfloat16, device="cuda")
        dB = torch.full((E, N, r), float("nan"), dtype=torch.bfloat16, device="cuda")
        Q.qlora_grouped_bwd(self.W, E, self.off, M, self.X, self.A, self.B, T, self.dY, dX, dA,
                            dB, r, self.p["s"], self.ws)
        return dX, dA, dB

    def status(self):
        return self.Q.qlora_get_device_status(self.ws)


def oracle_grouped(p):
    from oracle import oracle
    res = oracle.grouped_layer(p["fmt"], p["offsets"], p["N"], p["K"], p["r"], p["s"], p["codes"],
                               p["scales"], p["tensor_scale"], p["X"], p["A"], p["B"], p["dY"],
                               scales2=p.get("scales2"))
    cat = lambda k, w: (np.concatenate([d[k] for d in res], 0) if p["M"] else np.zeros((0, w)))
    return dict(Y=cat("Y", p["N"]), T=cat("T", p["r"]), dX=cat("dX", p["K"]),
                dA=np.stack([d["dA"] for d in res]), dB=np.stack([d["dB"] for d in res]))


GROUPED = [
    ("mxfp4", [0, 300, 1, 0, 129, 256, 17], 272, 320, 8),
    ("nf4", [200, 0, 513], 384, 192, 16),
    ("nvfp4", [64, 130, 0, 77], 256, 448, 64),
    ("mxfp4", [3, 5, 0, 2, 1, 7, 0, 0, 9, 4, 6, 8, 1, 1, 2, 40], 128, 256, 32),
    # per-expert second-level scales: 336 x 5 = 1680 first-level codes per expert (7 groups)
    ("nf4dq", [150, 0, 600, 33], 336, 320, 16),
]


@pytest.mark.parametrize("fmt,counts,N,K,r", GROUPED)
def test_grouped_matches_oracle(fmt, counts, N, K, r):
    p = synth.small_grouped(fmt, counts, N, K, r, seed=sum(counts) + N)
    g = GpuGrouped(p)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(T)
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = oracle_grouped(p)
    assert_close(to_f64(Y), ref["Y"], "Y")
    assert_close(to_f64(T), ref["T"], "T")
    assert_close(to_f64(dX), ref["dX"], "dX")
    for e in range(p["E"]):
        if counts[e] == 0:   # no rows: exact zeros
            assert torch.count_nonzero(dA[e].float()) == 0 and torch.count_nonzero(dB[e].float()) == 0
        else:
            assert_close(to_f64(dA[e]), ref["dA"][e], f"dA[{e}]")
            assert_close(to_f64(dB[e]), ref["dB"][e], f"dB[{e}]")


def test_grouped_recompute_t_and_no_dx():
    p = synth.small_grouped("nvfp4", [33, 0, 250, 96], 192, 256, 16, seed=5)
    g = GpuGrouped(p)
    Y, T = g.fwd()
    _, dA1, dB1 = g.bwd(T, want_dx=False)
    dX2, dA2, dB2 = g.bwd(None)
    torch.cuda.synchronize()
    assert g.status() == 0
    # recomputing T gives the same T bits, so the gradients agree exactly
    assert torch.equal(dA1.view(torch.int16), dA2.view(torch.int16))
    assert torch.equal(dB1.view(torch.int16), dB2.view(torch.int16))
    ref = oracle_grouped(p)
    assert_close(to_f64(dX2), ref["dX"], "dX")


def test_grouped_single_expert_equals_linear():
    # one expert covering every row is the single layer: identical bits
    from gpu_util import GpuLayer
    p = synth.small_grouped("nf4", [300], 256, 320, 16, seed=3)
    g = GpuGrouped(p)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(T)
    lp = dict(p, codes=p["codes"][0], scales=p["scales"][0], tensor_scale=1.0, A=p["A"][0],
              B=p["B"][0])
    l = GpuLayer(lp)
    Y1, T1 = l.fwd()
    dX1, dA1, dB1 = l.bwd(T1)
    torch.cuda.synchronize()
    for a, b in [(Y, Y1), (T, T1), (dX, dX1), (dA[0], dA1), (dB[0], dB1)]:
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_grouped_all_experts_empty():
    p = synth.small_grouped("mxfp4", [0, 0, 0], 128, 128, 8, seed=1)
    g = GpuGrouped(p)
    g.fwd()
    _, dA, dB = g.bwd(None, want_dx=False)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA.float()) == 0 and torch.count_nonzero(dB.float()) == 0


def test_grouped_bad_offsets_reported():
    # offsets whose last entry is not M_total: the device rejects the table and does no work
    p = synth.small_grouped("nf4", [64, 64], 128, 128, 8, seed=4)
    g = GpuGrouped(p)
    g.off.copy_(torch.tensor([0, 100, 90], dtype=torch.int32))
    g.fwd()
    g.bwd(None)
    torch.cuda.synchronize()
    assert g.status() == 1    # QLORA_ERR_INVALID_ARG
    g.Q.qlora_workspace_init(g.ws)
    assert g.status() == 0
