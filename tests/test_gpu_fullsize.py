"""GPU parity at the full workload sizes, through the same entry points and launch shapes the
benchmark times, on outputs the oracle can afford: sampled rows of Y and dX (the first and last
rows plus seeded random ones) and the full T, dA and dB (cheap: O(M r (N + K))).

Workloads (inputs from the seeded recipe of each):
  NF4 Llama-3-8B-shaped MLP up-proj, M=4096, N=14336, K=4096, r=64;
  MXFP4 Llama-3-70B-shaped gate-proj, M=8192, N=28672, K=8192, r=16 (W = 0.02 t5);
  NVFP4 Llama-3-70B-shaped decoder layer, its 7 projections, M=4096, r=16;
  MXFP4 MoE experts, 64 x {gate, up 2048x7168; down 7168x2048}, 16384 tokens top-8, r=8.
"""
import numpy as np
import pytest
import torch

from bit_quantized_base_b200 import synth
from gpu_util import GpuLayer, assert_close, to_f64

pytestmark = pytest.mark.gpu


def sample_rows(M, n, seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    pick = rng.choice(M, size=min(n, M), replace=False) if M > 0 else np.zeros(0, np.int64)
    rows = np.unique(np.concatenate([[0, M - 1], pick])) if M > 0 else pick
    return rows.astype(np.int64)


DENSE = ([("llama3_8b_up_nf4", 0), ("llama3_70b_gate_mxfp4", 0)] +
         [("llama3_70b_layer_nvfp4", i) for i in range(7)])


@pytest.mark.parametrize("name,proj", DENSE,
                         ids=[f"{synth.WORKLOADS[c].fmt}-{synth.WORKLOADS[c].projs[p].name}-"
                              f"{synth.WORKLOADS[c].projs[p].N}x{synth.WORKLOADS[c].projs[p].K}"
                              for c, p in DENSE])
def test_full_size_layer_sampled(name, proj):
    from oracle import oracle
    p = synth.layer_inputs(name, proj)
    g = GpuLayer(p)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(T)
    torch.cuda.synchronize()
    assert g.status() == 0
    rows = sample_rows(p["M"], 128, 7 + 100 * synth.WORKLOADS[name].seed_id + proj)
    ref = oracle.layer(p["fmt"], p["M"], p["N"], p["K"], p["r"], p["s"], p["codes"], p["scales"],
                       p["tensor_scale"], p["X"], p["A"], p["B"], p["dY"], rows=rows,
                       want=("Y", "dX", "T", "dA", "dB"))
    idx = torch.from_numpy(rows).cuda()
    assert_close(to_f64(Y.index_select(0, idx)), ref["Y"], "Y rows")
    assert_close(to_f64(dX.index_select(0, idx)), ref["dX"], "dX rows")
    assert_close(to_f64(T), ref["T"], "T")
    assert_close(to_f64(dA), ref["dA"], "dA")
    assert_close(to_f64(dB), ref["dB"], "dB")


# the single NF4 layer N = K = 1024 at its own batch of 256 rows (every output checked), then
# the full-size weights of the NF4 up-proj and the MXFP4 gate-proj under short batches
SHORT = [("nf4_1024x1024", 256), ("llama3_8b_up_nf4", 16), ("llama3_8b_up_nf4", 256),
         ("llama3_70b_gate_mxfp4", 64)]


@pytest.mark.parametrize("name,M", SHORT, ids=[f"{c}-M{m}" for c, m in SHORT])
def test_full_size_weight_short_batch(name, M):
    # the full-size weights of the NF4 up-proj and the MXFP4 gate-proj under the short batches of
    # the weight-stream sweep: every output row is checked
    from oracle import oracle
    p = synth.layer_inputs(name, 0, M=M)
    g = GpuLayer(p)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(T)
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = oracle.layer(p["fmt"], p["M"], p["N"], p["K"], p["r"], p["s"], p["codes"], p["scales"],
                       p["tensor_scale"], p["X"], p["A"], p["B"], p["dY"],
                       want=("Y", "dX", "T", "dA", "dB"))
    for name, got in (("Y", Y), ("dX", dX), ("T", T), ("dA", dA), ("dB", dB)):
        assert_close(to_f64(got), ref[name], name)


@pytest.mark.parametrize("proj", [0, 1, 2], ids=["gate", "up", "down"])
def test_full_size_grouped_sampled(proj):
    from oracle import oracle
    from bit_quantized_base_b200 import qlora as Q
    cfg = synth.WORKLOADS["moe64_mxfp4"]
    pr = cfg.projs[proj]
    E, N, K, r, s = cfg.experts, pr.N, pr.K, cfg.r, cfg.scale
    offsets = synth.moe_routing(cfg)
    M = int(offsets[-1])
    codes, scales, _ = synth.make_weight(cfg, proj, N, K, experts=E)
    A, B = synth.make_adapters(cfg, proj, N, K, experts=E)
    X, dY = synth.make_activations(cfg, proj, M, N, K)

    W = Q.weight_from_numpy(cfg.fmt, codes, scales, None)
    Xd, Ad, Bd, dYd = (Q.bf16_from_bits(a) for a in (X, A, B, dY))
    off = torch.from_numpy(offsets.astype(np.int32)).cuda()
    ws = Q.alloc_workspace(Q.OP_GROUPED_BWD, W, M, r, E)
    Q.qlora_workspace_init(ws)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((E, r, K), dtype=torch.bfloat16, device="cuda")
    dB = torch.empty((E, N, r), dtype=torch.bfloat16, device="cuda")
    Q.qlora_grouped_fwd(W, E, off, M, Xd, Ad, Bd, Y, T, r, s, ws)
    Q.qlora_grouped_bwd(W, E, off, M, Xd, Ad, Bd, T, dYd, dX, dA, dB, r, s, ws)
    torch.cuda.synchronize()
    assert Q.qlora_get_device_status(ws) == 0

    local = [sample_rows(int(offsets[e + 1] - offsets[e]), 6, 50 + 10 * proj + e) for e in range(E)]
    res = oracle.grouped_layer(cfg.fmt, offsets, N, K, r, s, codes, scales, None, X, A, B, dY,
                               rows_per_expert=local, want=("Y", "dX", "T", "dA", "dB"))
    rows = np.concatenate([offsets[e] + local[e] for e in range(E)])
    idx = torch.from_numpy(rows).cuda()
    assert_close(to_f64(Y.index_select(0, idx)), np.concatenate([d["Y"] for d in res]), "Y rows")
    assert_close(to_f64(dX.index_select(0, idx)), np.concatenate([d["dX"] for d in res]), "dX rows")
    assert_close(to_f64(T), np.concatenate([d["T"] for d in res]), "T")
    for e in range(E):
        assert_close(to_f64(dA[e]), res[e]["dA"], f"dA[{e}]")
        assert_close(to_f64(dB[e]), res[e]["dB"], f"dB[{e}]")
