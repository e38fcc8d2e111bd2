"""Run by tests/test_gpu_debug_build.py in a child process with QLORA_LIBRARY=debug: small ragged
problems through every kernel path of the bounds-checked build (CTA-pair tiles above 256 rows, the
streaming kernel at 65..256 rows, the short-batch kernels at <= 64 rows, the grouped path, NF4
with double-quantised absmax), each checked for a clean status word and against the oracle.
Prints one line per case and exits non-zero on the first failure."""
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

from bit_quantized_base_b200 import qlora as Q  # noqa: E402
from bit_quantized_base_b200 import synth  # noqa: E402
from oracle import oracle as O  # noqa: E402
from gpu_util import GpuLayer, assert_close, to_f64  # noqa: E402

assert os.path.basename(Q.LIB_PATH) == "libqlora_debug.so", Q.LIB_PATH
assert b"debug" in Q.lib.qlora_build_info()

CASES = [
    # fmt, M, N, K, r: pair tiles, streaming, short, ragged in every dimension
    ("nf4", 300, 400, 320, 16),
    ("mxfp4", 130, 272, 448, 8),
    ("nvfp4", 200, 528, 256, 32),
    ("nf4", 33, 144, 704, 64),
    ("mxfp4", 7, 1040, 192, 16),
    ("nvfp4", 64, 400, 960, 8),
    ("nf4", 40, 2064, 320, 32),      # short dX whose U = dY B runs on two clusters
    ("nf4dq", 270, 256, 512, 16),
]


def layer_case(fmt, M, N, K, r):
    p = synth.small_layer(fmt, M, N, K, r, s=2.0, seed=M + N + K + r)
    g = GpuLayer(p)
    Y, T = g.fwd()
    dX, dA, dB = g.bwd(None)
    torch.cuda.synchronize()
    st = g.status()
    if st != 0:
        raise SystemExit(f"{fmt} M={M} N={N} K={K} r={r}: device status {st}")
    ref = O.layer(fmt, M, N, K, r, p["s"], p["codes"], p["scales"], p["tensor_scale"], p["X"],
                  p["A"], p["B"], p["dY"], scales2=p.get("scales2"))
    for name, got in (("Y", Y), ("T", T), ("dX", dX), ("dA", dA), ("dB", dB)):
        assert_close(to_f64(got), ref[name], name)
    print(f"ok {fmt} M={M} N={N} K={K} r={r}", flush=True)


def grouped_case():
    pg = synth.small_grouped("mxfp4", [70, 0, 150, 9], 272, 320, 8, seed=3)
    W = Q.weight_from_numpy("mxfp4", pg["codes"], pg["scales"], None)
    X, A, B, dY = (Q.bf16_from_bits(pg[k]) for k in ("X", "A", "B", "dY"))
    E, M = 4, pg["M"]
    off = torch.from_numpy(pg["offsets"].astype(np.int32)).cuda()
    ws = Q.alloc_workspace(Q.OP_GROUPED_BWD, W, M, 8, E)
    Q.qlora_workspace_init(ws)
    Y = torch.empty((M, 272), dtype=torch.bfloat16, device="cuda")
    T = torch.empty((M, 8), dtype=torch.bfloat16, device="cuda")
    dX = torch.empty((M, 320), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((E, 8, 320), dtype=torch.bfloat16, device="cuda")
    dB = torch.empty((E, 272, 8), dtype=torch.bfloat16, device="cuda")
    Q.qlora_grouped_fwd(W, E, off, M, X, A, B, Y, T, 8, pg["s"], ws)
    Q.qlora_grouped_bwd(W, E, off, M, X, A, B, T, dY, dX, dA, dB, 8, pg["s"], ws)
    torch.cuda.synchronize()
    st = Q.qlora_get_device_status(ws)
    if st != 0:
        raise SystemExit(f"grouped: device status {st}")
    res = O.grouped_layer("mxfp4", pg["offsets"], 272, 320, 8, pg["s"], pg["codes"], pg["scales"],
                          None, pg["X"], pg["A"], pg["B"], pg["dY"])
    assert_close(to_f64(Y), np.concatenate([d["Y"] for d in res]), "Y")
    assert_close(to_f64(dX), np.concatenate([d["dX"] for d in res]), "dX")
    print("ok grouped mxfp4 experts [70, 0, 150, 9]", flush=True)


if __name__ == "__main__":
    torch.cuda.set_device(0)
    for c in CASES:
        layer_case(*c)
    grouped_case()
    print("all debug-build cases passed")
