"""Host-side checks of the C ABI that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments with the documented status before touching CUDA."""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def Q():
    from bit_quantized_base_b200 import build
    build.build()
    from bit_quantized_base_b200 import qlora
    return qlora


def _declared():
    src = open(os.path.join(ROOT, "include", "qlora.h")).read()
    return sorted(set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(qlora_\w+)\s*\(", src)))


def test_header_declarations_are_exported(Q):
    names = _declared()
    assert len(names) >= 11
    for n in names:
        getattr(Q.lib, n)                     # raises AttributeError if not exported
    assert sorted(Q.EXPORTS) == names


def test_status_strings(Q):
    for s in range(6):
        assert Q.lib.qlora_status_string(s)
    assert b"sm_100a" in Q.lib.qlora_build_info()


class FakeT:
    """Stands in for a device tensor: only data_ptr() / numel() are used by the binding."""

    def __init__(self, ptr, n=1 << 30):
        self.ptr, self.n = ptr, n

    def data_ptr(self):
        return self.ptr

    def numel(self):
        return self.n


def _w(Q, fmt="nf4", N=256, K=512, codes=0x1000, scales=0x2000, ts=None):
    W = Q.Weight.__new__(Q.Weight)
    W.fmt, W.N, W.K = fmt, N, K
    W.codes, W.scales, W.tensor_scale = None, None, None
    W.c = Q.qlora_weight_t(Q.FMT[fmt], 0, N, K, codes, scales, ts)
    return W


def test_workspace_size_rules(Q):
    W = _w(Q)
    assert Q.qlora_workspace_size(Q.OP_FWD, W, 1024, 16) > 0
    assert Q.qlora_workspace_size(Q.OP_BWD, W, 1024, 16) >= Q.qlora_workspace_size(Q.OP_FWD, W, 1024, 16)
    assert Q.qlora_workspace_size(Q.OP_FWD, W, 1024, 12) == 0          # rank not supported
    assert Q.qlora_workspace_size(Q.OP_FWD, _w(Q, K=96), 16, 16) == 0  # K % 64
    assert Q.qlora_workspace_size(Q.OP_FWD, _w(Q, N=40), 16, 16) == 0  # N % 16
    assert Q.qlora_workspace_size(Q.OP_FWD, _w(Q, fmt="nvfp4"), 16, 16) == 0   # NVFP4 needs tensor scale
    assert Q.qlora_workspace_size(Q.OP_FWD, _w(Q, codes=0x1008), 16, 16) == 0  # misaligned codes


@pytest.mark.parametrize("bad,status", [
    (dict(M=-1), "QLORA_ERR_INVALID_ARG"),
    (dict(r=12), "QLORA_ERR_UNSUPPORTED"),
    (dict(r=0), "QLORA_ERR_INVALID_ARG"),
    (dict(X=0x1004), "QLORA_ERR_INVALID_ARG"),
    (dict(Y=0), "QLORA_ERR_INVALID_ARG"),
    (dict(ws=0), "QLORA_ERR_WORKSPACE"),
    (dict(ws_bytes=64), "QLORA_ERR_WORKSPACE"),
    (dict(W=dict(K=100)), "QLORA_ERR_INVALID_ARG"),
    (dict(W=dict(fmt="nvfp4")), "QLORA_ERR_INVALID_ARG"),
])
def test_forward_rejects_bad_arguments(Q, bad, status):
    W = _w(Q, **bad.get("W", {}))
    args = dict(X=0x10000, A=0x20000, B=0x30000, Y=0x40000, T=0, M=64, r=16, ws=0x50000,
                ws_bytes=1 << 30)
    args.update({k: v for k, v in bad.items() if k != "W"})
    rc = Q.lib.qlora_linear_fwd(W.ref, args["X"], args["A"], args["B"], args["Y"],
                                args["T"] or None, args["M"], args["r"], 2.0,
                                args["ws"] or None, args["ws_bytes"], None)
    assert Q.STATUS[rc] == status


def test_backward_rejects_bad_arguments(Q):
    W = _w(Q)
    ok = dict(X=0x10000, A=0x20000, B=0x30000, T=None, dY=0x60000, dX=None, dA=0x70000,
              dB=0x80000)
    for key in ("X", "A", "B", "dY", "dA", "dB"):
        a = dict(ok)
        a[key] = None
        rc = Q.lib.qlora_linear_bwd(W.ref, a["X"], a["A"], a["B"], a["T"], a["dY"], a["dX"],
                                    a["dA"], a["dB"], 64, 16, 2.0, 0x50000, 1 << 30, None)
        assert Q.STATUS[rc] == "QLORA_ERR_INVALID_ARG", key
    a = dict(ok, dX=0x90008)   # misaligned optional output
    rc = Q.lib.qlora_linear_bwd(W.ref, a["X"], a["A"], a["B"], a["T"], a["dY"], a["dX"], a["dA"],
                                a["dB"], 64, 16, 2.0, 0x50000, 1 << 30, None)
    assert Q.STATUS[rc] == "QLORA_ERR_INVALID_ARG"


def test_workspace_sized_for_more_rows_serves_fewer(Q):
    # The workspace size is not monotone in M: one layer of at most 256 rows adds the short-batch
    # kernels' fp32 split partials, which larger batches do not use.  A workspace sized for more
    # rows is still accepted for fewer (the call then runs the tiled kernels); one without room
    # for Zs, T and U is rejected.  Without a GPU driver an accepted call stops at its first CUDA
    # call (QLORA_ERR_CUDA), before which nothing is enqueued.
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    W = _w(Q, N=14336, K=4096)
    r = 16
    for op in (Q.OP_FWD, Q.OP_BWD):
        big = Q.qlora_workspace_size(op, W, 1024, r)
        for M in (16, 64, 256):
            assert Q.qlora_workspace_size(op, W, M, r) > big      # the partials of the short path
            if op == Q.OP_FWD:
                rc = Q.lib.qlora_linear_fwd(W.ref, 0x10000, 0x20000, 0x30000, 0x40000, None, M, r,
                                            2.0, 0x50000, big, None)
            else:
                rc = Q.lib.qlora_linear_bwd(W.ref, 0x10000, 0x20000, 0x30000, None, 0x60000,
                                            0x90000, 0x70000, 0x80000, M, r, 2.0, 0x50000, big,
                                            None)
            assert Q.STATUS[rc] == "QLORA_ERR_CUDA", (op, M)
        # required: the 8192-byte header, Zs and T (and U) as 256-byte rounded [M, r] bf16 regions,
        # and for the backward lora_down's cluster sums (8 x 128 x r fp32)
        m = 256
        z = -(-m * r * 2 // 256) * 256
        need = 8192 + (3 * z + 8 * 128 * r * 4 if op == Q.OP_BWD else 2 * z)
        for nbytes, want in ((need - 16, "QLORA_ERR_WORKSPACE"), (need, "QLORA_ERR_CUDA")):
            if op == Q.OP_FWD:
                rc = Q.lib.qlora_linear_fwd(W.ref, 0x10000, 0x20000, 0x30000, 0x40000, None, m, r,
                                            2.0, 0x50000, nbytes, None)
            else:
                rc = Q.lib.qlora_linear_bwd(W.ref, 0x10000, 0x20000, 0x30000, None, 0x60000,
                                            0x90000, 0x70000, 0x80000, m, r, 2.0, 0x50000, nbytes,
                                            None)
            assert Q.STATUS[rc] == want, (op, nbytes)


def test_workspace_init_and_status_reject_null(Q):
    assert Q.STATUS[Q.lib.qlora_workspace_init(None, 1 << 20, None)] == "QLORA_ERR_WORKSPACE"
    assert Q.STATUS[Q.lib.qlora_get_device_status(None, None)] == "QLORA_ERR_WORKSPACE"
    assert Q.STATUS[Q.lib.qlora_debug_wait_timeout(0x1000, 1 << 20, 0, None)] == "QLORA_ERR_INVALID_ARG"


def test_quantize_rejects_bad_arguments(Q):
    def rc(W, v):
        return Q.STATUS[Q.lib.qlora_quantize(W.ref, v, 0, None)]
    assert rc(_w(Q), 0x1004) == "QLORA_ERR_INVALID_ARG"            # v not 16-byte aligned
    assert rc(_w(Q), None) == "QLORA_ERR_INVALID_ARG"
    assert rc(_w(Q, K=100), 0x10000) == "QLORA_ERR_INVALID_ARG"     # K % 64
    assert rc(_w(Q, fmt="nvfp4"), 0x10000) == "QLORA_ERR_INVALID_ARG"   # no tensor-scale slot
    assert rc(_w(Q, fmt="nf4dq"), 0x10000) == "QLORA_ERR_INVALID_ARG"   # no second-level scales


def test_merge_rejects_bad_arguments(Q):
    W, Wo = _w(Q), _w(Q, codes=0x3000, scales=0x4000)

    def rc(W_out=Wo, A=0x10000, B=0x20000, r=16, merged=0x30000):
        return Q.STATUS[Q.lib.qlora_merge_requantize(W.ref, A, B, r, 2.0, W_out.ref, merged, None)]
    assert rc(r=0) == "QLORA_ERR_INVALID_ARG"
    assert rc(r=1025) == "QLORA_ERR_INVALID_ARG"
    assert rc(A=None) == "QLORA_ERR_INVALID_ARG"
    assert rc(merged=0x30004) == "QLORA_ERR_INVALID_ARG"
    assert rc(W_out=_w(Q, N=512, codes=0x3000, scales=0x4000)) == "QLORA_ERR_INVALID_ARG"


def test_loftq_arguments(Q):
    N, K = 256, 512
    assert Q.qlora_loftq_workspace_size(N, K, 0) == 0
    assert Q.qlora_loftq_workspace_size(N, K, 97) == 0              # above the subspace limit
    assert Q.qlora_loftq_workspace_size(16, K, 32) == 0             # r > N
    need = Q.qlora_loftq_workspace_size(N, K, 16)
    assert need >= 4 * N * K
    W = _w(Q, N=N, K=K)

    def rc(r=16, scale=2.0, iters=5, power=4, work=0x100000, nbytes=need, errs=0x60000, v=0x70000):
        return Q.STATUS[Q.lib.qlora_loftq(v, W.ref, r, scale, iters, power, 0, 0x80000, 0x90000,
                                          errs, None, work, nbytes, None)]
    assert rc(r=0) == "QLORA_ERR_INVALID_ARG"
    assert rc(scale=0.0) == "QLORA_ERR_INVALID_ARG"
    assert rc(scale=float("nan")) == "QLORA_ERR_INVALID_ARG"
    assert rc(iters=0) == "QLORA_ERR_INVALID_ARG"
    assert rc(power=17) == "QLORA_ERR_INVALID_ARG"
    assert rc(work=0x100010) == "QLORA_ERR_INVALID_ARG"             # not 256-byte aligned
    assert rc(errs=None) == "QLORA_ERR_INVALID_ARG"
    assert rc(v=0x70008) == "QLORA_ERR_INVALID_ARG"
    assert rc(nbytes=need - 1) == "QLORA_ERR_WORKSPACE"


def test_valid_offline_calls_reach_cuda_without_a_gpu(Q):
    # arguments that pass every check: on a machine without a GPU driver the first CUDA call
    # fails and the entry point reports QLORA_ERR_CUDA (nothing is left half-done on the host)
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    N, K = 256, 512
    W = _w(Q, N=N, K=K)
    need = Q.qlora_loftq_workspace_size(N, K, 16)
    rc = Q.lib.qlora_loftq(0x70000, W.ref, 16, 2.0, 5, 4, 0, 0x80000, 0x90000, 0x60000, None,
                           0x100000, need, None)
    assert Q.STATUS[rc] == "QLORA_ERR_CUDA"
    assert Q.STATUS[Q.lib.qlora_quantize(W.ref, 0x10000, 0, None)] == "QLORA_ERR_CUDA"


@pytest.mark.parametrize("fmt,bs,sdt", [("nf4", 64, "float32"), ("nf4dq", 64, "uint8"),
                                        ("mxfp4", 32, "uint8"), ("nvfp4", 16, "uint8")])
def test_empty_weight_storage_shapes(Q, fmt, bs, sdt):
    # the binding's storage for a weight matches the layouts include/qlora.h states
    N, K = 48, 704
    W = Q.empty_weight(fmt, N, K, device="cpu")
    assert tuple(W.codes.shape) == (N, K // 2) and str(W.codes.dtype) == "torch.uint8"
    assert tuple(W.scales.shape) == (N, K // bs) and str(W.scales.dtype) == f"torch.{sdt}"
    assert (W.tensor_scale is not None) == (fmt == "nvfp4")
    if fmt == "nf4dq":
        assert W.scales2.numel() == -(-N * (K // 64) // 256)       # one per 256 first-level codes
    else:
        assert W.scales2 is None
    assert W.c.fmt == Q.FMT[fmt] and W.c.N == N and W.c.K == K


def test_noalloc_empty_batch_accepts_null_activations(Q):
    # M = 0 is a no-op, as for qlora_linear_fwd: NULL X and Y are accepted and nothing is enqueued
    rc = Q.lib.qlora_linear_fwd_noalloc(_w(Q).ref, None, 0x20000, 0x30000, None, None, 0, 16, 2.0,
                                        None)
    assert Q.STATUS[rc] == "QLORA_OK"
    rc = Q.lib.qlora_linear_fwd_noalloc(_w(Q).ref, None, 0x20000, 0x30000, None, None, 4, 16, 2.0,
                                        None)
    assert Q.STATUS[rc] == "QLORA_ERR_INVALID_ARG"


@pytest.mark.parametrize("keep_t,m_max", [(False, 16382), (True, 32766)])
def test_noalloc_size_limit_boundary(Q, keep_t, m_max):
    # r = 64: the largest batch that fits the fixed scratch passes the size check (on a machine
    # without a GPU it then fails at the first CUDA call); one row more is refused before any
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the accepted size would run")
    T = 0x60000 if keep_t else None

    def rc(M):
        return Q.STATUS[Q.lib.qlora_linear_fwd_noalloc(_w(Q).ref, 0x10000, 0x20000, 0x30000,
                                                       0x40000, T, M, 64, 2.0, None)]
    assert rc(m_max + 1) == "QLORA_ERR_WORKSPACE"
    assert rc(m_max) == "QLORA_ERR_CUDA"


@pytest.mark.parametrize("bad,status", [
    (dict(W=dict(fmt="nf4")), "QLORA_ERR_UNSUPPORTED"),             # E2M1 codes only: MXFP4
    (dict(W=dict(fmt="mxfp4", K=192)), "QLORA_ERR_UNSUPPORTED"),    # K % 128
    (dict(W=dict(fmt="mxfp4", codes=0x1010)), "QLORA_ERR_INVALID_ARG"),   # codes not 32-aligned
    (dict(M=-1), "QLORA_ERR_INVALID_ARG"),
    (dict(r=12), "QLORA_ERR_UNSUPPORTED"),
    (dict(X=0x1004), "QLORA_ERR_INVALID_ARG"),
    (dict(ws=0), "QLORA_ERR_WORKSPACE"),
    (dict(ws_bytes=64), "QLORA_ERR_WORKSPACE"),
])
def test_w4a8_forward_rejects_bad_arguments(Q, bad, status):
    wargs = dict(fmt="mxfp4")
    wargs.update(bad.get("W", {}))
    W = _w(Q, **wargs)
    args = dict(X=0x10000, A=0x20000, B=0x30000, Y=0x40000, M=64, r=16, ws=0x50000,
                ws_bytes=1 << 30)
    args.update({k: v for k, v in bad.items() if k != "W"})
    rc = Q.lib.qlora_linear_fwd_w4a8(W.ref, args["X"], args["A"], args["B"], args["Y"], None,
                                     args["M"], args["r"], 2.0, args["ws"] or None,
                                     args["ws_bytes"], None)
    assert Q.STATUS[rc] == status


def test_w4a8_workspace_and_quantizer_rules(Q):
    W = _w(Q, fmt="mxfp4", N=256, K=512)
    M, r = 300, 16
    n = Q.qlora_workspace_size(Q.OP_FWD_W4A8, W, M, r)
    # header + Zs + T + codes [M,K] + scales [M,K/32], each rounded up to 256 bytes
    up = lambda x: (x + 255) // 256 * 256
    assert n == 8192 + 2 * up(M * r * 2) + up(M * 512) + up(M * 512 // 32)
    assert Q.STATUS[Q.lib.qlora_mxfp8_quantize(0x10000, 4, 192, 0x20000, 0x30000, None)] == \
        "QLORA_ERR_INVALID_ARG"                                      # K % 128
    assert Q.STATUS[Q.lib.qlora_mxfp8_quantize(0x10008, 4, 256, 0x20000, 0x30000, None)] == \
        "QLORA_ERR_INVALID_ARG"                                      # misaligned X
    assert Q.STATUS[Q.lib.qlora_mxfp8_quantize(None, 0, 256, None, None, None)] == "QLORA_OK"
