"""Python binding of libqlora.so (include/qlora.h): argument marshalling only.

Every function here has the name of the C entry point it calls and takes torch tensors already on
the GPU (PyTorch provides device memory and streams; all computation happens in the library's
CUDA kernels).  A non-OK status raises QLoraError.  If libqlora.so is missing the import fails:
there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# QLORA_LIBRARY=debug selects the bounds-checked debug build (libqlora_debug.so, -DQLORA_DEBUG)
LIB_PATH = os.path.join(_PKG, "libqlora_debug.so" if os.environ.get("QLORA_LIBRARY") == "debug"
                        else "libqlora.so")

FMT = {"nf4": 0, "mxfp4": 1, "nvfp4": 2, "nf4dq": 3}
BLOCK = {"nf4": 64, "mxfp4": 32, "nvfp4": 16}
OP_FWD, OP_BWD, OP_GROUPED_FWD, OP_GROUPED_BWD, OP_FWD_W4A8 = 0, 1, 2, 3, 4

STATUS = {0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_UNSUPPORTED",
          3: "QLORA_ERR_WORKSPACE", 4: "QLORA_ERR_CUDA", 5: "QLORA_ERR_DEVICE_TIMEOUT"}

# every symbol include/qlora.h declares
EXPORTS = ("qlora_workspace_size", "qlora_workspace_init", "qlora_linear_fwd", "qlora_linear_bwd",
           "qlora_grouped_fwd", "qlora_grouped_bwd", "qlora_get_device_status",
           "qlora_debug_dequant", "qlora_debug_wait_timeout", "qlora_status_string",
           "qlora_build_info", "qlora_launch_count", "qlora_profile_enable",
           "qlora_profile_reset", "qlora_profile_read", "qlora_linear_fwd_noalloc",
           "qlora_linear_fwd_noalloc_status", "qlora_linear_fwd_w4a8", "qlora_mxfp8_quantize",
           "qlora_debug_decode_rate", "qlora_quantize", "qlora_merge_requantize",
           "qlora_loftq_workspace_size", "qlora_loftq")


class QLoraError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS.get(self.status, self.status)} "
                         f"({_status_string(self.status)})")


class qlora_weight_t(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("scales2", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python bit_quantized_base_b200/build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    c = ctypes
    P = c.c_void_p
    W = c.POINTER(qlora_weight_t)
    L.qlora_workspace_size.argtypes = [c.c_int, W, c.c_int64, c.c_int, c.c_int]
    L.qlora_workspace_size.restype = c.c_size_t
    L.qlora_workspace_init.argtypes = [P, c.c_size_t, P]
    L.qlora_linear_fwd.argtypes = [W, P, P, P, P, P, c.c_int64, c.c_int, c.c_float, P, c.c_size_t, P]
    L.qlora_linear_bwd.argtypes = [W, P, P, P, P, P, P, P, P, c.c_int64, c.c_int, c.c_float, P,
                                   c.c_size_t, P]
    L.qlora_grouped_fwd.argtypes = [W, c.c_int, P, c.c_int64, P, P, P, P, P, c.c_int, c.c_float,
                                    P, c.c_size_t, P]
    L.qlora_grouped_bwd.argtypes = [W, c.c_int, P, c.c_int64, P, P, P, P, P, P, P, P, c.c_int,
                                    c.c_float, P, c.c_size_t, P]
    L.qlora_get_device_status.argtypes = [P, P]
    L.qlora_debug_dequant.argtypes = [W, c.c_int, P, P]
    L.qlora_debug_wait_timeout.argtypes = [P, c.c_size_t, c.c_int, P]
    L.qlora_debug_decode_rate.argtypes = [c.c_int, c.c_int, c.POINTER(c.c_double)]
    L.qlora_quantize.argtypes = [W, P, c.c_int, P]
    L.qlora_merge_requantize.argtypes = [W, P, P, c.c_int, c.c_float, W, P, P]
    L.qlora_loftq_workspace_size.argtypes = [c.c_int64, c.c_int64, c.c_int]
    L.qlora_loftq_workspace_size.restype = c.c_size_t
    L.qlora_loftq.argtypes = [P, W, c.c_int, c.c_float, c.c_int, c.c_int, c.c_uint64, P, P, P, P,
                              P, c.c_size_t, P]
    L.qlora_status_string.argtypes = [c.c_int]
    L.qlora_status_string.restype = c.c_char_p
    L.qlora_build_info.restype = c.c_char_p
    L.qlora_launch_count.restype = c.c_int64
    L.qlora_linear_fwd_w4a8.argtypes = [W, P, P, P, P, P, c.c_int64, c.c_int, c.c_float, P,
                                        c.c_size_t, P]
    L.qlora_mxfp8_quantize.argtypes = [P, c.c_int64, c.c_int64, P, P, P]
    L.qlora_linear_fwd_noalloc.argtypes = [W, P, P, P, P, P, c.c_int64, c.c_int, c.c_float, P]
    L.qlora_linear_fwd_noalloc.restype = c.c_int
    L.qlora_linear_fwd_noalloc_status.argtypes = [P]
    L.qlora_linear_fwd_noalloc_status.restype = c.c_int
    L.qlora_profile_enable.argtypes = [c.c_int]
    L.qlora_profile_read.argtypes = [c.c_int, c.POINTER(c.c_int), c.POINTER(c.c_char_p),
                                     c.POINTER(c.c_int), c.POINTER(c.c_double)]
    for name in ("qlora_workspace_init", "qlora_linear_fwd", "qlora_linear_bwd",
                 "qlora_grouped_fwd", "qlora_grouped_bwd", "qlora_get_device_status",
                 "qlora_debug_dequant", "qlora_debug_wait_timeout", "qlora_debug_decode_rate",
                 "qlora_quantize", "qlora_merge_requantize", "qlora_loftq",
                 "qlora_linear_fwd_w4a8", "qlora_mxfp8_quantize",
                 "qlora_profile_enable",
                 "qlora_profile_reset", "qlora_profile_read"):
        getattr(L, name).restype = c.c_int
    return L


lib = _load()


def _status_string(s):
    return lib.qlora_status_string(int(s)).decode()


def _check(status, where):
    if status != 0:
        raise QLoraError(status, where)


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Weight:
    """A frozen 4-bit weight resident on the GPU (codes [.., N, K/2] uint8, scales, for NVFP4 the
    tensor scale and for NF4-DQ the second-level scales, as float32 device tensors)."""

    def __init__(self, fmt, N, K, codes, scales, tensor_scale=None, scales2=None):
        self.fmt, self.N, self.K = fmt, int(N), int(K)
        self.codes, self.scales, self.tensor_scale = codes, scales, tensor_scale
        self.scales2 = scales2
        self.c = qlora_weight_t(FMT[fmt], 0, self.N, self.K, _p(codes), _p(scales),
                                _p(tensor_scale), _p(scales2))

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def nbytes(self):
        n = self.codes.numel() * self.codes.element_size() + self.scales.numel() * self.scales.element_size()
        if self.tensor_scale is not None:
            n += self.tensor_scale.numel() * 4
        if self.scales2 is not None:
            n += self.scales2.numel() * 4
        return n


def qlora_workspace_size(op, W: Weight, M, r, E=0):
    return int(lib.qlora_workspace_size(int(op), W.ref, int(M), int(r), int(E)))


def qlora_workspace_init(ws, stream=None):
    _check(lib.qlora_workspace_init(_p(ws), ws.numel(), _stream(stream)), "qlora_workspace_init")


def qlora_linear_fwd(W: Weight, X, A, B, Y, T_save, M, r, scale, ws, stream=None):
    _check(lib.qlora_linear_fwd(W.ref, _p(X), _p(A), _p(B), _p(Y), _p(T_save), int(M), int(r),
                                float(scale), _p(ws), 0 if ws is None else ws.numel(),
                                _stream(stream)), "qlora_linear_fwd")


def qlora_linear_fwd_w4a8(W: Weight, X, A, B, Y, T_save, M, r, scale, ws, stream=None):
    """Opt-in native block-scaled forward (MXFP4 weight, activations quantised to MXFP8)."""
    _check(lib.qlora_linear_fwd_w4a8(W.ref, _p(X), _p(A), _p(B), _p(Y), _p(T_save), int(M), int(r),
                                     float(scale), _p(ws), 0 if ws is None else ws.numel(),
                                     _stream(stream)), "qlora_linear_fwd_w4a8")


def qlora_mxfp8_quantize(X, M, K, codes, scales, stream=None):
    """X [M,K] bf16 -> codes [M,K] uint8 (E4M3) and scales [M,K/32] uint8 (E8M0)."""
    _check(lib.qlora_mxfp8_quantize(_p(X), int(M), int(K), _p(codes), _p(scales), _stream(stream)),
           "qlora_mxfp8_quantize")


def qlora_linear_fwd_noalloc(W: Weight, X, A, B, Y, T_save, M, r, scale, stream=None):
    """Forward with the library's fixed internal scratch instead of a caller workspace."""
    _check(lib.qlora_linear_fwd_noalloc(W.ref, _p(X), _p(A), _p(B), _p(Y), _p(T_save), int(M),
                                        int(r), float(scale), _stream(stream)),
           "qlora_linear_fwd_noalloc")


def qlora_linear_fwd_noalloc_status(stream=None):
    """Synchronise the stream and return the no-alloc scratch's device status word (an int)."""
    return int(lib.qlora_linear_fwd_noalloc_status(_stream(stream)))


def qlora_linear_bwd(W: Weight, X, A, B, T, dY, dX, dA, dB, M, r, scale, ws, stream=None):
    _check(lib.qlora_linear_bwd(W.ref, _p(X), _p(A), _p(B), _p(T), _p(dY), _p(dX), _p(dA), _p(dB),
                                int(M), int(r), float(scale), _p(ws),
                                0 if ws is None else ws.numel(), _stream(stream)),
           "qlora_linear_bwd")


def qlora_grouped_fwd(W: Weight, E, offsets, M_total, X, A, B, Y, T_save, r, scale, ws,
                      stream=None):
    _check(lib.qlora_grouped_fwd(W.ref, int(E), _p(offsets), int(M_total), _p(X), _p(A), _p(B),
                                 _p(Y), _p(T_save), int(r), float(scale), _p(ws),
                                 0 if ws is None else ws.numel(), _stream(stream)),
           "qlora_grouped_fwd")


def qlora_grouped_bwd(W: Weight, E, offsets, M_total, X, A, B, T, dY, dX, dA, dB, r, scale, ws,
                      stream=None):
    _check(lib.qlora_grouped_bwd(W.ref, int(E), _p(offsets), int(M_total), _p(X), _p(A), _p(B),
                                 _p(T), _p(dY), _p(dX), _p(dA), _p(dB), int(r), float(scale),
                                 _p(ws), 0 if ws is None else ws.numel(), _stream(stream)),
           "qlora_grouped_bwd")


def qlora_get_device_status(ws, stream=None):
    return int(lib.qlora_get_device_status(_p(ws), _stream(stream)))


def qlora_debug_dequant(W: Weight, transposed, out, stream=None):
    _check(lib.qlora_debug_dequant(W.ref, int(transposed), _p(out), _stream(stream)),
           "qlora_debug_dequant")


def qlora_debug_wait_timeout(ws, limit_us, stream=None):
    _check(lib.qlora_debug_wait_timeout(_p(ws), ws.numel(), int(limit_us), _stream(stream)),
           "qlora_debug_wait_timeout")


def empty_weight(fmt, N, K, device="cuda"):
    """Device storage for a weight of this format and shape (contents undefined)."""
    fid = FMT[fmt]
    bs = {0: 64, 1: 32, 2: 16, 3: 64}[fid]
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((N, K // bs), dtype=torch.float32 if fid == 0 else torch.uint8,
                         device=device)
    ts = torch.empty(1, dtype=torch.float32, device=device) if fid == 2 else None
    s2 = (torch.empty((N * (K // 64) + 255) // 256, dtype=torch.float32, device=device)
          if fid == 3 else None)
    return Weight(fmt, N, K, codes, scales, ts, s2)


def qlora_quantize(W: Weight, v, stream=None):
    """Quantise the float weight v [N,K] (fp32 or bf16 device tensor) into W's storage."""
    _check(lib.qlora_quantize(W.ref, _p(v), 1 if v.dtype == torch.bfloat16 else 0, _stream(stream)),
           "qlora_quantize")


def qlora_merge_requantize(W: Weight, A, B, r, scale, W_out: Weight, merged, stream=None):
    """W_out = Q(deq(W) + scale B A); the merged fp32 values land in `merged` [N,K]."""
    _check(lib.qlora_merge_requantize(W.ref, _p(A), _p(B), int(r), float(scale), W_out.ref,
                                      _p(merged), _stream(stream)), "qlora_merge_requantize")


def qlora_loftq_workspace_size(N, K, r):
    return int(lib.qlora_loftq_workspace_size(int(N), int(K), int(r)))


def qlora_loftq(W_float, Q: Weight, r, scale, iters=5, power_iters=4, seed=0, A=None, B=None,
                errs=None, sigma=None, work=None, stream=None):
    """LoftQ initialisation: Q receives the last quantisation; returns (A [r,K] bf16, B [N,r]
    bf16, errs [iters+1] fp32, sigma [r] fp32), all device tensors."""
    N, K = Q.N, Q.K
    dev = W_float.device
    A = torch.empty((r, K), dtype=torch.bfloat16, device=dev) if A is None else A
    B = torch.empty((N, r), dtype=torch.bfloat16, device=dev) if B is None else B
    errs = torch.empty(iters + 1, dtype=torch.float32, device=dev) if errs is None else errs
    sigma = torch.empty(r, dtype=torch.float32, device=dev) if sigma is None else sigma
    if work is None:
        work = torch.empty(max(1, qlora_loftq_workspace_size(N, K, r)), dtype=torch.uint8,
                           device=dev)
    _check(lib.qlora_loftq(_p(W_float), Q.ref, int(r), float(scale), int(iters), int(power_iters),
                           int(seed), _p(A), _p(B), _p(errs), _p(sigma), _p(work), work.numel(),
                           _stream(stream)), "qlora_loftq")
    return A, B, errs, sigma


def qlora_debug_decode_rate(fmt, iters=2000):
    """Decoded weights per SM clock of the layer's dequant stage, measured on every SM."""
    v = ctypes.c_double(0.0)
    _check(lib.qlora_debug_decode_rate(FMT[fmt] if isinstance(fmt, str) else int(fmt), int(iters),
                                       ctypes.byref(v)), "qlora_debug_decode_rate")
    return v.value


def qlora_build_info():
    return lib.qlora_build_info().decode()


def qlora_launch_count():
    return int(lib.qlora_launch_count())


def qlora_profile_enable(enable=True):
    _check(lib.qlora_profile_enable(1 if enable else 0), "qlora_profile_enable")


def qlora_profile_reset():
    _check(lib.qlora_profile_reset(), "qlora_profile_reset")


def qlora_profile_read():
    """{kind: (launches, total_ms)} of the launches recorded since the last reset."""
    n = ctypes.c_int(0)
    cap = 16
    names = (ctypes.c_char_p * cap)()
    counts = (ctypes.c_int * cap)()
    ms = (ctypes.c_double * cap)()
    _check(lib.qlora_profile_read(cap, ctypes.byref(n), names, counts, ms), "qlora_profile_read")
    return {names[i].decode(): (int(counts[i]), float(ms[i])) for i in range(min(n.value, cap))}


# ------------------------------------------------------------------------------ convenience
def alloc_workspace(op, W: Weight, M, r, E=0, device="cuda"):
    """A zero-initialised workspace for `op` (uint8 tensor)."""
    n = qlora_workspace_size(op, W, M, r, E)
    if n == 0:
        raise QLoraError(1, "qlora_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def bf16_from_bits(a, device="cuda"):
    """numpy uint16 bf16 bit patterns -> torch bfloat16 tensor on `device`."""
    return torch.from_numpy(a.view("int16")).view(torch.bfloat16).to(device)


def weight_from_numpy(fmt, codes, scales, tensor_scale=None, device="cuda", scales2=None):
    """Upload a stored weight (numpy arrays as made by synth) to the GPU."""
    import numpy as np
    N = codes.shape[-2]
    K = codes.shape[-1] * 2
    c = torch.from_numpy(codes).to(device)
    s = torch.from_numpy(scales).to(device)
    ts = s2 = None
    if fmt == "nvfp4":
        ts = torch.from_numpy(np.atleast_1d(np.asarray(tensor_scale, np.float32))).to(device)
    if fmt == "nf4dq":
        s2 = torch.from_numpy(np.ascontiguousarray(scales2, np.float32)).to(device)
    return Weight(fmt, N, K, c, s, ts, s2)
