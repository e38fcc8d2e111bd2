"""ctypes wrapper of the fp64 CPU oracle (liboracle.so, built from qlora_oracle.cpp).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg
import this module.  It shares no code with the CUDA path: it takes numpy arrays of the raw
stored bytes (bf16 bit patterns as uint16, packed 4-bit codes as uint8, scales as float32/uint8)
and returns fp64 numpy arrays of the exact definition, or uint16 bf16 bit patterns for the
decoded weight.
"""
import ctypes
import os

import numpy as np

from . import build_oracle

FORMATS = {"nf4": 0, "mxfp4": 1, "nvfp4": 2, "nf4dq": 3}
BLOCK = {0: 64, 1: 32, 2: 16, 3: 64}
DQ_GROUP = 256   # NF4-DQ: first-level constants per fp32 second-level scale


def dq_groups(N, K):
    """Second-level scales of one [N, K] NF4-DQ weight."""
    return (N * (K // 64) + DQ_GROUP - 1) // DQ_GROUP

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        c = ctypes
        L.oracle_nf4_levels_spec.argtypes = [c.c_void_p]
        L.oracle_nf4_levels_as241.argtypes = [c.c_void_p]
        L.oracle_norm_ppf.argtypes = [c.c_double]
        L.oracle_norm_ppf.restype = c.c_double
        for name in ("oracle_decode_e2m1", "oracle_decode_e8m0", "oracle_decode_e4m3"):
            getattr(L, name).argtypes = [c.c_uint32]
            getattr(L, name).restype = c.c_float
        L.oracle_f32_to_bf16.argtypes = [c.c_float]
        L.oracle_f32_to_bf16.restype = c.c_uint16
        L.oracle_bf16_to_f32.argtypes = [c.c_uint16]
        L.oracle_bf16_to_f32.restype = c.c_float
        L.oracle_weight_bytes.argtypes = [c.c_int, c.c_int64, c.c_int64]
        L.oracle_weight_bytes.restype = c.c_int64
        L.oracle_dequant.argtypes = [c.c_int, c.c_int64, c.c_int64, c.c_void_p, c.c_void_p,
                                     c.c_void_p, c.c_float, c.c_int, c.c_void_p]
        L.oracle_dequant.restype = c.c_int
        L.oracle_layer.argtypes = [c.c_int, c.c_int64, c.c_int64, c.c_int64, c.c_int, c.c_double,
                                   c.c_void_p, c.c_void_p, c.c_void_p, c.c_float,
                                   c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                   c.c_void_p, c.c_int64,
                                   c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p,
                                   c.c_void_p, c.c_void_p]
        L.oracle_layer.restype = c.c_int
        L.oracle_num_threads.restype = c.c_int
        L.oracle_encode.argtypes = [c.c_int, c.c_int64, c.c_int64, c.c_void_p, c.c_void_p,
                                    c.c_void_p, c.c_void_p, c.c_void_p]
        L.oracle_encode.restype = c.c_int
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _fmt(fmt):
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def nf4_levels_spec():
    out = np.zeros(16, np.float32)
    lib().oracle_nf4_levels_spec(_ptr(out))
    return out


def nf4_levels_as241():
    out = np.zeros(16, np.float64)
    lib().oracle_nf4_levels_as241(_ptr(out))
    return out


def norm_ppf(p):
    return lib().oracle_norm_ppf(float(p))


def decode_e2m1(code):
    return lib().oracle_decode_e2m1(int(code))


def decode_e8m0(code):
    return lib().oracle_decode_e8m0(int(code))


def decode_e4m3(code):
    return lib().oracle_decode_e4m3(int(code))


def f32_to_bf16(x):
    return lib().oracle_f32_to_bf16(float(np.float32(x)))


def bf16_to_f32(h):
    return lib().oracle_bf16_to_f32(int(h))


def weight_bytes(fmt, N, K):
    return lib().oracle_weight_bytes(_fmt(fmt), int(N), int(K))


def _scales2(scales2):
    return None if scales2 is None else np.ascontiguousarray(scales2, np.float32)


def dequant(fmt, N, K, codes, scales, tensor_scale=1.0, with_tensor_scale=True, scales2=None):
    """Decoded weight [N,K] as bf16 bit patterns (uint16).  scales2: NF4-DQ second-level fp32
    scales [dq_groups(N, K)]."""
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales)
    s2 = _scales2(scales2)
    out = np.zeros((N, K), np.uint16)
    rc = lib().oracle_dequant(_fmt(fmt), N, K, _ptr(codes), _ptr(scales), _ptr(s2),
                              float(tensor_scale), 1 if with_tensor_scale else 0, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_dequant rejected its arguments")
    return out


def layer(fmt, M, N, K, r, s, codes, scales, tensor_scale, X, A, B, dY=None, rows=None,
          want=("Y", "dX", "T", "U", "dA", "dB"), scales2=None):
    """fp64 layer forward + backward.  X/A/B/dY are uint16 bf16 bit patterns.

    rows: optional int64 array of the rows of Y and dX to produce (None: all rows).
    Returns a dict of fp64 arrays for the names in `want`.
    """
    X = np.ascontiguousarray(X, np.uint16)
    A = np.ascontiguousarray(A, np.uint16)
    B = np.ascontiguousarray(B, np.uint16)
    dY = None if dY is None else np.ascontiguousarray(dY, np.uint16)
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nrows = M if rows_arr is None else len(rows_arr)
    out = {}
    out["Y"] = np.zeros((nrows, N)) if "Y" in want else None
    out["dX"] = np.zeros((nrows, K)) if ("dX" in want and dY is not None) else None
    out["T"] = np.zeros((M, r)) if "T" in want else None
    out["U"] = np.zeros((M, r)) if ("U" in want and dY is not None) else None
    out["dA"] = np.zeros((r, K)) if ("dA" in want and dY is not None) else None
    out["dB"] = np.zeros((N, r)) if ("dB" in want and dY is not None) else None
    s2 = _scales2(scales2)
    rc = lib().oracle_layer(_fmt(fmt), M, N, K, r, float(s), _ptr(codes), _ptr(scales), _ptr(s2),
                            float(tensor_scale), _ptr(X), _ptr(A), _ptr(B), _ptr(dY),
                            _ptr(rows_arr), nrows,
                            _ptr(out["Y"]), _ptr(out["dX"]), _ptr(out["T"]), _ptr(out["U"]),
                            _ptr(out["dA"]), _ptr(out["dB"]))
    if rc != 0:
        raise ValueError("oracle_layer rejected its arguments")
    return {k: v for k, v in out.items() if v is not None}


def grouped_layer(fmt, offsets, N, K, r, s, codes, scales, tensor_scales, X, A, B, dY=None,
                  rows_per_expert=None, want=("Y", "dX", "T", "U", "dA", "dB"), scales2=None):
    """The grouped (MoE) layer: the single layer above applied to each expert e on its rows
    [offsets[e], offsets[e+1]) of the packed X / dY with that expert's own weight and adapters.

    codes [E, N, K/2], scales [E, N, K/bs], tensor_scales [E] (NVFP4) or None, A [E, r, K],
    B [E, N, r], scales2 [E, dq_groups(N, K)] (NF4-DQ) or None.  rows_per_expert: optional list
    of local row indices per expert.
    Returns a list of per-expert dicts (row indices in each are local to the expert).
    """
    E = len(offsets) - 1
    res = []
    for e in range(E):
        m0, m1 = int(offsets[e]), int(offsets[e + 1])
        ts = 1.0 if tensor_scales is None else float(tensor_scales[e])
        rows = None if rows_per_expert is None else rows_per_expert[e]
        res.append(layer(fmt, m1 - m0, N, K, r, s, codes[e], scales[e], ts, X[m0:m1], A[e], B[e],
                         None if dY is None else dY[m0:m1], rows=rows, want=want,
                         scales2=None if scales2 is None else scales2[e]))
    return res


def encode(fmt, v):
    """Encode a float weight v [N,K] (float32) per the build's encoder rules.  Returns (codes
    [N,K/2] uint8, scales, tensor_scale (NVFP4, else None), scales2 (NF4-DQ, else None))."""
    f = _fmt(fmt)
    v = np.ascontiguousarray(v, np.float32)
    N, K = v.shape
    bs = BLOCK[f]
    codes = np.zeros((N, K // 2), np.uint8)
    scales = np.zeros((N, K // bs), np.float32 if f == 0 else np.uint8)
    ts = np.zeros(1, np.float32)
    s2 = np.zeros(dq_groups(N, K), np.float32) if f == 3 else None
    rc = lib().oracle_encode(f, N, K, _ptr(v), _ptr(codes), _ptr(scales), _ptr(ts), _ptr(s2))
    if rc != 0:
        raise ValueError("oracle_encode rejected its arguments")
    return codes, scales, (float(ts[0]) if f == 2 else None), s2


def merge(fmt, N, K, codes, scales, tensor_scale, A, B, s, scales2=None):
    """The adapter merged into the stored weight before requantisation, fp32 [N,K]:
    fp32(deq(W)[n,k] + s * sum_j B[n,j] A[j,k]).

    "Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §2 "Deployment: keep or merge": a merge
    adds the low-rank product B A, scaled, to the frozen weight; a quantised base is dequantised
    first and the sum requantised afterwards (encode() of the result).  The sum over
    j runs in order, in binary64 (each product of two bf16 values is exact), then s times it, then
    the decoded weight plus that, rounded to fp32 once.  A [r,K], B [N,r] as bf16 bit patterns."""
    A = np.ascontiguousarray(A, np.uint16)
    B = np.ascontiguousarray(B, np.uint16)
    r = A.shape[0]
    wide = lambda h: (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    w = wide(dequant(fmt, N, K, codes, scales, tensor_scale, scales2=scales2))
    Af, Bf = wide(A), wide(B)
    acc = np.zeros((N, K))
    for j in range(r):
        acc = acc + Bf[:, j:j + 1] * Af[j:j + 1, :]
    return (w + float(np.float32(s)) * acc).astype(np.float32)


def loftq(W, r, s, iters=5, fmt="nf4", quant=None):
    """LoftQ initialisation of the adapter for a quantised base, in fp64.

    "Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §4 "The algorithm: alternating
    quantization and SVD": minimise ||W - Q - s B A||_F by alternating the two sub-problems --
    Q = quantise(W - s B A) with the adapter fixed, then s B A = the best rank-r approximation of
    R = W - Q (Eckart-Young: the top r singular triplets of R) with Q fixed -- starting from
    B A = 0.  One iteration is one quantisation followed by one SVD, so a single iteration of the
    page's 3x3 example already recovers W; the page's default is 5.  The split of the rank-r
    factor follows the page, B = U_r sqrt(Sigma_r / s), A = sqrt(Sigma_r / s) V_r^T, the LoRA
    scale s carried as in the layer (s B A = U_r Sigma_r V_r^T).

    W: float array [N,K] (fp32 values; the quantiser reads W - s B A rounded to fp32).
    quant: optional function v -> decoded array (float64) standing in for the format's encode +
    decode (the page's worked example rounds to integers); default: encode() then dequant() in
    `fmt`, the decoded weight being the bf16 values the layer multiplies by.
    Returns dict: Q (decoded, float64), stored (codes, scales, ts, s2 of the last quantisation,
    or None with `quant`), A [r,K] and B [N,r] (float64, before any rounding to bf16),
    sigma (the top r singular values of the last residual), errs [iters+1]:
    errs[0] = ||W - Q_1|| (the plain QLoRA start, B = 0), errs[t] = ||W - Q_t - s B_t A_t||."""
    W = np.asarray(W, np.float64)
    N, K = W.shape

    def q(v):
        if quant is not None:
            return np.asarray(quant(v), np.float64), None
        st = encode(fmt, v.astype(np.float32))
        d = dequant(fmt, N, K, st[0], st[1], 1.0 if st[2] is None else st[2], scales2=st[3])
        return (d.astype(np.uint32) << 16).view(np.float32).astype(np.float64), st

    Q, stored = q(W)
    errs = [float(np.linalg.norm(W - Q))]
    A = np.zeros((r, K))
    B = np.zeros((N, r))
    sig = np.zeros(r)
    for t in range(1, iters + 1):
        if t > 1:
            Q, stored = q(W - s * (B @ A))
        R = W - Q
        U, S, Vt = np.linalg.svd(R, full_matrices=False)
        sig = S[:r].copy()
        root = np.sqrt(sig / s)
        B = U[:, :r] * root[None, :]
        A = root[:, None] * Vt[:r, :]
        errs.append(float(np.linalg.norm(R - s * (B @ A))))
    return {"Q": Q, "stored": stored, "A": A, "B": B, "sigma": sig, "errs": errs}


def _e4m3_table():
    return np.array([decode_e4m3(c) for c in range(0x7F)], np.float64)   # codes 0..126, ascending


def mxfp8_quantize(x):
    """Activations [M, K] (float) to MXFP8: E4M3 elements with one E8M0 scale per 32 along K.

    For the opt-in native block-scaled MMA forward ("Fine-Tuning 4-Bit Models", "Case 3": a
    W4AFP8 variant of a 4-bit checkpoint), which multiplies 4-bit weight codes by 8-bit
    activations.  The pages fix no rule; this follows the OCP MX shared-exponent rule as the
    weight encoder does for MXFP4: e = clamp(floor(log2 amax) - 8 + 127, 0, 254) (8 = E4M3's
    largest normal exponent; 0 for an all-zero block), elements = nearest E4M3 of x / 2^(e-127),
    ties to the even code, magnitudes saturating at 448, the sign kept only on a non-zero
    magnitude.  Returns (codes uint8 [M, K], scales uint8 [M, K/32])."""
    x = np.asarray(x, np.float64)
    M, K = x.shape
    xb = x.reshape(M, K // 32, 32)
    amax = np.abs(xb).max(axis=2)
    e = np.zeros((M, K // 32), np.int64)
    nz = amax > 0
    e[nz] = np.clip(np.floor(np.log2(amax[nz])).astype(np.int64) - 8 + 127, 0, 254)
    q = xb / np.exp2(e - 127.0)[:, :, None]
    t = _e4m3_table()
    mids = 0.5 * (t[:-1] + t[1:])
    a = np.minimum(np.abs(q), 448.0)
    c = np.searchsorted(mids, a, side="left")          # midpoints strictly below a
    tie = (c < len(mids)) & (a == mids[np.minimum(c, len(mids) - 1)])
    c = np.where(tie & (c % 2 == 1), c + 1, c)         # on a midpoint: the even code
    codes = np.where((c != 0) & (q < 0), c | 0x80, c).astype(np.uint8)
    return codes.reshape(M, K), e.astype(np.uint8)


def mxfp8_dequant(codes, scales):
    """Values of MXFP8 activations (fp64, exact)."""
    codes = np.asarray(codes, np.uint8)
    M, K = codes.shape
    t = _e4m3_table()
    mag = t[(codes & 0x7F).astype(np.int64)]
    v = np.where(codes & 0x80, -mag, mag)
    return (v.reshape(M, K // 32, 32) * np.exp2(np.asarray(scales, np.float64) - 127.0)[:, :, None]
            ).reshape(M, K)


def layer_w4a8_forward(fmt, M, N, K, r, s, codes, scales, tensor_scale, X, A, B):
    """Forward of the opt-in native block-scaled MMA variant, fp64: the base product takes X
    quantised to MXFP8 (mxfp8_quantize of the bf16 X) against the exact weight decode (E2M1 times
    its block scale, times the NVFP4 tensor scale, not rounded to bf16: the block-scaled MMA
    multiplies the codes themselves); the LoRA path is unchanged, T = X A^T from the bf16 X.
    Y = deq8(X) deq(W)^T + s T B^T.  Only MXFP4 and NVFP4 weights (E2M1 codes) apply."""
    if fmt not in ("mxfp4", "nvfp4"):
        raise ValueError("the native FP4 MMA takes E2M1 weight codes (MXFP4, NVFP4)")
    wide = lambda h: (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Xf = wide(X)
    xc, xs = mxfp8_quantize(Xf)
    Xq = mxfp8_dequant(xc, xs)
    # E2M1 x E8M0 and E2M1 x E4M3 are exact in bf16, so the bf16 decode without the tensor scale
    # is the exact block product; the tensor scale is applied in fp64
    Wd = wide(dequant(fmt, N, K, codes, scales, 1.0, with_tensor_scale=False))
    if fmt == "nvfp4":
        Wd = Wd * float(tensor_scale)
    T = Xf @ wide(A).T
    return Xq @ Wd.T + float(np.float32(s)) * (T @ wide(B).T)


def num_threads():
    return lib().oracle_num_threads()
