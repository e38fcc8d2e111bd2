"""Seeded synthetic inputs for the 4-bit-base LoRA linear (tests and benchmark).

This module only *makes inputs*: bf16 activations and adapters, and frozen weights already in
their stored 4-bit form (packed codes + block scales).  It holds none of the layer's arithmetic:
it never decodes a weight and never computes an output, so no expected value can come from here.
To turn a float weight matrix into stored codes it carries simple encoders (quantisers); those sit
outside the layer (the layer only ever decodes), and whatever codes they pick are valid inputs
that the CUDA path and the oracle then decode independently.  These encoders are not the
library's quantiser (qlora_quantize, tested against the oracle's own encoder) and need not agree
with it.

All draws use numpy PCG64 with seed = 1000*seed_id + 10*proj + tensor_id (seed_id: the workload's)
(tensor ids: X=1, W=2, A=3, B=4, dY=5, routing=6), then round to bf16 (round-to-nearest-even).

Layouts (row-major, K contiguous):
  X [M,K], A [r,K], B [N,r], dY [M,N]      uint16 bf16 bit patterns
  codes [N,K/2] uint8: element 2j in the low nibble of byte j, 2j+1 in the high nibble
  scales: NF4 float32 [N,K/64]; MXFP4 uint8 E8M0 [N,K/32]; NVFP4 uint8 E4M3 [N,K/16]
  tensor_scale (NVFP4 only): float32 decode multiplier
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from functools import lru_cache

import numpy as np
import torch

FORMATS = ("nf4", "mxfp4", "nvfp4")
FMT_ID = {"nf4": 0, "mxfp4": 1, "nvfp4": 2}
BLOCK = {"nf4": 64, "mxfp4": 32, "nvfp4": 16}
TID = {"X": 1, "W": 2, "A": 3, "B": 4, "dY": 5, "routing": 6}


def rng_for(seed_id: int, tensor: str, proj: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 * seed_id + 10 * proj + TID[tensor]))


# ---------------------------------------------------------------------------------------------
# bf16 bit patterns
# ---------------------------------------------------------------------------------------------
def to_bf16_bits(x) -> np.ndarray:
    """float -> bf16 bit patterns (uint16), round to nearest even; NaN kept as a quiet NaN.

    Normal numbers, zeros and infinities go through torch's CPU conversion (round to nearest
    even, multi-threaded); fp32 subnormals and NaNs, which a vectorised conversion may flush or
    canonicalise, are rounded from their bit patterns here."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    out = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out = out.reshape(f.shape)
    a = np.abs(f)
    odd = ~(a >= np.float32(1.17549435e-38)) & (f != 0)      # subnormal or NaN
    if odd.any():
        u = f.view(np.uint32)[odd].astype(np.uint64)
        nan = np.isnan(f[odd])
        r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
        r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
        out[odd] = r
    return out


def bf16_bits_to_f32(h) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def pack_nibbles(c: np.ndarray) -> np.ndarray:
    """[N,K] codes 0..15 -> [N,K/2] bytes, element 2j in the low nibble."""
    c = np.asarray(c, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


# ---------------------------------------------------------------------------------------------
# Encoders (test-data quantisers; the layer never runs these)
# ---------------------------------------------------------------------------------------------
@lru_cache(maxsize=1)
def _nf4_grid() -> np.ndarray:
    # The generator's own approximate NF4 grid (any grid gives valid codes).
    from scipy.special import ndtri
    d = 0.5 * (1 / 30 + 1 / 32)
    pos = ndtri(np.linspace(1 - d, 0.5, 9)[:-1])
    neg = -ndtri(np.linspace(1 - d, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, neg, [0.0]]))
    return v / np.abs(v).max()


_E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e2m1_code(x: np.ndarray) -> np.ndarray:
    """Round to the nearest E2M1 value, ties to the even code, saturating at +-6."""
    mag = np.minimum(np.abs(x), 6.0)
    mids = 0.5 * (_E2M1_MAG[1:] + _E2M1_MAG[:-1])
    lo = np.searchsorted(mids, mag, side="left")       # index of nearest, ties -> lower
    tie = np.zeros_like(lo, dtype=bool)
    inb = lo < len(mids)
    tie[inb] = mag[inb] == mids[lo[inb]]
    code = lo.copy()
    # at an exact midpoint between codes lo and lo+1 pick the one with mantissa bit 0
    code[tie & (lo % 2 == 1)] += 1
    sign = (np.signbit(x) & (code > 0)).astype(np.uint8)
    return (code.astype(np.uint8) | (sign << 3)).astype(np.uint8)


def _e4m3_table():
    vals = []
    for b in range(0x7F):  # positive finite codes 0x00..0x7e
        e, m = b >> 3, b & 7
        vals.append((m / 8) * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


_E4M3 = _e4m3_table()


def _e4m3_code(v: np.ndarray) -> np.ndarray:
    """Positive float -> nearest E4M3 code (ties to even code), saturating at 448."""
    v = np.minimum(np.asarray(v, np.float64), 448.0)
    idx = np.clip(np.searchsorted(_E4M3, v, side="left"), 1, len(_E4M3) - 1)
    lo, hi = _E4M3[idx - 1], _E4M3[idx]
    pick_hi = (hi - v < v - lo) | ((hi - v == v - lo) & (idx % 2 == 0))
    return np.where(pick_hi, idx, idx - 1).astype(np.uint8)


def encode(fmt: str, W: np.ndarray):
    """Quantise a float weight [N,K] -> (codes [N,K/2], scales, tensor_scale).

    Rows are independent given the (NVFP4) tensor scale, so row chunks are encoded on a thread
    pool; the result does not depend on the chunking."""
    W = np.asarray(W, np.float32)
    N, K = W.shape
    bs = BLOCK[fmt]
    assert K % bs == 0
    ts = None
    if fmt == "nvfp4":
        tmax = float(np.abs(W).max())
        ts = np.float32(tmax / (6 * 448)) if tmax > 0 else np.float32(1.0)
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, K // bs), np.float32 if fmt == "nf4" else np.uint8)
    step = max(1, min(N, (1 << 21) // K))

    def run(n0):
        n1 = min(N, n0 + step)
        codes[n0:n1], scales[n0:n1] = _encode_rows(fmt, W[n0:n1], ts)

    starts = range(0, N, step)
    if len(starts) > 1:
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(run, starts))
    else:
        run(0)
    return codes, scales, ts


def _encode_rows(fmt: str, W: np.ndarray, ts):
    N, K = W.shape
    bs = BLOCK[fmt]
    Wb = W.reshape(N, K // bs, bs)
    amax = np.abs(Wb).max(axis=2)
    if fmt == "nf4":
        grid = _nf4_grid()
        mids = 0.5 * (grid[1:] + grid[:-1])
        absmax = amax.astype(np.float32)
        safe = np.where(absmax > 0, absmax, 1.0)[:, :, None]
        x = (Wb / safe).astype(np.float64)
        c = np.searchsorted(mids, x, side="left").astype(np.uint8)
        c[np.broadcast_to(absmax[:, :, None] == 0, c.shape)] = 7
        return pack_nibbles(c.reshape(N, K)), absmax
    if fmt == "mxfp4":
        with np.errstate(divide="ignore"):
            e = np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2 + 127
        e = np.where(amax > 0, np.clip(e, 0, 254), 0).astype(np.uint8)
        scale = np.exp2(e.astype(np.float64) - 127)[:, :, None]
        c = _e2m1_code(Wb / scale)
        return pack_nibbles(c.reshape(N, K)), e
    # nvfp4
    sb = _e4m3_code(amax / (6 * float(ts)))
    sval = _E4M3[sb.astype(np.int64)] * float(ts)
    safe = np.where(sval > 0, sval, 1.0)[:, :, None]
    c = _e2m1_code(Wb / safe)
    c[np.broadcast_to(sval[:, :, None] == 0, c.shape)] = 0
    return pack_nibbles(c.reshape(N, K)), sb


DQ_GROUP = 256   # NF4 with double quantisation: first-level codes per fp32 second-level scale


def encode_nf4dq(W: np.ndarray):
    """Quantise a float weight [N,K] to NF4 with a double-quantised absmax -> (codes [N,K/2],
    first-level E4M3 codes [N,K/64] uint8, second-level fp32 scales [ceil(N*K/64 / 256)]).

    Test-data encoder (its choices are not part of the decode definition): the 64-block absmax
    is fp32 max|w|; every 256 consecutive absmax values (row-major) share s2 = max / 448; the
    first-level code is the nearest E4M3 of absmax / s2; the 4-bit codes are the nearest NF4
    levels of w / (decoded absmax)."""
    W = np.asarray(W, np.float32)
    N, K = W.shape
    assert K % 64 == 0
    nb = K // 64
    Wb = W.reshape(N, nb, 64)
    amax = np.abs(Wb).max(axis=2).astype(np.float32).reshape(-1)
    G = (amax.size + DQ_GROUP - 1) // DQ_GROUP
    pad = np.zeros(G * DQ_GROUP, np.float32)
    pad[:amax.size] = amax
    gmax = pad.reshape(G, DQ_GROUP).max(axis=1)
    s2 = np.where(gmax > 0, gmax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    s2_el = np.repeat(s2, DQ_GROUP)[:amax.size]
    c1 = _e4m3_code(amax / s2_el)
    absmax_d = (_E4M3[c1.astype(np.int64)].astype(np.float32) * s2_el).astype(np.float32)
    absmax_d = absmax_d.reshape(N, nb)
    grid = _nf4_grid()
    mids = 0.5 * (grid[1:] + grid[:-1])
    safe = np.where(absmax_d > 0, absmax_d, np.float32(1.0))[:, :, None]
    x = (Wb / safe).astype(np.float64)
    c = np.searchsorted(mids, x, side="left").astype(np.uint8)
    c[np.broadcast_to(absmax_d[:, :, None] == 0, c.shape)] = 7
    return pack_nibbles(c.reshape(N, K)), c1.reshape(N, nb), s2


def random_stored_weight(fmt: str, N: int, K: int, rng: np.random.Generator,
                         scale_codes=None):
    """Uniformly random codes and scales (every code and every scale pattern reachable).

    scale_codes: optional explicit array of scale values to draw from (E8M0/E4M3 bytes, or NF4
    float absmax values)."""
    bs = BLOCK[fmt]
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    nb = (N, K // bs)
    if fmt == "nf4":
        pool = (np.asarray(scale_codes, np.float32) if scale_codes is not None
                else np.float32(rng.uniform(0.0, 0.1, size=64)))
        scales = pool[rng.integers(0, len(pool), size=nb)].astype(np.float32)
        return codes, scales, None
    if fmt == "mxfp4":
        pool = np.arange(100, 140) if scale_codes is None else np.asarray(scale_codes)
        return codes, pool[rng.integers(0, len(pool), size=nb)].astype(np.uint8), None
    pool = np.arange(0x20, 0x58) if scale_codes is None else np.asarray(scale_codes)
    return codes, pool[rng.integers(0, len(pool), size=nb)].astype(np.uint8), np.float32(0.75)


# ---------------------------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------------------------
@dataclass
class Proj:
    name: str
    N: int
    K: int


@dataclass
class Config:
    seed_id: int
    fmt: str
    M: int
    projs: list
    r: int
    alpha: float
    w_dist: str = "normal"          # "normal": N(0, 0.02); "t5": 0.02 * Student-t(5)
    x_std: float = 1.0
    dy_std: float = 0.01
    b_std: float = 0.01
    experts: int = 0                # > 0: grouped (MoE)
    tokens: int = 0
    topk: int = 0
    zipf: float = 1.1
    desc: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return self.alpha / self.r


WORKLOADS = {
    "nf4_1024x1024": Config(1, "nf4", 256, [Proj("proj", 1024, 1024)], 16, 32.0, dy_std=1.0,
              desc="single LoRA linear, NF4, M=256, N=K=1024, r=16"),
    "llama3_8b_up_nf4": Config(2, "nf4", 4096, [Proj("up", 14336, 4096)], 64, 128.0,
              desc="Llama-3-8B-shaped MLP up-proj, NF4, M=4096, N=14336, K=4096, r=64"),
    "llama3_70b_gate_mxfp4": Config(3, "mxfp4", 8192, [Proj("gate", 28672, 8192)], 16, 32.0, w_dist="t5",
              desc="Llama-3-70B-shaped MLP gate-proj, MXFP4, M=8192, N=28672, K=8192, r=16"),
    "llama3_70b_layer_nvfp4": Config(4, "nvfp4", 4096,
              [Proj("q", 8192, 8192), Proj("k", 1024, 8192), Proj("v", 1024, 8192),
               Proj("o", 8192, 8192), Proj("gate", 28672, 8192), Proj("up", 28672, 8192),
               Proj("down", 8192, 28672)], 16, 32.0,
              desc="Llama-3-70B-shaped decoder layer, 7 NVFP4 projections, M=4096, r=16"),
    "moe64_mxfp4": Config(5, "mxfp4", 131072,
              [Proj("gate", 2048, 7168), Proj("up", 2048, 7168), Proj("down", 7168, 2048)],
              8, 16.0, experts=64, tokens=16384, topk=8,
              desc="MoE grouped experts, 64 x {gate,up 2048x7168; down 7168x2048}, MXFP4, "
                   "16384 tokens x top-8, r=8"),
}


def _normal(rng, shape, std):
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def make_weight(cfg: Config, proj: int, N: int, K: int, experts: int = 0):
    """Stored weight of projection `proj` ([E,...] stacked when experts > 0)."""
    rng = rng_for(cfg.seed_id, "W", proj)
    E = max(experts, 1)
    codes = np.empty((E, N, K // 2), np.uint8)
    scales = None
    ts = np.ones(E, np.float32)
    for e in range(E):
        if cfg.w_dist == "t5":
            W = (rng.standard_t(5, size=(N, K)) * 0.02).astype(np.float32)
        else:
            W = _normal(rng, (N, K), 0.02)
        c, s, t = encode(cfg.fmt, W)
        del W
        if scales is None:
            scales = np.empty((E,) + s.shape, s.dtype)
        codes[e], scales[e] = c, s
        if t is not None:
            ts[e] = t
    if experts == 0:
        return codes[0], scales[0], float(ts[0])
    return codes, scales, ts


def make_adapters(cfg: Config, proj: int, N: int, K: int, experts: int = 0):
    E = max(experts, 1)
    ra, rb = rng_for(cfg.seed_id, "A", proj), rng_for(cfg.seed_id, "B", proj)
    bound = 1.0 / math.sqrt(K)   # Kaiming-uniform (a = sqrt 5) bound for fan-in K
    A = to_bf16_bits(ra.uniform(-bound, bound, size=(E, cfg.r, K)).astype(np.float32))
    B = to_bf16_bits(_normal(rb, (E, N, cfg.r), cfg.b_std))
    return (A[0], B[0]) if experts == 0 else (A, B)


def make_activations(cfg: Config, proj: int, M: int, N: int, K: int):
    X = to_bf16_bits(_normal(rng_for(cfg.seed_id, "X", proj), (M, K), cfg.x_std))
    dY = to_bf16_bits(_normal(rng_for(cfg.seed_id, "dY", proj), (M, N), cfg.dy_std))
    return X, dY


def moe_routing(cfg: Config):
    """Per-expert token counts: each token takes `topk` distinct experts by Gumbel-top-k over
    Zipf(s) weights p_e ~ rank_e^-s, ranks assigned by a seeded random permutation.
    Returns int64 offsets [E+1] (exclusive prefix sum, offsets[E] = tokens * topk)."""
    rng = rng_for(cfg.seed_id, "routing")
    E = cfg.experts
    ranks = rng.permutation(E) + 1
    logp = -cfg.zipf * np.log(ranks.astype(np.float64))
    counts = np.zeros(E, np.int64)
    chunk = 4096
    for t0 in range(0, cfg.tokens, chunk):
        n = min(chunk, cfg.tokens - t0)
        g = rng.gumbel(size=(n, E))
        top = np.argpartition(-(logp[None, :] + g), cfg.topk, axis=1)[:, :cfg.topk]
        counts += np.bincount(top.ravel(), minlength=E)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    return offsets


def layer_inputs(name: str, proj: int = 0, M: int | None = None):
    """Inputs of one (non-grouped) projection: dict with fmt, M, N, K, r, s, codes, scales,
    tensor_scale, X, A, B, dY."""
    cfg = WORKLOADS[name]
    p = cfg.projs[proj]
    M = cfg.M if M is None else M
    codes, scales, ts = make_weight(cfg, proj, p.N, p.K)
    A, B = make_adapters(cfg, proj, p.N, p.K)
    X, dY = make_activations(cfg, proj, M, p.N, p.K)
    return dict(fmt=cfg.fmt, M=M, N=p.N, K=p.K, r=cfg.r, s=cfg.scale, codes=codes, scales=scales,
                tensor_scale=ts, X=X, A=A, B=B, dY=dY)


def small_layer(fmt: str, M: int, N: int, K: int, r: int, s: float = 2.0, seed: int = 0,
                random_codes: bool = False, x_std=1.0, dy_std=1.0, b_std=0.01):
    """A small seeded problem for parity tests (W ~ N(0, 0.02) quantised, or random codes).
    fmt "nf4dq" (NF4 with double-quantised absmax) adds scales2, the second-level scales."""
    rng = np.random.Generator(np.random.PCG64(seed))
    scales2 = None
    if fmt == "nf4dq":
        codes, scales, scales2 = encode_nf4dq(_normal(rng, (N, K), 0.02))
        ts = 1.0
    elif random_codes:
        codes, scales, ts = random_stored_weight(fmt, N, K, rng)
        ts = 1.0 if ts is None else float(ts)
    else:
        codes, scales, ts = encode(fmt, _normal(rng, (N, K), 0.02))
        ts = 1.0 if ts is None else float(ts)
    bound = 1.0 / math.sqrt(K)
    A = to_bf16_bits(rng.uniform(-bound, bound, size=(r, K)).astype(np.float32))
    B = to_bf16_bits(_normal(rng, (N, r), b_std))
    X = to_bf16_bits(_normal(rng, (M, K), x_std))
    dY = to_bf16_bits(_normal(rng, (M, N), dy_std))
    return dict(fmt=fmt, M=M, N=N, K=K, r=r, s=s, codes=codes, scales=scales, tensor_scale=ts,
                scales2=scales2, X=X, A=A, B=B, dY=dY)


def small_grouped(fmt: str, counts, N: int, K: int, r: int, s: float = 2.0, seed: int = 0,
                  b_std=0.01):
    """A small seeded grouped (MoE) problem: expert e owns counts[e] consecutive rows of the packed
    activations.  Expert e's weight is N(0, 0.02 * (1 + e % 3)) quantised, so NVFP4 experts get
    different tensor scales.  Returns a dict with offsets int64 [E+1] and stacked arrays."""
    rng = np.random.Generator(np.random.PCG64(seed))
    E = len(counts)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(np.asarray(counts, np.int64))
    M = int(offsets[-1])
    codes = np.empty((E, N, K // 2), np.uint8)
    scales = None
    scales2 = None
    ts = np.ones(E, np.float32)
    for e in range(E):
        if fmt == "nf4dq":
            c, sc, s2 = encode_nf4dq(_normal(rng, (N, K), 0.02 * (1 + e % 3)))
            if scales2 is None:
                scales2 = np.empty((E,) + s2.shape, np.float32)
            scales2[e] = s2
            t = None
        else:
            c, sc, t = encode(fmt, _normal(rng, (N, K), 0.02 * (1 + e % 3)))
        if scales is None:
            scales = np.empty((E,) + sc.shape, sc.dtype)
        codes[e], scales[e] = c, sc
        if t is not None:
            ts[e] = t
    bound = 1.0 / math.sqrt(K)
    A = to_bf16_bits(rng.uniform(-bound, bound, size=(E, r, K)).astype(np.float32))
    B = to_bf16_bits(_normal(rng, (E, N, r), b_std))
    X = to_bf16_bits(_normal(rng, (M, K), 1.0))
    dY = to_bf16_bits(_normal(rng, (M, N), 1.0))
    return dict(fmt=fmt, E=E, offsets=offsets, M=M, N=N, K=K, r=r, s=s, codes=codes,
                scales=scales, tensor_scale=ts if fmt == "nvfp4" else None, scales2=scales2,
                X=X, A=A, B=B, dY=dY)
