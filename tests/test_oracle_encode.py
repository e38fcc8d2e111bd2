"""Pins of the oracle's encoders (float weight -> stored codes and scales) against brute-force
nearest-value searches, numpy's log2 and exact tie cases (CPU only).

The encode rules are this build's reading (the pages print none): nearest representable value,
ties to the lower NF4 code and to the even E2M1/E4M3 code, saturating, scales as stated in
include/qlora.h.  Each pin restates the rule differently from the oracle (an argmin over every
candidate instead of the oracle's midpoint walk), so a wrong midpoint, index or tie direction in
the oracle fails here."""
import math

import numpy as np
import pytest

from oracle import oracle as O


def _unpack(codes, N, K):
    c = np.empty((N, K), np.int64)
    c[:, 0::2], c[:, 1::2] = codes & 15, codes >> 4
    return c


def _argmin_ties(cands, x, prefer):
    """Index of the candidate nearest to x (float64); at an exact tie the index prefer() picks."""
    d = np.abs(np.asarray(cands, np.float64) - x)
    best = np.flatnonzero(d == d.min())
    return prefer(best)


E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E4M3_POS = np.array([O.decode_e4m3(c) for c in range(0x7F)], np.float64)


def _e2m1_code(x):
    m = _argmin_ties(E2M1_MAG, min(abs(x), 6.0), lambda b: b[(b % 2) == 0][0] if (b % 2 == 0).any() else b[0])
    return m | 8 if (m != 0 and math.copysign(1.0, x) < 0) else m


def _e4m3_code(q):
    return _argmin_ties(E4M3_POS, min(q, 448.0), lambda b: b[(b % 2) == 0][0] if (b % 2 == 0).any() else b[0])


def test_encode_nf4_brute_force():
    rng = np.random.default_rng(11)
    N, K = 6, 512
    v = (rng.standard_normal((N, K)) * 0.03).astype(np.float32)
    v[2, 64:128] = 0.0                                   # an all-zero block
    codes, absmax, _, _ = O.encode("nf4", v)
    c = _unpack(codes, N, K)
    L = O.nf4_levels_spec().astype(np.float64)
    assert np.array_equal(absmax, np.abs(v.reshape(N, K // 64, 64)).max(axis=2))
    for n in range(N):
        for k in range(K):
            a = float(absmax[n, k // 64])
            if a == 0.0:
                assert c[n, k] == 7
            else:
                assert c[n, k] == _argmin_ties(L * a, float(v[n, k]), lambda b: b[0])


def test_encode_mxfp4_scale_and_ties():
    rng = np.random.default_rng(12)
    N, K = 4, 256
    v = (rng.standard_normal((N, K)) * np.exp2(rng.integers(-30, 30, size=(N, 1)))).astype(np.float32)
    # block (0, 0): amax in [4, 8) (e = 127, scale 1) and every E2M1 midpoint as an element
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.75, -2.5, -0.25, 7.0, -7.5]   # |v| < 8: e = 127
    v[0, :32] = 0.0
    v[0, 0] = 4.0
    v[0, 1:1 + len(ties)] = ties
    v[1, 32:64] = 0.0                                    # an all-zero block: e = 0
    codes, e, _, _ = O.encode("mxfp4", v)
    c = _unpack(codes, N, K)
    amax = np.abs(v.reshape(N, K // 32, 32)).max(axis=2).astype(np.float64)
    with np.errstate(divide="ignore"):
        want_e = np.where(amax > 0, np.clip(np.floor(np.log2(amax)) - 2 + 127, 0, 254), 0)
    assert np.array_equal(e.astype(np.int64), want_e.astype(np.int64))
    assert e[0, 0] == 127 and e[1, 1] == 0
    want_ties = [0, 2, 2, 4, 4, 6, 6, 8 | 2, 8 | 4, 0, 7, 8 | 7]
    assert list(c[0, 1:1 + len(ties)]) == want_ties
    for n in range(N):
        for k in range(K):
            sc = math.ldexp(1.0, int(e[n, k // 32]) - 127)
            assert c[n, k] == _e2m1_code(float(v[n, k]) / sc)


def test_encode_nvfp4_brute_force():
    rng = np.random.default_rng(13)
    N, K = 8, 128
    v = (rng.standard_normal((N, K)) * 0.05).astype(np.float32)
    v[3, 16:32] = 0.0
    codes, sb, ts, _ = O.encode("nvfp4", v)
    c = _unpack(codes, N, K)
    T = float(np.abs(v).max())
    assert ts == float(np.float32(T / 2688.0))
    amax = np.abs(v.reshape(N, K // 16, 16)).max(axis=2).astype(np.float64)
    for n in range(N):
        for b in range(K // 16):
            assert sb[n, b] == _e4m3_code(amax[n, b] / (6.0 * ts))
    for n in range(N):
        for k in range(K):
            d = float(E4M3_POS[sb[n, k // 16]]) * ts
            want = _e2m1_code(float(v[n, k]) / d) if d > 0 else 0
            assert c[n, k] == want


def test_encode_e4m3_ties_to_even():
    # block absmax values placed exactly halfway between E4M3 neighbours (s_t chosen so that
    # amax / (6 s_t) is exact): the block code must be the even one of the two
    vals = [(0x38, 0x39), (0x39, 0x3A), (0x07, 0x08), (0x00, 0x01), (0x7D, 0x7E)]
    N, K = len(vals), 32
    T = 448.0 * 6.0 * 0.5                       # s_t = T / 2688 = 0.5 exactly: q = amax / 3
    v = np.zeros((N, K), np.float32)
    for i, (lo, hi) in enumerate(vals):
        q = 0.5 * (O.decode_e4m3(lo) + O.decode_e4m3(hi))
        v[i, 0] = np.float32(q * 3.0)
        assert float(v[i, 0]) == q * 3.0          # the tie is representable
    v[0, 16] = T                                 # puts the tensor amax at T (own block)
    _, sb, ts, _ = O.encode("nvfp4", v)
    assert ts == 0.5
    for i, (lo, hi) in enumerate(vals):
        assert sb[i, 0] == (lo if lo % 2 == 0 else hi)


def test_encode_nf4dq_brute_force():
    rng = np.random.default_rng(14)
    N, K = 9, 64 * 70                             # 630 blocks: 3 groups, straddling rows
    v = (rng.standard_normal((N, K)) * np.exp2(rng.integers(-4, 4, size=(N, 1))) * 0.01).astype(np.float32)
    codes, c1, _, s2 = O.encode("nf4dq", v)
    c = _unpack(codes, N, K)
    a = np.abs(v.reshape(N, K // 64, 64)).max(axis=2).reshape(-1).astype(np.float32)
    G = O.dq_groups(N, K)
    assert len(s2) == G == 3
    L = O.nf4_levels_spec().astype(np.float64)
    for g in range(G):
        gmax = a[g * 256:(g + 1) * 256].max()
        assert s2[g] == np.float32(gmax / np.float32(448.0))
    f = np.arange(a.size)
    for i in range(a.size):
        assert c1.reshape(-1)[i] == _e4m3_code(float(a[i]) / float(s2[f[i] // 256]))
    dec = (np.array([O.decode_e4m3(int(x)) for x in c1.reshape(-1)], np.float32) *
           s2[f // 256]).astype(np.float32).reshape(N, K // 64)
    for n in range(N):
        for k in range(0, K, 7):
            d = float(dec[n, k // 64])
            want = _argmin_ties(L * d, float(v[n, k]), lambda b: b[0]) if d > 0 else 7
            assert c[n, k] == want


@pytest.mark.parametrize("fmt", ["nf4", "nf4dq", "mxfp4", "nvfp4"])
def test_encode_decode_error_bound(fmt):
    # decode(encode(v)) is within half the largest gap of the format's grid times the block scale
    rng = np.random.default_rng(15)
    N, K = 16, 512
    v = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    codes, scales, ts, s2 = O.encode(fmt, v)
    w = O.dequant(fmt, N, K, codes, scales, 1.0 if ts is None else ts, scales2=s2)
    wf = (w.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bs = {"nf4": 64, "nf4dq": 64, "mxfp4": 32, "nvfp4": 16}[fmt]
    amax = np.repeat(np.abs(v.reshape(N, K // bs, bs)).max(axis=2), bs, axis=1).astype(np.float64)
    # largest half gap relative to the block amax: NF4 (levels in [-1, 1]) < 0.2; E2M1 with its
    # scale rounding (amax <= 6 * scale * 2): < 2 / 6 + a bf16 ulp
    bound = {"nf4": 0.2, "nf4dq": 0.22, "mxfp4": 0.34, "nvfp4": 0.2}[fmt]
    assert np.all(np.abs(wf - v) <= bound * amax + 1e-12)


def test_encode_mxfp4_round_trip_of_decoded_weight():
    # an MXFP4-decoded weight is exactly representable again: encoding it and decoding the result
    # gives it back bit for bit (the new block exponent may be finer when the block's largest
    # code is small, but every E2M1 value times a power of two stays on the finer grid); equal as
    # values: code 8 (-0) comes back as +0, the encoder gives the sign only to non-zero magnitudes
    rng = np.random.default_rng(16)
    N, K = 8, 256
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    e = rng.integers(100, 150, size=(N, K // 32)).astype(np.uint8)
    w = O.dequant("mxfp4", N, K, codes, e)
    wf = (w.astype(np.uint32) << 16).view(np.float32)
    c2, e2, _, _ = O.encode("mxfp4", wf)
    w2 = (O.dequant("mxfp4", N, K, c2, e2).astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(w2, wf)
    assert not np.any(_unpack(c2, N, K) == 8)


try:
    from hypothesis import given, settings, strategies as st
except ImportError:                                  # pragma: no cover
    given = None


if given is not None:
    @settings(max_examples=25, deadline=None, derandomize=True)
    @given(fmt=st.sampled_from(["nf4", "mxfp4", "nvfp4"]), rows=st.integers(1, 3),
           blocks=st.integers(1, 3), log_scale=st.integers(-40, 40), seed=st.integers(0, 2**31))
    def test_encode_random_shapes_and_scales(fmt, rows, blocks, log_scale, seed):
        # random shapes (K a multiple of 64) and magnitudes from 2^-40 to 2^40: every code is the
        # brute-force nearest value under the format's block scale
        rng = np.random.default_rng(seed)
        N, K = rows, 64 * blocks
        v = (rng.standard_normal((N, K)) * math.ldexp(1.0, log_scale)).astype(np.float32)
        codes, scales, ts, _ = O.encode(fmt, v)
        c = _unpack(codes, N, K)
        if fmt == "nf4":
            L = O.nf4_levels_spec().astype(np.float64)
            for n in range(N):
                for k in range(K):
                    a = float(scales[n, k // 64])
                    assert c[n, k] == (_argmin_ties(L * a, float(v[n, k]), lambda b: b[0]) if a > 0 else 7)
        elif fmt == "mxfp4":
            for n in range(N):
                for k in range(K):
                    sc = math.ldexp(1.0, int(scales[n, k // 32]) - 127)
                    assert c[n, k] == _e2m1_code(float(v[n, k]) / sc)
        else:
            for n in range(N):
                for k in range(K):
                    d = float(E4M3_POS[scales[n, k // 16]]) * ts
                    assert c[n, k] == (_e2m1_code(float(v[n, k]) / d) if d > 0 else 0)
