"""Pins of the oracle's format decoding against hand-worked tables, closed forms, invariants and
independent library decoders (CPU only).

Each test would fail under a plausible slip in the oracle: a wrong bias or subnormal rule (the
exhaustive E4M3/E8M0 cross-checks against torch's own fp8 decoders), a swapped nibble order
(test_nibble_order), a wrong NF4 level (the AS 241 recomputation and scipy's ndtri), an extra
rounding step in the decode chain (test_dequant_* compare against torch's binary32 multiply and
bf16 rounding)."""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from oracle import oracle as O


# ---------------------------------------------------------------- element and scale decodes
def test_e2m1_hand_table():
    for code, val in read_golden("e2m1_values.txt"):
        got = O.decode_e2m1(int(code))
        want = float(val)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (code, got, want)


def test_scale_hand_table():
    for fmt, code, val in read_golden("scale_values.txt"):
        c = int(code, 0)
        got = O.decode_e8m0(c) if fmt == "e8m0" else O.decode_e4m3(c)
        want = float(val)
        if math.isnan(want):
            assert math.isnan(got), (fmt, code)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want), (fmt, code, got)


def test_e4m3_exhaustive_vs_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        got = O.decode_e4m3(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c] and math.copysign(1, got) == math.copysign(1, ref[c]), c


def test_e8m0_exhaustive_vs_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).float().numpy()
    for c in range(256):
        got = O.decode_e8m0(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c], c
    # closed form over the finite range
    for c in range(255):
        assert O.decode_e8m0(c) == math.ldexp(1.0, c - 127)


def test_e2m1_invariants():
    vals = [O.decode_e2m1(c) for c in range(16)]
    assert vals[:8] == sorted(vals[:8]) and len(set(vals[:8])) == 8
    for c in range(8):                       # sign bit mirrors every magnitude
        assert vals[c + 8] == -vals[c]
    assert math.copysign(1, vals[8]) == -1.0  # code 8 is -0


# ---------------------------------------------------------------- NF4 levels
def test_nf4_levels_match_fixture_and_as241():
    spec = O.nf4_levels_spec()
    rows = read_golden("nf4_levels.txt")
    want_bits = np.array([int(h, 16) for _, h, _ in rows], np.uint32)
    assert np.array_equal(spec.view(np.uint32), want_bits)
    rec = O.nf4_levels_as241()
    assert np.array_equal(rec.astype(np.float32).view(np.uint32), want_bits)


def test_as241_against_scipy_ndtri():
    from scipy.special import ndtri
    ps = np.concatenate([np.linspace(1e-6, 1 - 1e-6, 501), [1e-12, 1e-30, 0.5, 0.425, 0.075, 0.925,
                                                           1 - 1e-9]])
    for p in ps:
        got, want = O.norm_ppf(p), float(ndtri(p))
        assert abs(got - want) <= 4e-15 * max(1.0, abs(want)), (p, got, want)


def test_nf4_level_invariants():
    v = O.nf4_levels_spec().astype(np.float64)
    assert len(v) == 16 and np.all(np.diff(v) > 0)           # 16 distinct, ascending
    assert v[0] == -1.0 and v[15] == 1.0 and v[7] == 0.0      # normalised by absmax, exact zero
    assert (v < 0).sum() == 7 and (v > 0).sum() == 8
    gaps_pos = np.diff(v[7:])                                 # denser near zero
    gaps_neg = -np.diff(v[:8][::-1])
    assert np.all(np.diff(gaps_pos) > 0) and np.all(np.diff(gaps_neg) > 0)


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_rounding_vs_torch():
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.standard_normal(4000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-38).astype(np.float32),     # subnormal range
        np.array([0.0, -0.0, np.inf, -np.inf, 3.3961e38, -3.3961e38, 1.00390625, 1.01171875,
                  1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 2 ** -133, 2 ** -134, 1e-45], np.float32),
    ])
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([O.f32_to_bf16(x) for x in xs], np.uint16)
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- whole-weight decode
def test_nibble_order():
    # byte 0x21: element 0 is code 1 (low nibble), element 1 is code 2 (high nibble)
    codes = np.zeros((1, 32), np.uint8)
    codes[0, 0] = 0x21
    scales = np.full((1, 2), 127, np.uint8)   # MXFP4: scale 1.0
    out = O.dequant("mxfp4", 1, 64, codes, scales)
    f = (out.astype(np.uint32) << 16).view(np.float32)
    assert f[0, 0] == 0.5 and f[0, 1] == 1.0 and np.all(f[0, 2:] == 0.0)


def _levels32():
    return O.nf4_levels_spec()


def _bf16_bits_of_f32_product(a32, b32):
    """torch binary32 product rounded to bf16 by torch: an independent statement of the
    fp32-then-RNE decode rule."""
    p = torch.from_numpy(np.asarray(a32, np.float32)) * torch.from_numpy(np.asarray(b32, np.float32))
    return p.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_dequant_nf4_brute_force():
    rng = np.random.default_rng(1)
    N, K = 16, 256
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    pool = np.array([0.02, 1.0, 3.0e-39, 1e-41, 7.3e37, 2.5e38, 0.0, 1.234567e-5], np.float32)
    scales = pool[rng.integers(0, len(pool), size=(N, K // 64))]
    out = O.dequant("nf4", N, K, codes, scales)
    c = np.empty((N, K), np.int64)
    c[:, 0::2], c[:, 1::2] = codes & 15, codes >> 4
    lv = _levels32()[c]
    sc = np.repeat(scales, 64, axis=1)
    assert np.array_equal(out, _bf16_bits_of_f32_product(lv, sc))


def test_dequant_mxfp4_exact_closed_form():
    rng = np.random.default_rng(2)
    N, K = 8, 512
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    e = rng.integers(0, 254, size=(N, K // 32), dtype=np.uint8)     # all finite scales
    e[0, 0], e[0, 1] = 0, 253
    out = O.dequant("mxfp4", N, K, codes, e)
    f = (out.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mag = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    c = np.empty((N, K), np.int64)
    c[:, 0::2], c[:, 1::2] = codes & 15, codes >> 4
    val = np.where(c >= 8, -mag[c & 7], mag[c & 7]) * np.exp2(np.repeat(e, 32, 1).astype(np.float64) - 127)
    with np.errstate(invalid="ignore"):
        val = np.where(np.abs(val) > 3.3895313892515355e38, np.sign(val) * np.inf, val)  # bf16 overflow
    assert np.array_equal(f, val)


def test_dequant_mxfp4_scale_edges():
    codes = np.full((1, 32), 0x7F, np.uint8)       # element codes 15 (-6) and 7 (+6)
    for e, expect in [(254, np.inf), (255, np.nan), (0, 6 * 2.0 ** -127)]:
        out = O.dequant("mxfp4", 1, 64, codes, np.full((1, 2), e, np.uint8))
        f = (out.astype(np.uint32) << 16).view(np.float32)
        if np.isnan(expect):
            assert np.all(np.isnan(f))
        else:
            assert f[0, 1] == np.float32(expect) and f[0, 0] == -np.float32(expect)


def test_dequant_nvfp4_block_exact_and_tensor_scale_chain():
    rng = np.random.default_rng(3)
    N, K = 8, 256
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sb = rng.integers(0, 0x7F, size=(N, K // 16), dtype=np.uint8)   # positive finite E4M3
    sb[0, :4] = [0x01, 0x07, 0x08, 0x7E]                            # subnormals and the max
    ts = np.float32(0.0123)
    blk = O.dequant("nvfp4", N, K, codes, sb, ts, with_tensor_scale=False)
    full = O.dequant("nvfp4", N, K, codes, sb, ts, with_tensor_scale=True)
    c = np.empty((N, K), np.int64)
    c[:, 0::2], c[:, 1::2] = codes & 15, codes >> 4
    mag = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    e2 = np.where(c >= 8, -mag[c & 7], mag[c & 7])
    e4 = torch.from_numpy(np.repeat(sb, 16, 1)).view(torch.float8_e4m3fn).double().numpy()
    exact = e2 * e4                                   # E2M1 x E4M3 is exact in bf16
    fb = (blk.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(fb, exact)
    want = _bf16_bits_of_f32_product(exact.astype(np.float32), np.full(exact.shape, ts, np.float32))
    assert np.array_equal(full, want)


def test_weight_bytes_pins_memory_table():
    # NF4 without double quantisation is 4.5 bits per weight: 65B params -> 36.6 GB
    for name, params, bits, gb in read_golden("memory_table.txt"):
        P = int(float(params))
        if name == "nf4":
            N, K = 1000, int(P // 1000)
            K -= K % 64
            nbytes = O.weight_bytes("nf4", N, K)
            assert nbytes * 8 == N * K * 4.5
            assert round(P * 4.5 / 8 / 1e9, 1) == float(gb)
        elif name == "fp16":
            assert round(P * int(bits) / 8 / 1e9, 1) == float(gb)
        elif name == "nf4dq":
            # 8-bit first level per 64 weights + one fp32 per 256 first-level constants
            N, K = 4096, 16384
            bpw = O.weight_bytes("nf4dq", N, K) * 8 / (N * K)
            assert abs(bpw - (4 + 8 / 64 + 32 / (64 * 256))) < 1e-12
            assert round(bpw, 3) == float(bits)
            assert round(P * bpw / 8 / 1e9, 1) == float(gb)
            assert abs((4.5 - bpw) - 0.373) < 5e-4            # "net savings: about 0.373 bits"
    assert O.weight_bytes("mxfp4", 64, 1024) * 8 == 64 * 1024 * 4.25
    assert O.weight_bytes("nvfp4", 64, 1024) * 8 == 64 * 1024 * 4.5 + 32
    assert O.weight_bytes("nf4", 64, 100) == -1                 # K must be a whole number of blocks


# ---------------------------------------------------------------- NF4 with double quantisation
def _e4m3_values32(c1):
    return np.array([O.decode_e4m3(int(v)) for v in np.asarray(c1).reshape(-1)],
                    np.float32).reshape(np.asarray(c1).shape)


def test_dequant_nf4dq_reduces_to_nf4_with_unit_second_level():
    # s2 = 1: the absmax is the first-level E4M3 value itself, so the decode must equal the
    # (separately pinned) NF4 decode with that fp32 absmax, bit for bit, for every E4M3 code
    rng = np.random.default_rng(3)
    N, K = 24, 64 * 64
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    c1 = rng.integers(0, 256, size=(N, K // 64), dtype=np.uint8)
    c1.reshape(-1)[:256] = np.arange(256, dtype=np.uint8)        # every first-level code
    s2 = np.ones(O.dq_groups(N, K), np.float32)
    got = O.dequant("nf4dq", N, K, codes, c1, scales2=s2)
    ref = O.dequant("nf4", N, K, codes, _e4m3_values32(c1))
    assert np.array_equal(got, ref)


def test_dequant_nf4dq_second_level_groups():
    # distinct power-of-two s2 per group (exact products), 300 blocks per row: groups of 256
    # consecutive first-level constants straddle rows.  Each block must take the s2 of its own
    # group, i.e. equal NF4 with absmax = e4m3(c1) * s2[f // 256], f the row-major block index.
    rng = np.random.default_rng(4)
    N, K = 7, 64 * 300
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    c1 = rng.integers(0x20, 0x60, size=(N, K // 64), dtype=np.uint8)
    G = O.dq_groups(N, K)
    assert G == math.ceil(N * 300 / 256)
    s2 = np.ldexp(np.ones(G, np.float32), np.arange(G) - 4).astype(np.float32)
    got = O.dequant("nf4dq", N, K, codes, c1, scales2=s2)
    f = np.arange(N * 300).reshape(N, 300)
    absmax = (_e4m3_values32(c1) * s2[f // 256]).astype(np.float32)
    ref = O.dequant("nf4", N, K, codes, absmax)
    assert np.array_equal(got, ref)
    # and a different group assignment (a shift by one block) would not match
    wrong = (_e4m3_values32(c1) * s2[(f + 1) // 256]).astype(np.float32)
    assert not np.array_equal(got, O.dequant("nf4", N, K, codes, wrong))


def test_nf4dq_encoder_absmax_within_e4m3_bound():
    # the test-data encoder's stored absmax (decoded by the oracle: e4m3(c1) * s2) is within the
    # E4M3 rounding bound (relative 2^-4) of the true block absmax wherever absmax / s2 is in
    # E4M3's normal range
    from bit_quantized_base_b200 import synth
    rng = np.random.default_rng(5)
    N, K = 40, 64 * 50
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    codes, c1, s2 = synth.encode_nf4dq(W)
    true = np.abs(W.reshape(N, 50, 64)).max(axis=2).reshape(-1)
    f = np.arange(true.size)
    dec = _e4m3_values32(c1).reshape(-1).astype(np.float64) * s2[f // 256]
    normal = true / s2[f // 256] >= 2.0 ** -6
    assert normal.mean() > 0.9
    rel = np.abs(dec[normal] - true[normal]) / true[normal]
    assert rel.max() <= 2.0 ** -4 + 1e-7


def test_dequant_rejects_bad_shape():
    with pytest.raises(ValueError):
        O.dequant("nf4", 2, 96, np.zeros((2, 48), np.uint8), np.zeros((2, 2), np.float32))
