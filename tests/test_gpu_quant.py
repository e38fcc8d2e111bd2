"""The GPU quantiser (float weight -> stored codes and scales) and the merge of a trained adapter
with requantisation, against the oracle bit for bit (integer and byte results: exact).

"Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §3 "The setup" (the base is quantised once,
before training) and §2 "Deployment: keep or merge" (W' = W + (alpha/r) B A, requantised for a
quantised base); "Fine-Tuning 4-Bit Models", "Case 2" / "Case 3" (requantising a merged result to
NVFP4 / MXFP4).  Both sides follow the same stated encode rules; every quotient is binary64 on
both, so the comparison is exact, not within a tolerance."""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from bit_quantized_base_b200 import synth

pytestmark = pytest.mark.gpu

FMTS = ["nf4", "nf4dq", "mxfp4", "nvfp4"]
BS = {"nf4": 64, "nf4dq": 64, "mxfp4": 32, "nvfp4": 16}


def _Q():
    from bit_quantized_base_b200 import qlora as Q
    return Q


def _weight_v(N, K, seed):
    """Seeded float weight: N(0, 0.02) rows at scales 2^-3..2^3, with the special blocks the
    encoders treat apart (a zero block, a zero row, fp32 subnormals, exact NF4 and E2M1
    midpoints under MXFP4 and NVFP4 scales)."""
    rng = np.random.default_rng(seed)
    v = (rng.standard_normal((N, K)) * 0.02 * np.exp2(rng.integers(-3, 4, size=(N, 1)))).astype(np.float32)
    v[1, 64:128] = 0.0                                        # one zero block in every format
    v[2, :] = 0.0                                             # a zero row
    v[3, :64] = (rng.standard_normal(64) * 1e-41).astype(np.float32)   # subnormals: MXFP4 e = 0
    v[4, :32] = 0.0                                           # MXFP4 block with amax 4 (e = 127)
    v[4, 0] = 4.0
    v[4, 1:13] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.75, -2.5, -0.25, 7.0, -7.5]
    # NF4 block with absmax 1 holding the four NF4 level midpoints that binary32 represents
    # exactly: each is a tie, which goes to the lower code
    v[5, :64] = 0.0
    v[5, 0] = 1.0
    v[5, 1:5] = [-0.45999518036842346, -0.04552498832345009, 0.03979015722870827,
                 0.861478328704834]
    # NVFP4: the tensor max 1344 (s_t = 1344 / 2688 = 0.5) and a 16-block with amax 3 (block
    # scale exactly 1, element step d = 0.5) holding every E2M1 midpoint times d: ties to even
    v[7, 32:48] = 0.0
    v[7, 32] = 1344.0
    v[6, :16] = 0.0
    v[6, 0] = 3.0
    v[6, 1:15] = [0.125, 0.375, 0.625, 0.875, 1.25, 1.75, 2.5,
                  -0.125, -0.375, -0.625, -0.875, -1.25, -1.75, -2.5]
    return v


def _stored(W):
    """The GPU weight's arrays as numpy (codes, scales, tensor scale or None, scales2 or None)."""
    ts = None if W.tensor_scale is None else float(W.tensor_scale.cpu().numpy()[0])
    s2 = None if W.scales2 is None else W.scales2.cpu().numpy()
    return W.codes.cpu().numpy(), W.scales.cpu().numpy(), ts, s2


def _assert_same_encoding(fmt, got, want, rows=None):
    gc, gs, gts, gs2 = got
    wc, ws, wts, ws2 = want
    sl = slice(None) if rows is None else rows
    assert np.array_equal(gc[sl], wc), f"{fmt}: codes differ at {np.argwhere(gc[sl] != wc)[:5]}"
    if fmt == "nf4":
        assert np.array_equal(gs[sl].view(np.uint32), ws.view(np.uint32)), f"{fmt}: absmax differ"
    else:
        assert np.array_equal(gs[sl], ws), f"{fmt}: block scales differ"
    if fmt == "nvfp4":
        assert np.float32(gts).view(np.uint32) == np.float32(wts).view(np.uint32), (gts, wts)
    if fmt == "nf4dq" and rows is None:
        assert np.array_equal(gs2.view(np.uint32), ws2.view(np.uint32)), f"{fmt}: scales2 differ"


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("shape", [(48, 704), (64, 1024), (16, 64)])
def test_quantize_matches_oracle(fmt, shape):
    # (48, 704): block counts 528 / 1056 / 2112 -- several CTAs and a ragged last one; rows
    # straddle the NF4-DQ groups.  (64, 1024): rows 16..31 zero make NF4-DQ group 1 all zero.
    # (16, 64): one CTA, fewer blocks than threads.
    Q = _Q()
    N, K = shape
    v = _weight_v(N, K, 21)
    if shape == (64, 1024):
        v[16:32] = 0.0
    W = Q.empty_weight(fmt, N, K)
    Q.qlora_quantize(W, torch.from_numpy(v).cuda())
    torch.cuda.synchronize()
    want = O.encode(fmt, v)
    _assert_same_encoding(fmt, _stored(W), want)
    if fmt == "nf4dq" and shape == (64, 1024):
        assert want[3][1] == 1.0
    c = want[0]
    lo, hi = c & 15, c >> 4
    if fmt == "nf4":          # ties to the lower code: levels 2, 6, 7, 14 (not 3, 7, 8, 15)
        assert [int(x) for x in (hi[5, 0], lo[5, 1], hi[5, 1], lo[5, 2])] == [2, 6, 7, 14]
    if fmt == "nvfp4":        # ties to the even E2M1 code; -0.125 rounds to magnitude 0: +0
        assert want[2] == 0.5 and int(want[1][6, 0]) == 0x38
        got = [int(x) for x in np.stack([lo[6, :8], hi[6, :8]], 1).reshape(-1)[1:15]]
        assert got == [0, 2, 2, 4, 4, 6, 6, 0, 10, 10, 12, 12, 14, 14]


@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_bf16_input(fmt):
    Q = _Q()
    N, K = 32, 512
    v = _weight_v(N, K, 22)
    vb = torch.from_numpy(v).to(torch.bfloat16)
    W = Q.empty_weight(fmt, N, K)
    Q.qlora_quantize(W, vb.cuda())
    torch.cuda.synchronize()
    _assert_same_encoding(fmt, _stored(W), O.encode(fmt, vb.float().numpy()))


@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_full_size(fmt):
    # the Llama-3-8B-shaped up-projection weight (N=14336, K=4096), every byte compared
    Q = _Q()
    N, K = 14336, 4096
    rng = np.random.default_rng(23)
    v = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W = Q.empty_weight(fmt, N, K)
    Q.qlora_quantize(W, torch.from_numpy(v).cuda())
    torch.cuda.synchronize()
    _assert_same_encoding(fmt, _stored(W), O.encode(fmt, v))


def test_quantize_rejects_bad_arguments():
    Q = _Q()
    W = Q.empty_weight("nf4", 32, 128)
    v = torch.zeros((32, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(RuntimeError):
        Q.qlora_quantize(W, v.view(torch.uint8).view(-1)[1:])                 # v misaligned
    bad = Q.Weight("nf4", 32, 100, W.codes, W.scales)                        # K % 64 != 0
    with pytest.raises(RuntimeError):
        Q.qlora_quantize(bad, v)
    dq = Q.Weight("nf4dq", 32, 128, W.codes, W.scales.view(torch.uint8), None, None)  # no scales2
    with pytest.raises(RuntimeError):
        Q.qlora_quantize(dq, v)


def _merge_problem(fmt_in, N, K, r, seed):
    rng = np.random.default_rng(seed)
    codes, scales, ts, s2 = O.encode(fmt_in, (rng.standard_normal((N, K)) * 0.02).astype(np.float32))
    bound = 1.0 / np.sqrt(K)
    A = synth.to_bf16_bits(rng.uniform(-bound, bound, size=(r, K)).astype(np.float32))
    B = synth.to_bf16_bits((rng.standard_normal((N, r)) * 0.05).astype(np.float32))
    return codes, scales, (1.0 if ts is None else ts), s2, A, B


def _gpu_merge(fmt_in, fmt_out, N, K, r, s, codes, scales, ts, s2, A, B):
    Q = _Q()
    W = Q.weight_from_numpy(fmt_in, codes, scales, ts, "cuda", scales2=s2)
    W_out = Q.empty_weight(fmt_out, N, K)
    merged = torch.empty((N, K), dtype=torch.float32, device="cuda")
    Q.qlora_merge_requantize(W, Q.bf16_from_bits(A, "cuda"), Q.bf16_from_bits(B, "cuda"), r, s,
                             W_out, merged)
    torch.cuda.synchronize()
    return merged.cpu().numpy(), _stored(W_out)


@pytest.mark.parametrize("fmt_in,fmt_out,r", [
    ("nf4", "nf4", 64), ("nf4dq", "nf4dq", 16), ("mxfp4", "mxfp4", 64), ("nvfp4", "nvfp4", 64),
    ("nf4", "nvfp4", 8), ("mxfp4", "nf4", 1), ("nvfp4", "mxfp4", 3)])
def test_merge_requantize_matches_oracle(fmt_in, fmt_out, r):
    N, K, s = 48, 704, 2.0
    codes, scales, ts, s2, A, B = _merge_problem(fmt_in, N, K, r, 31)
    merged, got = _gpu_merge(fmt_in, fmt_out, N, K, r, s, codes, scales, ts, s2, A, B)
    want_m = O.merge(fmt_in, N, K, codes, scales, ts, A, B, s, scales2=s2)
    assert np.array_equal(merged.view(np.uint32), want_m.view(np.uint32)), \
        np.argwhere(merged != want_m)[:5]
    _assert_same_encoding(fmt_out, got, O.encode(fmt_out, want_m))


@pytest.mark.parametrize("fmt", ["nf4", "nf4dq", "mxfp4"])
def test_merge_requantize_full_size_sampled(fmt):
    # Llama-3-8B-shaped up-projection (N=14336, K=4096, r=64): the merge and the NF4 / MXFP4
    # encodes are row-local, NF4-DQ's groups are 4 whole rows here, so sampled 4-row slices
    # (group-aligned) are checked against the oracle run on those rows alone
    N, K, r, s = 14336, 4096, 64, 2.0
    codes, scales, ts, s2, A, B = _merge_problem(fmt, N, K, r, 32)
    merged, got = _gpu_merge(fmt, fmt, N, K, r, s, codes, scales, ts, s2, A, B)
    per_group = 256 // (K // 64)
    for n0 in (0, 4, 7164, N - 4):
        rows = slice(n0, n0 + 4)
        g = None if s2 is None else s2[n0 // per_group:(n0 + 4) // per_group]
        want_m = O.merge(fmt, 4, K, codes[rows], scales[rows], ts, A, B[rows], s, scales2=g)
        assert np.array_equal(merged[rows].view(np.uint32), want_m.view(np.uint32)), n0
        want = O.encode(fmt, want_m)
        _assert_same_encoding(fmt, got, want, rows=rows)
        if fmt == "nf4dq":
            assert np.array_equal(got[3][n0 // per_group:(n0 + 4) // per_group].view(np.uint32),
                                  want[3].view(np.uint32))
