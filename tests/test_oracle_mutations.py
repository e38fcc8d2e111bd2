"""The oracle's pins catch plausible mistakes: each case plants one mistake in a copy of an
oracle function (a dropped term, a wrong split, a missing step, an off-by-one exponent, a wrong
tie direction), installs it in place of the original for the duration of the case, and checks that
at least one of the pins written for that function then fails.  CPU only; the oracle itself is
not modified."""
import numpy as np
import pytest

from oracle import oracle as O
import test_oracle_loftq as TL
import test_oracle_merge as TM
import test_oracle_w4a8 as TW

_orig_merge, _orig_loftq, _orig_q8 = O.merge, O.loftq, O.mxfp8_quantize


def _merge_without_scale(fmt, N, K, codes, scales, tensor_scale, A, B, s, scales2=None):
    return _orig_merge(fmt, N, K, codes, scales, tensor_scale, A, B, 1.0, scales2=scales2)


def _merge_with_dropped_rank(fmt, N, K, codes, scales, tensor_scale, A, B, s, scales2=None):
    A = np.ascontiguousarray(A, np.uint16)[:-1] if np.asarray(A).shape[0] > 1 else np.zeros_like(A)
    B = np.ascontiguousarray(B, np.uint16)[:, :-1] if np.asarray(B).shape[1] > 1 else np.zeros_like(B)
    return _orig_merge(fmt, N, K, codes, scales, tensor_scale, A, B, s, scales2=scales2)


def _loftq_split_without_scale(W, r, s, iters=5, fmt="nf4", quant=None):
    res = _orig_loftq(W, r, s, iters, fmt, quant)
    root = np.sqrt(s)                     # B = U sqrt(S), A = sqrt(S) V^T: s B A = s L
    res["B"], res["A"] = res["B"] * root, res["A"] * root
    return res


def _loftq_without_requantisation(W, r, s, iters=5, fmt="nf4", quant=None):
    res = _orig_loftq(W, r, s, 1, fmt, quant)
    res["errs"] = res["errs"] + [res["errs"][-1]] * (iters - 1)
    return res


def _q8_emax7(x):
    # the shared exponent one too large (E4M3's largest exponent taken as 7): the block scale is
    # doubled, the elements are quantised against it
    x = np.asarray(x, np.float64)
    _, e = _orig_q8(x)
    e2 = np.where(e > 0, np.minimum(e.astype(np.int64) + 1, 254), 0).astype(np.uint8)
    M, K = x.shape
    shift = np.repeat(e2.astype(np.float64) - e.astype(np.float64), 32, axis=1)
    codes, _ = _orig_q8(x / np.exp2(shift))               # x at the doubled scale, same exponent
    return codes, e2


def _q8_ties_lower(x):
    codes, e = _orig_q8(x)
    x = np.asarray(x, np.float64)
    M, K = x.shape
    q = np.abs(x.reshape(M, K // 32, 32) / np.exp2(e.astype(np.float64) - 127.0)[:, :, None]).reshape(M, K)
    t = np.array([O.decode_e4m3(c) for c in range(0x7F)])
    mids = 0.5 * (t[:-1] + t[1:])
    on_mid = np.isin(q, mids)
    lower = np.searchsorted(mids, q, side="left")
    mag = np.where(on_mid, lower, codes & 0x7F)
    return np.where(codes & 0x80, mag | 0x80, mag).astype(np.uint8), e


CASES = [
    ("merge", _merge_without_scale, [TM.test_merge_cancelling_adapter_gives_zero,
                                     lambda: TM.test_merge_matches_float64_matmul("nf4")]),
    ("merge", _merge_with_dropped_rank, [lambda: TM.test_merge_matches_float64_matmul("nvfp4")]),
    ("loftq", _loftq_split_without_scale, [lambda: TL.test_loftq_worked_example(2.0)]),
    ("loftq", _loftq_without_requantisation, [TL.test_loftq_alternation_is_monotone_with_an_exact_projection]),
    ("mxfp8_quantize", _q8_emax7, [TW.test_mxfp8_quantize_brute_force]),
    ("mxfp8_quantize", _q8_ties_lower, [TW.test_mxfp8_quantize_brute_force]),
]


@pytest.mark.parametrize("name,mutant,pins", CASES, ids=[f"{c[0]}-{c[1].__name__}" for c in CASES])
def test_pins_catch_planted_mistake(monkeypatch, name, mutant, pins):
    for pin in pins:                                       # the pins pass on the real oracle
        pin()
    monkeypatch.setattr(O, name, mutant)
    caught = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin caught {mutant.__name__}"
