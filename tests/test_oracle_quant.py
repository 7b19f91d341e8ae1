"""Pins of the reference quantisers against things other than themselves.

* hand-worked examples in ``golden/quant_examples.json``, including scales that
  are not powers of two, with values whose code changes if the quotient x / s
  is replaced by a multiplication with a rounded reciprocal or folded factor, or
  by multiplying first (expected codes derived with exact rationals by
  ``golden/make_quant_quotient_cases.py``, never by the oracle);
* the E4M3 encoder against an exhaustive nearest-value search over the finite
  codes decoded from the format definition (ties to the even code), on a dense
  sweep of float32 values;
* the E4M3 encoder against torch's CPU float8_e4m3fn cast (an independent
  library routine) inside the finite range;
* INT8 properties: the block maximum maps to +-127, codes stay in range, the
  dequantised error is at most half a step, ties go to even, partial last
  blocks and all-zero blocks;
* V quantiser: transposed layout with zero padding, per-channel scales.
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import (dequantize_qk, dequantize_v, fp8_e4m3_decode, fp8_e4m3_encode, padded_len,
                    quantize_qk_int8, quantize_v_fp8)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_int8_worked_examples():
    d = json.load(open(os.path.join(GOLDEN, "quant_examples.json")))
    for ex in d["int8"]:
        x = np.array(ex["x"], dtype=np.float32).reshape(1, 1, 1, -1)
        codes, scales = quantize_qk_int8(x)
        assert codes.ravel().tolist() == ex["codes"], ex
        assert scales.ravel().tolist() == [ex["scale"]], ex


def test_e4m3_worked_examples():
    d = json.load(open(os.path.join(GOLDEN, "quant_examples.json")))
    for ex in d["e4m3"]:
        got = int(fp8_e4m3_encode(np.float32(ex["x"])))
        assert got == int(ex["code"], 16), ex


def _golden():
    return json.load(open(os.path.join(GOLDEN, "quant_examples.json")))


def _stand_ins(x, amax, qmax):
    """float32 values of the three stand-ins for the quotient x / RN(amax / qmax)."""
    f = np.float32
    x, amax, qmax = f(x), f(amax), f(qmax)
    s = f(amax / qmax)
    return {"times_reciprocal": f(x * f(f(1) / s)),
            "times_folded_factor": f(x * f(qmax / amax)),
            "multiply_first": f(f(x * qmax) / amax)}


def test_int8_quotient_cases():
    import sys
    sys.path.insert(0, GOLDEN)

    import make_quant_quotient_cases as mk
    cases = _golden()["int8_quotient"]
    assert len(cases) >= 3
    caught = set()
    for ex in cases:
        x = np.array(ex["x"], dtype=np.float32).reshape(1, 1, 1, -1)
        codes, scales = quantize_qk_int8(x)
        assert codes.ravel().tolist() == ex["codes"], ex
        assert scales.ravel().tolist() == [ex["scale"]], ex
        amax, xv = ex["x"]
        # the stored code is the exact-rational one, and each listed stand-in gives another
        assert mk.int8_code(mk.variants(xv, amax, 127)["quotient"]) == ex["codes"][1]
        alt = _stand_ins(xv, amax, 127)
        for kind, code in ex["wrong"].items():
            assert int(np.clip(np.rint(alt[kind]), -127, 127)) == code != ex["codes"][1]
            caught.add(kind)
    assert caught == set(mk.KINDS)


def test_e4m3_quotient_cases():
    import sys
    sys.path.insert(0, GOLDEN)

    import make_quant_quotient_cases as mk
    cases = _golden()["e4m3_quotient"]
    assert len(cases) >= 2
    caught = set()
    for ex in cases:
        v = np.array(ex["v"], dtype=np.float32).reshape(1, 1, -1, 1)   # one channel, 2 tokens
        codes, scales = quantize_v_fp8(v)
        assert codes[0, 0, 0, :2].tolist() == ex["codes"], ex
        assert scales.ravel().tolist() == [ex["scale"]], ex
        amax, vv = ex["v"]
        assert mk.e4m3_code(mk.variants(vv, amax, 448)["quotient"]) == ex["codes"][1]
        alt = _stand_ins(vv, amax, 448)
        for kind, code in ex["wrong"].items():
            assert int(fp8_e4m3_encode(alt[kind])) == code != ex["codes"][1]
            caught.add(kind)
    assert caught == set(mk.KINDS)


def test_quotient_cases_catch_a_reciprocal_quantiser():
    # A quantiser that multiplies by RN(1/s) instead of dividing (a plausible slip)
    # fails the quotient cases.
    def int8_by_reciprocal(x):
        x = np.asarray(x, dtype=np.float32)
        s = np.float32(np.abs(x).max() / np.float32(127))
        return np.clip(np.rint(x * np.float32(np.float32(1) / s)), -127, 127).astype(np.int64)
    missed = [ex for ex in _golden()["int8_quotient"]
              if int8_by_reciprocal(ex["x"]).tolist() != ex["codes"]]
    assert missed, "the quotient cases do not tell division from a reciprocal multiply"


def _finite_code_table():
    codes = np.arange(128, dtype=np.uint8)           # non-negative codes
    vals = fp8_e4m3_decode(codes)
    keep = ~np.isnan(vals)
    return codes[keep], vals[keep]


def _nearest_even_search(x):
    """Brute force: nearest finite E4M3 value; ties go to the even code; saturate."""
    codes, vals = _finite_code_table()
    out = np.empty(x.shape, dtype=np.uint8)
    for n, xv in enumerate(x.astype(np.float64)):
        a = min(abs(xv), 448.0)
        dist = np.abs(vals - a)
        best = np.flatnonzero(dist == dist.min())
        if len(best) > 1:
            best = [b for b in best if codes[b] % 2 == 0]
        c = int(codes[best[0]])
        if np.signbit(xv):
            c |= 0x80
        out[n] = c
    return out


def test_e4m3_decode_table():
    codes, vals = _finite_code_table()
    assert len(codes) == 127
    assert vals.max() == 448.0 and vals[1] == 2.0 ** -9 and vals[8] == 2.0 ** -6
    assert np.all(np.diff(vals) > 0)


def test_e4m3_encoder_matches_nearest_search():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.uniform(-500, 500, 3000),
        rng.uniform(-1, 1, 3000) * 2.0 ** rng.integers(-12, 9, 3000),
        # every midpoint between neighbouring codes, and its float32 neighbours
    ]).astype(np.float32)
    _, vals = _finite_code_table()
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    mids = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    x = np.concatenate([x, mids, -mids, vals.astype(np.float32), np.float32([448, 449, 1e30, -1e30])])
    assert np.array_equal(fp8_e4m3_encode(x), _nearest_even_search(x))


def test_e4m3_encoder_matches_torch_cast_in_range():
    rng = np.random.default_rng(12)
    x = np.concatenate([rng.uniform(-448, 448, 200000),
                        rng.standard_normal(200000) * 2.0 ** rng.integers(-14, 8, 200000)]).astype(np.float32)
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8_e4m3_encode(x), ref)


def test_e4m3_sweep_float32_grid():
    # Every float32 in [2^-12, 2^-5) with the 10 low mantissa bits stepped
    # (covers the subnormal/normal boundary and the 2^-9 quantum densely).
    lo = np.float32(2.0 ** -12).view(np.uint32)
    hi = np.float32(2.0 ** -5).view(np.uint32)
    bits = np.arange(lo, hi, 1 << 10, dtype=np.uint32)
    x = bits.view(np.float32)
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8_e4m3_encode(x), ref)


@pytest.mark.parametrize("S,D", [(300, 64), (128, 128), (5, 16)])
def test_int8_block_properties(S, D):
    rng = np.random.default_rng(S + D)
    x = (rng.standard_normal((2, 3, S, D)) * rng.uniform(0.1, 10, (2, 3, 1, 1))).astype(np.float32)
    x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()  # bf16-exact inputs
    codes, scales = quantize_qk_int8(x)
    nblk = (S + 127) // 128
    assert scales.shape == (2, 3, nblk) and codes.dtype == np.int8
    assert np.all(np.abs(codes.astype(np.int32)) <= 127)
    for t in range(nblk):
        blk = x[:, :, t * 128:(t + 1) * 128]
        amax = np.abs(blk).max(axis=(2, 3))
        assert np.array_equal(scales[:, :, t], (amax / np.float32(127)).astype(np.float32))
        cb = codes[:, :, t * 128:(t + 1) * 128]
        # the largest magnitude element maps to +-127
        assert np.all(np.abs(cb.astype(np.int32)).max(axis=(2, 3)) == 127)
    err = np.abs(dequantize_qk(codes, scales) - x)
    step = np.repeat(scales, 128, axis=2)[:, :, :S, None].astype(np.float64)
    # half a step, plus the fp32 rounding of x / s (at most 127 * 2^-24 steps)
    assert np.all(err <= (0.5 + 127 * 2.0 ** -23) * step + 1e-30)


def test_int8_zero_and_partial_blocks():
    x = np.zeros((1, 1, 130, 4), dtype=np.float32)
    x[0, 0, 129, 2] = -3.0           # only the partial second block is nonzero
    codes, scales = quantize_qk_int8(x)
    assert scales[0, 0, 0] == 0 and np.all(codes[0, 0, :128] == 0)
    assert scales[0, 0, 1] == np.float32(3.0) / np.float32(127)
    assert codes[0, 0, 129, 2] == -127


def test_v_quantiser_layout_and_scales():
    rng = np.random.default_rng(13)
    S, D = 200, 8
    v = rng.standard_normal((1, 2, S, D)).astype(np.float32)
    v[0, 1, :, 3] = 0.0  # an all-zero channel
    codes, scales = quantize_v_fp8(v)
    assert codes.shape == (1, 2, D, padded_len(S)) and padded_len(S) == 256
    assert np.all(codes[:, :, :, S:] == 0)
    assert scales[0, 1, 3] == 0 and np.all(codes[0, 1, 3] == 0)
    amax = np.abs(v).max(axis=2)
    assert np.array_equal(scales, (amax / np.float32(448)).astype(np.float32))
    # each channel's largest magnitude maps to +-448 exactly
    dec = fp8_e4m3_decode(codes[:, :, :, :S])
    for b in range(1):
        for h in range(2):
            for c in range(D):
                if scales[b, h, c] > 0:
                    assert np.abs(dec[b, h, c]).max() == 448.0
    # dequantised values are within half an E4M3 step (relative 2^-4) or the subnormal step
    back = dequantize_v(codes, scales, S)
    tol = np.maximum(np.abs(v) * 2.0 ** -4, scales[:, :, None, :] * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(back - v) <= tol)
    # code of channel c, token j sits at [.., c, j]
    direct = fp8_e4m3_encode((v[0, 0, 17, 5] / scales[0, 0, 5]).astype(np.float32))
    assert codes[0, 0, 5, 17] == direct
