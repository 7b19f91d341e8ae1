"""Writes the quotient cases of ``quant_examples.json`` with exact rational arithmetic.

The INT8 and E4M3 quantisers divide each value by a block or channel scale that
is itself a rounded float32 quotient (s = amax / 127, or amax / 448), and the
definition asks for the correctly rounded float32 quotient x / s before the
final rounding to a code.  Scales that are powers of two cannot tell that
quotient apart from cheaper stand-ins, so this script picks values whose code
changes if the quotient is replaced by

  * x * RN(1 / s)          (multiplying by a rounded reciprocal),
  * x * RN(127 / amax)     (folding the scale into one rounded factor),
  * RN(x * 127) / amax     (the operations in the other order).

Every expected code is derived here from the definition with
``fractions.Fraction`` (exact rationals, rounding written out), never from the
oracle: ``RN`` rounds an exact rational to the nearest float32 with ties to even,
and the code is the nearest integer (INT8, ties to even, clamped to +-127) or
the nearest E4M3 value (OCP E4M3, ties to the even code, saturating at 448).

Run ``python tests/golden/make_quant_quotient_cases.py`` to rewrite the two
lists in place; the test ``tests/test_oracle_quant.py`` recomputes each case
the same way and checks the oracle against it.
"""

from __future__ import annotations

import json
import os
import struct
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))
PATH = os.path.join(HERE, "quant_examples.json")


def f32(v: float) -> float:
    """The float32 value nearest to a Python float (the inputs below are float32-exact)."""
    return struct.unpack("<f", struct.pack("<f", v))[0]


def rn32(q: Fraction) -> Fraction:
    """Exact rational q rounded to the nearest float32 (ties to even); normal range only."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    assert -126 <= e <= 127, "only normal float32 results are used here"
    quantum = Fraction(2) ** (e - 23)
    return sign * round(a / quantum) * quantum      # Fraction.__round__ ties to even


def int8_code(y: Fraction) -> int:
    return max(-127, min(127, round(y)))            # ties to even


def e4m3_value(y: Fraction) -> Fraction:
    """Nearest E4M3 value to y (ties to the even code), saturating at +-448."""
    sign = -1 if y < 0 else 1
    a = min(abs(y), Fraction(448))
    if a < Fraction(1, 64):
        quantum = Fraction(1, 512)                  # subnormals: spacing 2^-9
    else:
        e = 0
        while Fraction(2) ** (e + 1) <= a:
            e += 1
        while Fraction(2) ** e > a:
            e -= 1
        quantum = Fraction(2) ** (e - 3)            # three mantissa bits
    n = round(a / quantum)
    return sign * min(n * quantum, Fraction(448))


def e4m3_code(y: Fraction) -> int:
    v = e4m3_value(y)
    s = 0x80 if (v < 0 or (v == 0 and y < 0)) else 0
    a = abs(v)
    if a < Fraction(1, 64):
        return s | int(a * 512)
    e = 0
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    while Fraction(2) ** e > a:
        e -= 1
    m = int((a / Fraction(2) ** e - 1) * 8)
    return s | ((e + 7) << 3) | m


def next_up(x: float, k: int) -> float:
    """The float32 k steps above x (k may be negative); x > 0."""
    b = struct.unpack("<I", struct.pack("<f", x))[0] + k
    return struct.unpack("<f", struct.pack("<I", b))[0]


def variants(x: float, amax: float, qmax: int):
    """Rounded float32 values of the exact quotient and of its three stand-ins."""
    X, A, Q = Fraction(x), Fraction(amax), Fraction(qmax)
    s = rn32(A / Q)
    return {
        "quotient": rn32(X / s),
        "times_reciprocal": rn32(X * rn32(1 / s)),
        "times_folded_factor": rn32(X * rn32(Q / A)),
        "multiply_first": rn32(rn32(X * Q) / A),
    }


KINDS = ("times_reciprocal", "times_folded_factor", "multiply_first")


def find_cases(amax: float, qmax: int, code, centres, per_kind=2):
    """Values x (|x| < amax) near rounding boundaries whose code differs from the
    exact-quotient code for at least one stand-in, until every stand-in is caught
    per_kind times.  Returns [(x, code, {stand-in: its code})]."""
    found, seen, count = [], set(), dict.fromkeys(KINDS, 0)
    for c in centres:
        x0 = f32(float(c))
        for k in range(-3, 4):
            x = next_up(x0, k)
            if x in seen or not (0 < x < amax):
                continue
            seen.add(x)
            v = variants(x, amax, qmax)
            want = code(v["quotient"])
            wrong = {kind: code(v[kind]) for kind in KINDS if code(v[kind]) != want}
            if any(count[kind] < per_kind for kind in wrong):
                found.append((x, want, wrong))
                for kind in wrong:
                    count[kind] += 1
        if all(n >= per_kind for n in count.values()):
            break
    return found


def dump(d):
    """JSON with one line per example (the file's hand-written layout)."""
    out = ["{"]
    keys = list(d)
    for i, key in enumerate(keys):
        sep = "," if i + 1 < len(keys) else ""
        val = d[key]
        if isinstance(val, list):
            out.append(f" {json.dumps(key)}: [")
            for j, item in enumerate(val):
                out.append("  " + json.dumps(item, ensure_ascii=False) +
                           ("," if j + 1 < len(val) else ""))
            out.append(" ]" + sep)
        else:
            out.append(f" {json.dumps(key)}: {json.dumps(val, ensure_ascii=False)}{sep}")
    out.append("}")
    return "\n".join(out) + "\n"


def main():
    d = json.load(open(PATH))
    # INT8: amax 100, s = RN(100 / 127) (not a power of two); the values sit near
    # (n + 1/2) * s, where the rounding of the quotient decides the code.
    amax_i = 100.0
    s_i = rn32(Fraction(amax_i) / 127)
    centres = [(n + Fraction(1, 2)) * s_i for n in range(0, 126)]
    int8 = [{"x": [amax_i, x], "scale": float(s_i), "codes": [127, want], "wrong": wrong,
             "why": f"s = RN(100/127); the rounded quotient RN(x/s) gives code {want}"}
            for x, want, wrong in find_cases(amax_i, 127, int8_code, centres)]
    # E4M3: one channel with amax 300, s = RN(300 / 448); the values sit near the
    # midpoints of neighbouring E4M3 values times s.
    amax_e = 300.0
    s_e = rn32(Fraction(amax_e) / 448)
    grid = sorted({e4m3_value(Fraction(n, 64)) for n in range(1, 448 * 64)})
    mids = [(a + b) / 2 * s_e for a, b in zip(grid[:-1], grid[1:]) if b <= 448]
    e4 = [{"v": [amax_e, x], "scale": float(s_e), "codes": [0x7E, want], "wrong": wrong,
           "why": f"s = RN(300/448); E4M3 of the rounded quotient RN(v/s) is code {want:#04x}"}
          for x, want, wrong in find_cases(amax_e, 448, e4m3_code, mids)]
    d["int8_quotient"] = int8
    d["e4m3_quotient"] = e4
    d["about_quotient"] = ("int8_quotient / e4m3_quotient: one block (INT8) or one channel (E4M3) "
                           "holding amax and x; expected codes derived with exact rational "
                           "arithmetic by make_quant_quotient_cases.py, chosen so that "
                           "multiplying by a rounded reciprocal or folded factor, or multiplying "
                           "before dividing, gives another code ('wrong').")
    with open(PATH, "w") as f:
        f.write(dump(d))
    print(f"{len(int8)} INT8 and {len(e4)} E4M3 quotient cases")


if __name__ == "__main__":
    main()
