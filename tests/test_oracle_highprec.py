"""The oracle's FP8 attention against an independent high-precision
re-evaluation of the same rule (the quantized attention has no worked
example on the pages, so this is what pins it beyond its own definition).

The re-evaluation here shares nothing with the oracle's C code:
  - E4M3 values are decoded from the OCP 8-bit floating point definition
    (bias 7, subnormals m/8 * 2^-6) into exact fractions, and the encoder is a
    nearest-value search over that table with ties to the even code;
  - the code dot products are exact integers (every E4M3 value times 2^9 is
    an integer);
  - scores, exponentials, the running maximum, l, P and the output are
    evaluated in 40-digit decimal arithmetic.
The rule (KV tiles of 128 keys, exact running maximum, p = 2^(x - m),
P = E4M3(p * 448 * sv_J / sv_max), l = sum of unquantized p,
out = O * (sv_max / 448) / l) is the reading the oracle follows
("NVIDIA RTX AI optimiert FLUX.1 fuer Bilddaten mit niedriger Genauigkeit",
SDPA quantization paragraph, for the quantized Q, K, V and FP8 attention).
Where a P code lies within binary32 evaluation error of an E4M3 rounding
midpoint the oracle's ambiguity bound is non-zero; those elements are
compared within that bound, every other one to 1e-10.
"""

from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import fqa_synth as synth
import oracle

getcontext().prec = 40
LN2 = Decimal(2).ln()
LOG2E = 1 / LN2


def _e4m3_table():
    """Exact values of the 256 E4M3 codes (None for the two NaN codes)."""
    t = []
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 0xF, c & 7
        if e == 15 and m == 7:
            t.append(None)
            continue
        v = Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        t.append(-v if s else v)
    return t


TABLE = _e4m3_table()
POS = sorted((v, c) for c, v in enumerate(TABLE) if v is not None and v >= 0 and c < 128)


def _encode_nonneg(x: Decimal) -> Fraction:
    """Round-to-nearest-even E4M3 value of x >= 0 (saturating at 448)."""
    xf = Fraction(x)
    if xf >= POS[-1][0]:
        return POS[-1][0]
    lo = max(i for i, (v, _) in enumerate(POS) if v <= xf)
    v0, c0 = POS[lo]
    v1, c1 = POS[lo + 1]
    if xf - v0 < v1 - xf:
        return v0
    if xf - v0 > v1 - xf:
        return v1
    return v0 if c0 % 2 == 0 else v1


def _dec(f) -> Decimal:
    f = Fraction(f)
    return Decimal(f.numerator) / Decimal(f.denominator)


def _reference_rows(qz, h, rows, scale, bc=128):
    q8, k8, v8 = qz["q8"][0, h], qz["k8"][0, h], qz["v8"][0, h]
    sq, sk, sv, svmax = qz["sq"][0, h], qz["sk"][0, h], qz["sv"][0, h], float(qz["sv_max"][0, h])
    N, d = q8.shape
    ints = np.array([int(v * 512) if v is not None else 0 for v in TABLE], dtype=np.int64)
    qi, ki = ints[q8], ints[k8]
    S = qi[rows] @ ki.T                       # exact: code values x 2^9, products x 2^18
    vvals = [[_dec(TABLE[c]) for c in row] for row in v8]
    sc, s2 = _dec(Fraction(float(np.float32(scale)))), Decimal(2) ** -18
    out = []
    for r, i in enumerate(rows):
        a_i = _dec(Fraction(float(sq[i // 64]))) * sc * LOG2E * s2
        m, l = None, Decimal(0)
        acc = [Decimal(0)] * d
        for t0 in range(0, N, bc):
            xs = [Decimal(int(S[r, j])) * a_i * _dec(Fraction(float(sk[j // 64])))
                  for j in range(t0, min(t0 + bc, N))]
            m_new = max(xs) if m is None else max(m, max(xs))
            if m is not None:
                alpha = ((m - m_new) * LN2).exp()
                l *= alpha
                acc = [a * alpha for a in acc]
            for jj, x in enumerate(xs):
                j = t0 + jj
                p = ((x - m_new) * LN2).exp()
                P = _dec(_encode_nonneg(p * 448 * _dec(Fraction(float(sv[j // 64]))) / _dec(Fraction(svmax))))
                l += p
                if P:
                    vj = vvals[j]
                    acc = [a + P * vj[c] for c, a in enumerate(acc)]
            m = m_new
        fin = _dec(Fraction(svmax)) / 448 / l
        out.append([float(a * fin) for a in acc])
    return np.array(out)


@pytest.mark.parametrize("h", [0, 1])
def test_oracle_fp8_matches_high_precision_reevaluation(h):
    w = synth.workload("tiny_n256")
    g = synth.generate(w)
    qz = oracle.quantize(g["q"], g["k"], g["v"])
    scale = oracle.softmax_scale()
    rows = [0, 1, 63, 64, 130, 200, 255]
    ref = _reference_rows(qz, h, rows, scale)
    got, amb, _ = oracle.attention_fp8(qz, scale, heads=[(0, h)], rows=rows, with_ambiguity=True)
    err = np.abs(got[0] - ref)
    assert np.all(err <= 1e-10 * np.maximum(1.0, np.abs(ref)) + amb[0]), float(err.max())


def test_oracle_fp8_ragged_length_matches_high_precision_reevaluation():
    """N = 200: a short last 64-token block (8 tokens) and a short last KV tile
    (72 keys); the re-evaluation runs the rule over the keys that exist."""
    w = synth.workload("tiny_n256")
    g = synth.generate(w)
    q, k, v = (np.ascontiguousarray(g[t][:, :, :200]) for t in "qkv")
    qz = oracle.quantize(q, k, v)
    assert qz["sq"].shape == (1, 2, 4)
    scale = oracle.softmax_scale()
    rows = [0, 127, 128, 191, 192, 199]
    ref = _reference_rows(qz, 1, rows, scale)
    got, amb, _ = oracle.attention_fp8(qz, scale, heads=[(0, 1)], rows=rows, with_ambiguity=True)
    err = np.abs(got[0] - ref)
    assert np.all(err <= 1e-10 * np.maximum(1.0, np.abs(ref)) + amb[0]), float(err.max())


def test_encoder_table_against_the_oracle_codec():
    """The decimal-side codec agrees with the oracle's on a sweep of values
    (ties included), so the comparison above tests the attention rule and not
    two codecs against each other."""
    xs = [Fraction(k, 64) for k in range(0, 64 * 16)] + [Fraction(k, 8) for k in range(0, 8 * 448 + 1, 3)]
    got = oracle.e4m3_encode(np.array([float(x) for x in xs], dtype=np.float32))
    for x, c in zip(xs, got):
        assert TABLE[int(c)] == _encode_nonneg(_dec(x)), (x, int(c))
