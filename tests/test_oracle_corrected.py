"""Pins for the oracle's error-corrected FP8 attention ("FLUX 3 Image Klein
Base: 생성 3.46배, 8장 확장 병목", section "왜 이런 차이가 나나": VC-Attention
FP8 corrects only the tokens with large error, rho = 0.005).

Readings under test: the corrected tokens are the ceil(rho*N) keys per head
with the largest quantization error (squared distance between the smoothed
key and its dequantized code, binary32, pinned order); their part of the
softmax is exact, the rest follows the FP8 rule, and the two partial
softmaxes are merged by their maxima and row sums."""

import numpy as np
import pytest
import scipy.special

import fqa_synth as s
import oracle

LOG2E = 1.4426950408889634


def _bf16(x):
    return s.round_to_bf16_bits(np.asarray(x, dtype=np.float64))


# ------------------------------------------------------------- key error

def _order_block():
    # One 64-token block, scale s = 1 (amax = 448 in channel 1), every channel
    # summing to zero over the block so k_mean = 0 exactly.  Token 0:
    #   ch 0:  432 -> RNE tie between 416 (odd mantissa) and 448 -> 448, r = -16, r^2 = 256
    #   ch 8, ch 72: 2^-4 + 2^-8 -> tie between 2^-4 and 2^-4 + 2^-7 -> 2^-4, r^2 = 2^-16
    # Token 1 holds the negated values (same squares).
    k = np.zeros((1, 1, 64, 128))
    for c, x in ((0, 432.0), (1, 448.0), (8, 2.0 ** -4 + 2.0 ** -8), (72, 2.0 ** -4 + 2.0 ** -8)):
        k[0, 0, 0, c] = x
        k[0, 0, 1, c] = -x
    return _bf16(k)


def test_key_error_pinned_order_hand_case():
    # Pinned order: group sums g_i over channels 8i..8i+7, then
    # a_i = g_i + g_i+8, b_i = a_i + a_i+4, c_i = b_i + b_i+2, e = c_0 + c_1:
    #   g0 = 256, g1 = g9 = 2^-16 -> a1 = 2^-15 -> c1 = 2^-15 -> e = 256 + 2^-15
    # (exact).  A sequential channel sum would absorb each 2^-16 into 256
    # (ties to even) and give 256.
    k = _order_block()
    qz = oracle.quantize(k, k, k)
    assert qz["sk"][0, 0, 0] == 1.0 and np.all(qz["k_mean"] == 0)
    err = oracle.key_error(k, qz)
    assert err[0, 0, 0] == np.float32(256.0 + 2.0 ** -15)
    assert err[0, 0, 1] == np.float32(256.0 + 2.0 ** -15)
    assert np.all(err[0, 0, 2:] == 0)


def test_key_error_zero_for_exactly_representable_keys():
    # s = 1 and every value an E4M3 code: the dequantized key is the key.
    rng = np.random.default_rng(40)
    vals = np.array([0, 1, 1.5, 2, 3.5, 8, 12, 26, 64, 96, 240, 448], dtype=np.float64)
    x = rng.choice(vals, size=(1, 1, 32, 128)) * rng.choice([-1.0, 1.0], size=(1, 1, 32, 128))
    x[0, 0, 0, 0] = 448.0
    k = np.concatenate([x, -x], axis=2)              # channel means exactly 0
    kb = _bf16(k)
    qz = oracle.quantize(kb, kb, kb)
    assert np.all(qz["k_mean"] == 0) and qz["sk"][0, 0, 0] == 1.0
    assert np.all(oracle.key_error(kb, qz) == 0)


def test_key_error_against_binary64_formula():
    # The binary32 pinned-order sum stays within a few ulp of the plain
    # binary64 sum of squared residuals (an independent evaluation).
    w = s.workload(1)
    g = s.generate(w, heads=[(0, 5)])
    k = np.ascontiguousarray(g["k"][:, 5:6])
    qz = oracle.quantize(k, k, k)
    err = oracle.key_error(k, qz).astype(np.float64)[0, 0]
    x = s.bf16_bits_to_f32(k[0, 0]).astype(np.float32) - qz["k_mean"][0, 0][None, :]
    dq = oracle.e4m3_decode(qz["k8"][0, 0]) * np.repeat(qz["sk"][0, 0].astype(np.float64), 64)[:, None]
    ref = ((x.astype(np.float64) - dq) ** 2).sum(axis=1)
    assert np.all(np.abs(err - ref) <= 1e-5 * ref + 1e-30)
    assert np.all(err > 0)


# ------------------------------------------------------------- selection

def test_select_keys_brute_force_with_ties():
    rng = np.random.default_rng(41)
    err = rng.integers(0, 5, size=(2, 3, 37)).astype(np.float32)    # many ties
    for kc in (0, 1, 5, 36, 37, 50):
        sel = oracle.select_keys(err, kc)
        for b in range(2):
            for h in range(3):
                e = err[b, h]
                order = sorted(range(37), key=lambda j: (-e[j], j))   # largest first, ties low index
                want = np.zeros(37, np.uint8)
                want[order[:min(kc, 37)]] = 1
                assert np.array_equal(sel[b, h], want), (kc, b, h)


def test_n_corrected_rounds_up():
    assert oracle.n_corrected(8704, 0.005) == 44
    assert oracle.n_corrected(1280, 0.005) == 7
    assert oracle.n_corrected(1280, 0.05) == 64      # fl32(0.05) * 1280 = 64.000001
    assert oracle.n_corrected(100, 0.0) == 0
    assert oracle.n_corrected(100, 1.0) == 100
    assert oracle.n_corrected(200, 0.005) == 1
    assert oracle.n_corrected(65536, 0.005) == 328


# ----------------------------------------------------- corrected attention

def _small_case(N=256, H=2, seed=42):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, H, N, 128)) * 2
    k = rng.standard_normal((1, H, N, 128)) * 2 + rng.standard_normal((1, H, 1, 128))
    v = rng.standard_normal((1, H, N, 128))
    g = {t: _bf16(x) for t, x in zip("qkv", (q, k, v))}
    return g, oracle.quantize(g["q"], g["k"], g["v"])


def test_no_corrected_key_is_the_fp8_rule():
    g, qz = _small_case()
    sel = np.zeros(qz["q8"].shape[:3], np.uint8)
    sc = oracle.softmax_scale()
    got = oracle.attention_fp8_corrected(g, qz, sel, sc)
    ref = oracle.attention_fp8(qz, sc)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_every_key_corrected_is_exact_attention():
    g, qz = _small_case(N=200)
    sel = np.ones(qz["q8"].shape[:3], np.uint8)
    sc = oracle.softmax_scale()
    got = oracle.attention_fp8_corrected(g, qz, sel, sc)
    ref = oracle.attention_exact(g["q"], g["k"], g["v"], sc)
    assert np.max(np.abs(got - ref)) < 1e-12


@pytest.mark.parametrize("N", [256, 200])
def test_merge_of_the_two_parts_is_softmax_over_the_mixed_scores(N):
    # With the FP8 part's P left unrounded, the merged result must be softmax
    # attention over one score vector: the dequantized (smoothed) scores for
    # the uncorrected keys and the exact scores on the smoothed keys for the
    # corrected ones, with V dequantized or exact accordingly.
    g, qz = _small_case(N=N, H=1, seed=43)
    rng = np.random.default_rng(44)
    sel = (rng.random((1, 1, N)) < 0.1).astype(np.uint8)
    sel[0, 0, 0] = 1
    sc = oracle.softmax_scale()
    got = oracle.attention_fp8_corrected(g, qz, sel, sc, quantize_p=False)[0]
    rep = lambda a: np.repeat(a[0, 0].astype(np.float64), 64)[:N, None]
    qd = oracle.e4m3_decode(qz["q8"][0, 0]) * rep(qz["sq"])
    kd = oracle.e4m3_decode(qz["k8"][0, 0]) * rep(qz["sk"])
    vd = oracle.e4m3_decode(qz["v8"][0, 0]) * rep(qz["sv"])
    qf, kf, vf = (s.bf16_bits_to_f32(g[t][0, 0]).astype(np.float64) for t in "qkv")
    mu = qz["k_mean"][0, 0].astype(np.float64)
    f32sc = float(np.float32(sc))
    S = (qd @ kd.T) * f32sc
    S_exact = (qf @ (kf - mu).T) * f32sc
    C = sel[0, 0].astype(bool)
    S[:, C] = S_exact[:, C]
    V = vd.copy()
    V[C] = vf[C]
    ref = scipy.special.softmax(S, axis=1) @ V
    assert np.max(np.abs(got - ref)) < 1e-10


def test_correcting_the_worst_keys_raises_accuracy_on_outlier_workload():
    # dit512 (x20 outlier channels): correcting the 5% worst keys moves the
    # result toward exact attention on every sampled head.
    w = s.workload(1)
    heads = [(0, 0), (0, 7)]
    g = s.generate(w, heads=heads)
    qz = oracle.quantize(g["q"], g["k"], g["v"])
    sc = oracle.softmax_scale()
    rows = list(range(0, w.N, 5))
    err = oracle.key_error(g["k"], qz)
    sel = oracle.select_keys(err, oracle.n_corrected(w.N, 0.05))
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], sc, heads=heads, rows=rows)
    plain = oracle.attention_fp8(qz, sc, heads=heads, rows=rows)
    corr = oracle.attention_fp8_corrected(g, qz, sel, sc, heads=heads, rows=rows)
    cos = lambda a, b: float((a * b).sum() / np.sqrt((a * a).sum() * (b * b).sum()))
    for hh in range(len(heads)):
        assert cos(corr[hh], ex[hh]) > cos(plain[hh], ex[hh]) + 0.01
