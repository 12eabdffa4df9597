"""Pins for the oracle's NVFP4 Q.K variant ("NVIDIA RTX AI optimiert FLUX.1
fuer Bilddaten mit niedriger Genauigkeit", SDPA quantization paragraph: the
FP8 and FP4 schemes differ only in the precision of the Q, K, V projections;
attention stays in FP8).

Readings under test: Q and smoothed K in NVFP4 -- E2M1 elements (OCP MX
specification: values 0, 0.5, 1, 1.5, 2, 3, 4, 6), one unsigned E4M3 scale per
16 channels -- under the FP8 path's per-64-token-block FP32 scale
s1 = amax / (6 * 448); the group scale s2 = E4M3(amax_g / fl32(6 s1)); the code
E2M1(x / fl32(s1 dec(s2))); V, P and the softmax unchanged."""

import numpy as np
import pytest

import fqa_synth as s
import oracle

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _bf16(x):
    return s.round_to_bf16_bits(np.asarray(x, dtype=np.float64))


def test_e2m1_decode_table_is_the_spec():
    for c in range(16):
        v = E2M1[c & 7]
        got = oracle.e2m1_decode(c)[()]
        assert got == (-v if c & 8 else v) and (np.signbit(got) == bool(c & 8))


def _nearest_even(x):
    a = abs(x)
    if a >= 6.0:
        return 7 | (8 if x < 0 or np.signbit(x) else 0)
    best = min(range(8), key=lambda c: (abs(E2M1[c] - a), c & 1))
    return best | (8 if np.signbit(x) else 0)


def test_e2m1_encode_brute_force_with_ties():
    xs = [i / 8 for i in range(-64, 65)] + [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.9, 6.0, 7.0, 1e9, -0.0]
    for x in xs:
        assert oracle.e2m1_encode_f64(x) == _nearest_even(x), x
    # the ties by hand: 0.25 -> 0, 0.75 -> 1.0, 1.25 -> 1.0, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    assert [oracle.e2m1_encode_f64(x) for x in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)] == [0, 2, 2, 4, 4, 6, 6]


def _nib(q4, n, c):
    b = q4[n, c // 2]
    return (b >> 4) & 15 if c & 1 else b & 15


def test_block_hand_case():
    # One 64-token block of Q with amax = 2688 -> s1 = 1 exactly.
    #   token 0, group 0: 2688 at channel 0 -> amax_g = 2688, t = 448 -> s2 = 448
    #     (0x7E), dg = 448: 2688 / 448 = 6 -> code 7; 1000 at ch 1 -> 2.232 -> 2 (code 4)
    #   token 1, group 1 (ch 16..31): values 6, -3, 0.5, 5 -> amax_g = 6, t = 1,
    #     s2 = 1 (0x38), dg = 1: codes 7, 0xD (-3), 1 (0.5), 6 (5 -> tie -> 4)
    #   token 2: all zero -> s2 = 0, codes 0
    q = np.zeros((1, 1, 64, 128))
    q[0, 0, 0, 0], q[0, 0, 0, 1] = 2688.0, 1000.0
    q[0, 0, 1, 16:20] = [6.0, -3.0, 0.5, 5.0]
    qb = _bf16(q)
    assert s.bf16_bits_to_f32(qb[0, 0, 0, :2]).tolist() == [2688.0, 1000.0]
    z = np.zeros_like(qb)
    r = oracle.quantize_nvfp4(qb, z, z)
    assert r["sq1"][0, 0, 0] == 1.0
    assert r["sfq"][0, 0, 0, 0] == 0x7E and r["sfq"][0, 0, 1, 1] == 0x38
    q4 = r["q4"][0, 0]
    assert (_nib(q4, 0, 0), _nib(q4, 0, 1)) == (7, 4)
    assert [_nib(q4, 1, 16 + i) for i in range(4)] == [7, 0xD, 1, 6]
    assert np.all(r["sfq"][0, 0, 2] == 0) and np.all(q4[2] == 0)
    # an all-zero block flushes: s1 = 0, every group scale and code 0
    assert r["sk1"][0, 0, 0] == 0 and np.all(r["k4"] == 0) and np.all(r["sfk"] == 0)


def test_dequantized_error_bound():
    w = s.workload(1)
    g = s.generate(w, heads=[(0, 2)])
    q = np.ascontiguousarray(g["q"][:, 2:3])
    r = oracle.quantize_nvfp4(q, q, q)
    x = s.bf16_bits_to_f32(q[0, 0]).astype(np.float64)
    N = w.N
    s1 = np.repeat(r["sq1"][0, 0].astype(np.float64), 64)[:N]
    s2 = oracle.e4m3_decode(r["sfq"][0, 0]).astype(np.float64)            # [N, 8]
    dg = (s1[:, None] * s2).astype(np.float32).astype(np.float64)           # fl32(s1 * dec(s2))
    codes = np.stack([np.array([_nib(r["q4"][0, 0], n, c) for c in range(128)]) for n in range(0, N, 97)])
    rows = list(range(0, N, 97))
    deq = oracle.e2m1_decode(codes) * np.repeat(dg[rows], 16, axis=1)
    xr = x[rows]
    # within one E2M1 step of the scaled grid (the largest step, 4 -> 6, is 2), or
    # saturated at 6 dg where the group scale rounded down
    step = np.repeat(dg[rows], 16, axis=1)
    assert np.all((np.abs(xr - deq) <= step + 1e-30) | (np.abs(deq) == 6 * step))
    # the largest value of a block maps near the top of the grid
    assert np.all(s2.max(axis=1) <= 448.0)


def test_attention_decodes_codes_like_an_independent_decoder():
    # orc_attention_nvfp4 = the pinned tiled core on the dequantized Q and K;
    # decode the packed nibbles and group scales here, independently, and run
    # the core on them: the two must agree exactly.
    rng = np.random.default_rng(60)
    N = 256
    q, k, v = (_bf16(rng.standard_normal((1, 1, N, 128)) * 2) for _ in range(3))
    r = oracle.quantize_nvfp4(q, k, v)
    sc = oracle.softmax_scale()

    def deq(q4, sf):
        lo, hi = q4 & 15, (q4 >> 4) & 15
        codes = np.empty((N, 128), np.uint8)
        codes[:, 0::2], codes[:, 1::2] = lo, hi
        return oracle.e2m1_decode(codes) * np.repeat(oracle.e4m3_decode(sf), 16, axis=1)

    qc, kc = deq(r["q4"][0, 0], r["sfq"][0, 0]), deq(r["k4"][0, 0], r["sfk"][0, 0])
    vc = oracle.e4m3_decode(r["v8"][0, 0])
    ref = oracle.attention_core(qc, kc, vc, r["sq1"][0, 0], r["sk1"][0, 0], r["sv"][0, 0],
                                float(r["sv_max"][0, 0]), sc)
    got = oracle.attention_nvfp4(r, sc)[0]
    assert np.array_equal(got, ref)


def test_nvfp4_outputs_follow_exact_attention_on_mild_inputs():
    # without outliers the 4-bit Q.K still tracks exact attention
    w = s.workload(0)
    g = s.generate(w)
    r = oracle.quantize_nvfp4(g["q"], g["k"], g["v"])
    sc = oracle.softmax_scale()
    got = oracle.attention_nvfp4(r, sc)
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], sc)
    cos = float((got * ex).sum() / np.sqrt((got * got).sum() * (ex * ex).sum()))
    assert cos > 0.95
