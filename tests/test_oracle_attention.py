"""Pins for the oracle's attention: the exact FP64 reference against library and
brute-force evaluations, the tiled skeleton against exact softmax attention,
invariants of softmax attention, and hand-worked cases of the FP8 P rule
(tests/golden/p_rounding_cases.json)."""

import json
import math
import os

import numpy as np
import pytest
import scipy.special

import fqa_synth as s
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p_rounding_cases.json")
LN2 = math.log(2.0)


def _bf16(x):
    return s.round_to_bf16_bits(np.asarray(x, dtype=np.float64))


def _scipy_attention(q, k, v, scale):
    p = scipy.special.softmax((q @ k.T) * scale, axis=-1)
    return p @ v


def test_exact_matches_scipy_softmax():
    w = s.workload(0)
    g = s.generate(w)
    sc = oracle.softmax_scale()
    out = oracle.attention_exact(g["q"], g["k"], g["v"], sc)
    for hh, (b, h) in enumerate([(0, 0), (0, 1)]):
        q, k, v = (s.bf16_bits_to_f32(g[t][b, h]).astype(np.float64) for t in "qkv")
        ref = _scipy_attention(q, k, v, float(np.float32(sc)))
        assert np.max(np.abs(out[hh] - ref)) < 1e-12


def test_exact_brute_force_tiny():
    rng = np.random.default_rng(5)
    N, d = 8, 4
    q, k, v = (rng.integers(-4, 5, size=(1, 1, N, d)).astype(np.float64) for _ in range(3))
    out = oracle.attention_exact(_bf16(q), _bf16(k), _bf16(v), 0.3)[0]
    for i in range(N):
        sc = [0.3 * math.fsum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(d)) for j in range(N)]
        mx = max(sc)
        e = [math.exp(x - mx) for x in sc]
        den = math.fsum(e)
        for c in range(d):
            ref = math.fsum(e[j] * v[0, 0, j, c] for j in range(N)) / den
            assert abs(out[i, c] - ref) < 1e-13


def test_exact_d1_n2_by_hand():
    # scores [0, ln 2] -> weights [1/3, 2/3]; V = [3, 6] -> 5
    q = _bf16(np.ones((1, 1, 2, 1)))
    k = _bf16(np.array([0.0, 1.0]).reshape(1, 1, 2, 1))
    v = _bf16(np.array([3.0, 6.0]).reshape(1, 1, 2, 1))
    out = oracle.attention_exact(q, k, v, LN2)
    assert abs(out[0, 0, 0] - 5.0) < 1e-14 and abs(out[0, 1, 0] - 5.0) < 1e-14


def test_exact_invariant_under_kv_permutation_and_k_shift():
    rng = np.random.default_rng(6)
    N, d = 256, 128
    q = rng.integers(-3, 4, size=(1, 1, N, d)).astype(np.float64)
    k = rng.integers(-3, 4, size=(1, 1, N, d)).astype(np.float64)
    v = rng.standard_normal((1, 1, N, d))
    base = oracle.attention_exact(_bf16(q), _bf16(k), _bf16(v), 0.05)
    perm = rng.permutation(N)
    pk, pv = k[:, :, perm], v[:, :, perm]
    assert np.max(np.abs(oracle.attention_exact(_bf16(q), _bf16(pk), _bf16(pv), 0.05) - base)) < 1e-12
    off = rng.integers(-5, 6, size=d).astype(np.float64)
    assert np.max(np.abs(oracle.attention_exact(_bf16(q), _bf16(k + off), _bf16(v), 0.05) - base)) < 1e-12


@pytest.mark.parametrize("bc", [16, 64, 128, 256])
def test_tiled_core_identity_codec_is_exact_attention(bc):
    # With P left unrounded the tiled rule is softmax attention on the
    # dequantized operands (qc*sq_I, kc*sk_J, vc*sv_J), for any tile size.
    rng = np.random.default_rng(7)
    N, d = 256, 128
    qc, kc, vc = (rng.standard_normal((N, d)) * 3 for _ in range(3))
    sq, sk, sv = (rng.uniform(0.2, 2.0, N // 64).astype(np.float32) for _ in range(3))
    sv_max = float(sv.max())
    scale = 0.088
    out = oracle.attention_core(qc, kc, vc, sq, sk, sv, sv_max, scale, bc=bc, quantize_p=False)
    rep = lambda a: np.repeat(a.astype(np.float64), 64)[:, None]
    ref = _scipy_attention(qc * rep(sq), kc * rep(sk), vc * rep(sv), scale)
    assert np.max(np.abs(out - ref)) < 1e-12


@pytest.mark.parametrize("N,bc", [(200, 128), (77, 64), (129, 128), (1, 128)])
def test_tiled_core_identity_codec_ragged_length(N, bc):
    # N not a multiple of the tile (nor of the 64-token block): the last tile
    # holds the remaining keys and the last block's scale covers the
    # remaining tokens; unrounded, the rule is still exact softmax attention.
    rng = np.random.default_rng(17)
    d = 128
    nb = (N + 63) // 64
    qc, kc, vc = (rng.standard_normal((N, d)) * 3 for _ in range(3))
    sq, sk, sv = (rng.uniform(0.2, 2.0, nb).astype(np.float32) for _ in range(3))
    scale = 0.088
    out = oracle.attention_core(qc, kc, vc, sq, sk, sv, float(sv.max()), scale, bc=bc, quantize_p=False)
    rep = lambda a: np.repeat(a.astype(np.float64), 64)[:N, None]
    ref = _scipy_attention(qc * rep(sq), kc * rep(sk), vc * rep(sv), scale)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_exact_matches_scipy_ragged_length():
    rng = np.random.default_rng(18)
    N, d = 77, 128
    q, k, v = (_bf16(rng.standard_normal((1, 1, N, d)) * 2) for _ in range(3))
    sc = oracle.softmax_scale()
    out = oracle.attention_exact(q, k, v, sc)[0]
    qf, kf, vf = (s.bf16_bits_to_f32(t[0, 0]).astype(np.float64) for t in (q, k, v))
    assert np.max(np.abs(out - _scipy_attention(qf, kf, vf, float(np.float32(sc))))) < 1e-12


def test_rows_sum_to_one_identity_codec():
    rng = np.random.default_rng(8)
    N, d = 384, 128
    qc, kc = rng.standard_normal((N, d)) * 4, rng.standard_normal((N, d)) * 4
    ones = np.ones((N, d))
    u = np.ones(N // 64, np.float32)
    out = oracle.attention_core(qc, kc, ones, u, u, u, 1.0, 0.1, quantize_p=False)
    assert np.max(np.abs(out - 1.0)) < 1e-13


def test_uniform_scores_give_mean_of_dequantized_v():
    # Q = 0: every block scale is 0, all scores are 0, p = 1, and with every V
    # block sharing one amax (V tiles one 64x128 block) rv = 1, P = 448
    # exactly, so O is the plain mean of the dequantized V rows.
    rng = np.random.default_rng(9)
    blk = rng.standard_normal((64, 128))
    v = np.tile(blk, (4, 1)).reshape(1, 1, 256, 128)
    k = rng.standard_normal((1, 1, 256, 128))
    qz = oracle.quantize(_bf16(np.zeros_like(k)), _bf16(k), _bf16(v))
    assert np.all(qz["sq"] == 0)
    out = oracle.attention_fp8(qz, oracle.softmax_scale())[0]
    deq = oracle.e4m3_decode(qz["v8"][0, 0]) * np.repeat(qz["sv"][0, 0].astype(np.float64), 64)[:, None]
    ref = deq.mean(axis=0)
    assert np.max(np.abs(out - ref[None, :])) < 1e-13


def test_zero_v_gives_zero_output():
    rng = np.random.default_rng(10)
    q = _bf16(rng.standard_normal((1, 1, 128, 128)))
    z = np.zeros((1, 1, 128, 128), np.uint16)
    qz = oracle.quantize(q, q, z)
    assert np.all(oracle.attention_fp8(qz, oracle.softmax_scale()) == 0.0)


def _golden_inputs(case):
    N, d = case["N"], 128
    qc = np.zeros((N, d))
    qc[0, 0] = case["q_row0_channel0"]
    kc = np.zeros((N, d))
    kc[:, 0] = case["filler_key_value"]
    for j, t in case["keys"].items():
        kc[int(j), 0] = t
    vc = np.zeros((N, d))
    for j, c in case["v_unit_rows"].items():
        vc[int(j), c] = 1.0
    return qc, kc, vc


@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_hand_worked_p_rounding_cases(idx):
    case = json.load(open(GOLDEN))["cases"][idx]
    qc, kc, vc = _golden_inputs(case)
    out, amb, namb = oracle.attention_core(
        qc, kc, vc, np.array(case["sq"], np.float32), np.array(case["sk"], np.float32),
        np.array(case["sv"], np.float32), case["sv_max"], LN2, bc=case["bc"], quantize_p=True,
        rows=[0], with_ambiguity=True)
    out, amb, namb = out[0], amb[0], int(namb[0])
    exp_amb = np.zeros(128)
    for c, val in case.get("expected_amb", {}).items():
        exp_amb[int(c)] = val
    assert namb == case.get("expected_namb", 0)
    assert np.max(np.abs(amb - exp_amb)) < 1e-9
    l = eval(case["expected_l"], {"__builtins__": {}})
    if "expected_weights" in case:
        weights = [eval(wt, {"__builtins__": {}}) for wt in case["expected_weights"]]
    else:
        weights = [p / 448.0 for p in case["expected_P"]]
    expect = np.zeros(128)
    for c, wt in enumerate(weights):
        expect[c] = wt / l
    assert np.max(np.abs(out - expect)) < 1e-12


def test_small_workload_quantized_close_to_exact():
    """On tiny_n256 (no outlier channels) the FP8 scheme stays within
    cos 0.995 of exact attention."""
    w = s.workload("tiny_n256")
    g = s.generate(w)
    sc = oracle.softmax_scale()
    qz = oracle.quantize(g["q"], g["k"], g["v"])
    a = oracle.attention_fp8(qz, sc)
    e = oracle.attention_exact(g["q"], g["k"], g["v"], sc)
    cos = float((a * e).sum() / np.sqrt((a * a).sum() * (e * e).sum()))
    assert cos > 0.995


def test_ambiguity_bound_covers_binary32_evaluation():
    """Re-evaluate the P codes of a workload head the way a binary32 kernel
    does (scores, scales and the running max rounded to binary32, P values
    rounded to binary32 before encoding): every code that differs from the
    binary64 oracle's is one the oracle flagged, and the binary32 result lies
    within the reported bound."""
    w = s.workload(1)
    g = s.generate(w, heads=[(0, 0)])
    qz = oracle.quantize(g["q"][:, :1], g["k"][:, :1], g["v"][:, :1])
    ref, amb, namb = oracle.attention_fp8(qz, oracle.softmax_scale(), with_ambiguity=True)
    dec = oracle.e4m3_decode
    qc, kc, vc = (dec(qz[t][0, 0]) for t in ("q8", "k8", "v8"))
    sq, sk, sv = (qz[t][0, 0] for t in ("sq", "sk", "sv"))
    svm = qz["sv_max"][0, 0]
    c = np.float32(np.float32(oracle.softmax_scale()) * np.float32(1.4426950408889634))
    a32 = (np.repeat(sq, 64)[:, None] * np.repeat((sk * c).astype(np.float32), 64)[None, :]).astype(np.float32)
    x32 = ((qc @ kc.T).astype(np.float32) * a32).astype(np.float32)
    cj = np.repeat((np.float32(448.0) * (sv / svm).astype(np.float32)).astype(np.float32), 64)
    N = w.N
    m = np.full(N, -np.inf, np.float32)
    acc = np.zeros((N, 128))
    l = np.zeros(N)
    for t0 in range(0, N, 128):
        sl = slice(t0, t0 + 128)
        m_new = np.maximum(m, x32[:, sl].max(1))
        alpha = np.exp2(m.astype(np.float64) - m_new)
        p = np.exp2((x32[:, sl] - m_new[:, None]).astype(np.float32)).astype(np.float32)
        P = dec(oracle.e4m3_encode((p * cj[None, sl]).astype(np.float32)))
        acc = acc * alpha[:, None] + P @ vc[sl]
        l = l * alpha + p.astype(np.float64).sum(1)
        m = m_new
    out32 = acc * (float(svm) / 448.0) / l[:, None]
    # beyond flipped codes, binary32 scores shift O by ~1e-4 (alpha, l)
    assert np.all(np.abs(out32 - ref[0]) <= amb[0] + 1e-3)
