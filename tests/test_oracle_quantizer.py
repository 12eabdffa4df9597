"""Pins for the oracle's quantizer (K mean, block scales, E4M3 codes).

Readings under test: one FP32 absmax scale per (b, h, 64-token block) over all
128 channels; s = amax/448, inv = 448/amax (binary32 divisions; amax == 0
gives 0, 0); code = E4M3(fl32(x * inv)); K smoothed as fl32(k - mu[c]) with
mu summed per 64-token block, then over blocks, in ascending order, then
divided by N; sv_max = max of the head's V block scales.
"""

import numpy as np
import torch

import fqa_synth as s
import oracle

F32_EPS = 2.0 ** -24


def _bf16(x):
    return s.round_to_bf16_bits(np.asarray(x, dtype=np.float64))


def test_k_mean_exact_on_small_integers():
    rng = np.random.default_rng(0)
    k = rng.integers(-50, 50, size=(1, 2, 256, 128)).astype(np.float64)
    mu = oracle.k_mean(_bf16(k))
    assert np.array_equal(mu.astype(np.float64), k.mean(axis=2))   # sums exact, N = 2^8


def test_k_mean_sequential_order_hand_case():
    # Block 0 of channel 0 holds 2^24 then 63 ones: adding 1 to 2^24 in
    # binary32 is a tie that rounds back to 2^24 (even), so the pinned
    # ascending order gives p_0 = 2^24 exactly; a pairwise or reversed order
    # would keep the ones (2^24 + 62 or + 64).  Block 1 holds 64 ones -> 64.
    N = 128
    k = np.zeros((1, 1, N, 128))
    k[0, 0, 0, 0] = 2.0 ** 24
    k[0, 0, 1:64, 0] = 1.0
    k[0, 0, 64:128, 0] = 1.0
    mu = oracle.k_mean(_bf16(k))
    assert mu[0, 0, 0] == np.float32((2.0 ** 24 + 64.0) / 128.0)
    assert np.all(mu[0, 0, 1:] == 0.0)


def test_k_mean_error_bound_random():
    w = s.workload(2)
    g = s.generate(w, "k", heads=[(0, 0)])
    k = g["k"][:, :1]
    mu = oracle.k_mean(k).astype(np.float64)[0, 0]
    kf = s.bf16_bits_to_f32(k[0, 0]).astype(np.float64)
    exact = kf.mean(axis=0)
    nblk = w.N // 64
    bound = (64 + nblk + 1) * F32_EPS * np.abs(kf).sum(axis=0) / w.N + F32_EPS * np.abs(exact)
    assert np.all(np.abs(mu - exact) <= bound)


def test_block_with_amax_448_codes_equal_plain_cast():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 1, 64, 128)) * 40.0
    x[0, 0, 3, 7] = 448.0
    x = np.clip(x, -440, 440)
    x[0, 0, 3, 7] = 448.0
    q = _bf16(x)
    r = oracle.quantize(q, q, q)
    assert r["sq"][0, 0, 0] == 1.0
    xf = s.bf16_bits_to_f32(q)
    ref = torch.from_numpy(xf).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(r["q8"], ref)
    assert np.array_equal(r["v8"], ref)


def test_block_amax_one_scale_and_codes():
    # amax = 1: s = fl32(1/448), inv = 448 exactly; codes = E4M3(fl32(x*448)).
    rng = np.random.default_rng(2)
    x = rng.uniform(-1, 1, (1, 1, 64, 128))
    x[0, 0, 0, 0] = -1.0
    q = _bf16(x)
    r = oracle.quantize(q, np.zeros_like(q), q)
    assert r["sq"][0, 0, 0] == np.float32(1.0) / np.float32(448.0)
    xf = s.bf16_bits_to_f32(q).astype(np.float32) * np.float32(448.0)
    ref = torch.from_numpy(xf).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(r["q8"], ref)
    assert r["q8"][0, 0, 0, 0] == 0xFE                      # -448


def test_zero_block_gives_zero_scale_and_codes():
    z = np.zeros((1, 1, 128, 128), dtype=np.uint16)
    r = oracle.quantize(z, z, z)
    assert np.all(r["sq"] == 0) and np.all(r["sk"] == 0) and np.all(r["sv"] == 0)
    assert np.all(r["q8"] == 0) and np.all(r["v8"] == 0) and r["sv_max"][0, 0] == 0


def test_codes_within_half_ulp_and_peak_maps_to_448():
    w = s.workload(1)
    g = s.generate(w, heads=[(0, 3)])
    q, k, v = (g[t][:, 3:4] for t in "qkv")
    r = oracle.quantize(q, k, v)
    dec = oracle.e4m3_decode
    mu = r["k_mean"][0, 0]
    for name, x in (("q", s.bf16_bits_to_f32(q[0, 0])),
                    ("k", s.bf16_bits_to_f32(k[0, 0]) - mu[None, :]),
                    ("v", s.bf16_bits_to_f32(v[0, 0]))):
        codes = r[name + "8"][0, 0]
        scl = r["s" + name][0, 0]
        for j in range(w.N // 64):
            xb = x[64 * j:64 * j + 64].astype(np.float64)
            amax = np.abs(xb).max()
            assert scl[j] == np.float32(np.float32(amax) / np.float32(448.0))
            y = xb * float(np.float32(448.0) / np.float32(amax))
            dv = dec(codes[64 * j:64 * j + 64])
            err = np.abs(dv - y)
            # half an E4M3 ulp: 2^-4 relative for normals, 2^-10 absolute below 2^-6
            assert np.all(err <= np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6))
            assert np.abs(dv).max() == 448.0
    assert r["sv_max"][0, 0] == r["sv"][0, 0].max()


def test_k_smoothing_absorbs_channel_offset():
    # integer K plus an integer per-channel offset: the mean shifts by exactly
    # the offset, so the smoothed values, the K scales and the K codes are equal.
    rng = np.random.default_rng(3)
    k = rng.integers(-8, 8, size=(1, 1, 256, 128)).astype(np.float64)
    off = rng.integers(-20, 20, size=128).astype(np.float64)
    a = oracle.quantize(_bf16(k), _bf16(k), _bf16(k))
    b = oracle.quantize(_bf16(k), _bf16(k + off), _bf16(k))
    assert np.array_equal(a["k8"], b["k8"]) and np.array_equal(a["sk"], b["sk"])
    assert np.array_equal(b["k_mean"] - a["k_mean"], off[None, None, :].astype(np.float32))
