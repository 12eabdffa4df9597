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


# ---------------------------------------------------------------- tiny blocks
# Two regimes where the plain rule code = E4M3(fl32(x * fl32(448/amax))) has
# no finite answer; the pages are silent on both, so the readings are:
#   448/amax overflows binary32  -> code = E4M3(fl32(x / s)), s = fl32(amax/448)
#   amax/448 underflows to s = 0 -> the block is flushed: inv = 0, signed-zero codes
# The expected values below were worked by hand; the comments give the steps.

def _bits(x: float) -> int:
    """BF16 bit pattern of a value exactly representable in BF16."""
    b = s.round_to_bf16_bits(np.array([x], dtype=np.float64))[0]
    assert s.bf16_bits_to_f32(np.array([b], np.uint16))[0] == np.float32(x)
    return int(b)


def test_block_whose_inverse_scale_overflows_divides_by_the_scale():
    # amax = 2^-123 (a BF16 normal); 448 * 2^123 = 7 * 2^129 > FLT_MAX, so
    # inv overflows.  s = fl32(2^-123 / 448) = fl32(2^-129 / 7): subnormal,
    # 2^20 / 7 = 149796.57 units of 2^-149 -> 149797 * 2^-149.
    #   x =  2^-123: x/s = 2^26/149797 = 447.998 -> 448       -> 0x7E
    #   x = -2^-123:                              -> -448     -> 0xFE
    #   x =  2^-130 (BF16 subnormal): 2^19/149797 = 3.49999 -> 3.5 = 1.75*2^1 -> 0x46
    #   x =  2^-133 (smallest BF16): 2^16/149797 = 0.437505 -> 0.4375 = 1.75*2^-2 -> 0x2E
    #   x =  0                                               -> 0x00 (not 0*inf = NaN)
    blk = np.zeros((1, 1, 64, 128), dtype=np.uint16)
    blk[0, 0, 0, 0] = _bits(2.0 ** -123)
    blk[0, 0, 1, 5] = _bits(-(2.0 ** -123))
    blk[0, 0, 2, 9] = _bits(2.0 ** -130)
    blk[0, 0, 3, 127] = _bits(2.0 ** -133)
    z = np.zeros_like(blk)
    r = oracle.quantize(blk, z, blk)
    s_expect = np.float32(149797 * 2.0 ** -149)
    assert r["sq"][0, 0, 0] == s_expect and r["sv"][0, 0, 0] == s_expect
    assert r["sv_max"][0, 0] == s_expect
    for name in ("q8", "v8"):
        c = r[name][0, 0]
        assert (c[0, 0], c[1, 5], c[2, 9], c[3, 127]) == (0x7E, 0xFE, 0x46, 0x2E)
        nz = np.zeros_like(c, dtype=bool)
        nz[0, 0] = nz[1, 5] = nz[2, 9] = nz[3, 127] = True
        assert np.all(c[~nz] == 0)                    # zeros stay zeros
    # the same numbers from exact rational arithmetic and the spec's code table
    from fractions import Fraction as F
    table = {i: oracle.e4m3_decode(i) for i in range(256) if not np.isnan(oracle.e4m3_decode(i))}
    sF = F(149797, 2 ** 149)
    for x, code in ((F(1, 2 ** 123), 0x7E), (F(1, 2 ** 130), 0x46), (F(1, 2 ** 133), 0x2E)):
        y = float(np.float32(float(x / sF)))          # the binary32 quotient
        best = min((c for c in table if table[c] >= 0), key=lambda c: abs(table[c] - y))
        assert best == code


def test_smoothed_k_block_whose_scale_underflows_is_flushed():
    # N = 1024, channel 0 of K holds 2^-133 at token 1000 and 0 elsewhere:
    #   mu[0] = 2^-133 / 1024 = 2^-143 (exact: 64 units of 2^-149)
    #   blocks 0..14: x = 0 - 2^-143 in channel 0, 0 elsewhere; amax = 2^-143,
    #     s = fl32(2^-143 / 448) = fl32(0.1429 * 2^-149) = 0  -> flushed: s = 0,
    #     codes fl32(x * 0) = -0 -> 0x80 in channel 0, +0 -> 0x00 elsewhere
    #   block 15 (tokens 960..1023): x(token 1000) = 2^-133 - 2^-143 =
    #     65472 * 2^-149 = amax; s = fl32(65472/448 = 146.14 units) = 146 * 2^-149;
    #     448/amax overflows -> divide: 65472/146 = 448.4 -> 0x7E;
    #     the other tokens: -64/146 = -0.4384 -> -0.4375 -> 0xAE
    N = 1024
    k = np.zeros((1, 1, N, 128), dtype=np.uint16)
    k[0, 0, 1000, 0] = _bits(2.0 ** -133)
    z = np.zeros_like(k)
    r = oracle.quantize(z, k, z)
    assert r["k_mean"][0, 0, 0] == np.float32(2.0 ** -143) and np.all(r["k_mean"][0, 0, 1:] == 0)
    sk, k8 = r["sk"][0, 0], r["k8"][0, 0]
    assert np.all(sk[:15] == 0) and sk[15] == np.float32(146 * 2.0 ** -149)
    assert np.all(k8[:960, 0] == 0x80) and np.all(k8[:960, 1:] == 0x00)
    assert k8[1000, 0] == 0x7E
    other = np.ones(64, dtype=bool)
    other[40] = False
    assert np.all(k8[960:][other, 0] == 0xAE) and np.all(k8[960:, 1:] == 0x00)
    # no code anywhere is a NaN (S.1111.111)
    for name in ("q8", "k8", "v8"):
        assert not np.any((r[name] & 0x7F) == 0x7F)


# ------------------------------------------------- sequences not a multiple of 64
# [reading] the last block of a head holds the remaining N - 64*(nblk-1) tokens;
# its scale is the absmax of those tokens alone; the K mean sums the short
# block like the others and divides by N.

def test_k_mean_short_last_block_exact_on_small_integers():
    rng = np.random.default_rng(21)
    k = rng.integers(-50, 50, size=(1, 2, 100, 128)).astype(np.float64)
    mu = oracle.k_mean(_bf16(k)).astype(np.float64)
    # every partial and total sum is an exact small integer, so only the final
    # division rounds
    assert np.array_equal(mu, (k.sum(axis=2) / 100.0).astype(np.float32).astype(np.float64))


def test_k_mean_short_last_block_order_hand_case():
    # N = 66: block 0 = 2^24 then 63 ones (each +1 is a tie back to 2^24), so
    # p_0 = 2^24; block 1 has the 2 remaining tokens, 1 and 1: p_1 = 2;
    # T = 2^24 + 2 (exact); mu = fl32((2^24 + 2) / 66).
    k = np.zeros((1, 1, 66, 128))
    k[0, 0, 0, 0] = 2.0 ** 24
    k[0, 0, 1:66, 0] = 1.0
    mu = oracle.k_mean(_bf16(k))
    assert mu[0, 0, 0] == np.float32(np.float32(2.0 ** 24 + 2.0) / np.float32(66.0))


def test_short_last_block_scale_is_its_own_absmax():
    # N = 70: block 0 reaches |x| = 300, the 6-token block 1 only 3, so
    # sq[1] = fl32(3/448) and its codes are E4M3(fl32(x * fl32(448/3))).
    rng = np.random.default_rng(22)
    x = rng.uniform(-2.5, 2.5, (1, 1, 70, 128))
    x[0, 0, :64] *= 100.0
    x[0, 0, 10, 3] = 300.0
    x[0, 0, 66, 100] = -3.0
    q = _bf16(x)
    r = oracle.quantize(q, q, q)
    assert r["sq"].shape == (1, 1, 2)
    assert r["sq"][0, 0, 0] == np.float32(300.0) / np.float32(448.0)
    assert r["sq"][0, 0, 1] == np.float32(3.0) / np.float32(448.0)
    xf = s.bf16_bits_to_f32(q[0, 0, 64:]).astype(np.float32) * (np.float32(448.0) / np.float32(3.0))
    ref = torch.from_numpy(xf).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(r["q8"][0, 0, 64:], ref)
    assert r["sv_max"][0, 0] == r["sv"][0, 0, 0]
