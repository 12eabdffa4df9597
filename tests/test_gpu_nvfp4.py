"""The NVFP4 Q.K variant on the GPU against the oracle ("NVIDIA RTX AI
optimiert FLUX.1 fuer Bilddaten mit niedriger Genauigkeit", SDPA quantization
paragraph: the FP8 and FP4 schemes differ only in the precision of the Q, K,
V projections; attention itself stays in FP8).

- the E2M1 conversion: bit-exact with the oracle's codec on every tie, its
  neighbours and a random spread of binary32 values, nibble order included;
- fqa_quantize_nvfp4_qk: codes, group scales and block scales bit-exact with
  the oracle on every workload shape, on ragged N and on tiny blocks;
- fqa_attention_nvfp4: every element within 1e-2 + amb of the oracle (amb:
  the oracle's bound on P codes the binary32 evaluation may round either
  way), mean relative error <= 2e-3 -- the FP8 path's bar; all rows on the
  small cases, sampled rows at full size; any sequence length.
"""

import numpy as np
import pytest
import torch

import fqa_synth as synth
import oracle
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _fqa():
    import quantized_fp8_attention_b200 as fqa
    return fqa


def _gen(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return synth.round_to_bf16_bits(rng.standard_normal(shape) * scale)


def _gpu_nvfp4(bits):
    fqa = _fqa()
    q, k, v = (U.to_device(bits[t]) for t in "qkv")
    qz = fqa.quantize(q, k, v)
    qn = fqa.quantize_nvfp4_qk(q, k, qz.k_mean)
    return qz, qn


def _as_oracle(qz, qn) -> dict:
    d = U.to_oracle_quant(qz)
    d.update({name: t.cpu().numpy() for name, t in zip(qn._fields, qn)})
    return d


# ------------------------------------------------------------------ codec

def test_e2m1_codec_matches_oracle():
    fqa = _fqa()
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)
    ties = (grid[1:] + grid[:-1]) / 2
    pts = np.concatenate([grid, ties, [0.25, 6.5, 7.0, 1e9, 3.4e38, 1e-45, 1e-40]]).astype(np.float32)
    up = np.nextafter(pts, np.float32(np.inf))
    dn = np.nextafter(pts, np.float32(0))
    rng = np.random.default_rng(7)
    spread = (rng.standard_normal(6000) * np.exp2(rng.uniform(-12, 5, 6000))).astype(np.float32)
    x = np.concatenate([pts, up, dn, -pts, -up, -dn, spread]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(-0.0))
    got = fqa.e2m1_encode(torch.from_numpy(x).cuda()).cpu().numpy()
    want = np.array([oracle.e2m1_encode_f64(float(a)) for a in x], np.uint8)
    lo, hi = got & 15, got >> 4
    bad = np.flatnonzero((lo != want[0::2]) | (hi != want[1::2]))
    assert bad.size == 0, [(float(x[2 * i]), float(x[2 * i + 1]), int(got[i])) for i in bad[:8]]


# -------------------------------------------------------------- quantizer

def _check_quant_bit_exact(bits):
    qz, qn = _gpu_nvfp4(bits)
    ref = oracle.quantize_nvfp4(bits["q"], bits["k"], bits["v"])
    for name, t in zip(qn._fields, qn):
        got = t.cpu().numpy()
        assert got.shape == ref[name].shape, name
        if got.dtype == np.float32:
            assert np.array_equal(got.view(np.uint32), ref[name].view(np.uint32)), name
        else:
            assert np.array_equal(got, ref[name]), (name, int((got != ref[name]).sum()))


@pytest.mark.parametrize("idx", [0, 1, 3])
def test_quantize_nvfp4_bit_exact(idx):
    _check_quant_bit_exact(U.host_inputs(idx))


@pytest.mark.parametrize("N", [1, 100, 200, 1000])
def test_quantize_nvfp4_ragged_bit_exact(N):
    shape = (1, 3, N, 128)
    _check_quant_bit_exact({t: _gen(shape, 80 + i, 3.0) for i, t in enumerate("qkv")})


def test_quantize_nvfp4_tiny_blocks_bit_exact():
    """Blocks of subnormal inputs (s1 and the group scales deep in the
    binary32 subnormal range), next to
    ordinary blocks and an all-zero block."""
    shape = (1, 2, 320, 128)
    bits = {t: _gen(shape, 90 + i, 1.0) for i, t in enumerate("qkv")}
    x = synth.bf16_bits_to_f32(bits["q"]).astype(np.float64)
    x[0, 0, 0:64] *= 1e-38          # s1 subnormal
    x[0, 0, 64:128] *= 1e-40        # BF16 subnormals, many rounding to 0
    x[0, 0, 128:192] = 0.0
    x[0, 1, 192:256] *= 1e-36
    bits["q"] = synth.round_to_bf16_bits(x)
    _check_quant_bit_exact(bits)


# -------------------------------------------------------------- attention

def _compare(out, ref, amb):
    got = out.reshape(ref.shape)
    m = U.metrics(got, ref)
    err = np.abs(got - ref)
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(err <= 1e-2 + amb), float((err - amb).max())
    return m


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
def test_attention_nvfp4_matches_oracle(idx):
    fqa = _fqa()
    w = synth.workload(idx)
    g = U.host_inputs(idx)
    qz, qn = _gpu_nvfp4(g)
    out = fqa.attention_nvfp4(qn, qz, U.SCALE, fqa.FQA_OUT_F32)
    out16 = fqa.attention_nvfp4(qn, qz, U.SCALE, fqa.FQA_OUT_BF16)
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    small = idx == 0
    heads = None if small else U.sample_heads(w)
    rows = None if small else U.sample_rows(w.N)
    # the oracle runs on the GPU's own quantizer outputs (bit-exact with its own)
    ref, amb, _ = oracle.attention_nvfp4(_as_oracle(qz, qn), U.SCALE, heads=heads, rows=rows,
                                         with_ambiguity=True)
    hs = heads or [(b, h) for b in range(w.B) for h in range(w.H)]
    rs = rows or list(range(w.N))
    o = out.cpu().numpy()
    got = np.stack([o[b, h][rs] for b, h in hs])
    m = _compare(got, ref, amb)
    print(f"\n[{w.name}] nvfp4 fp32 out vs oracle: {m}")
    o16 = out16.float().cpu().numpy()
    got16 = np.stack([o16[b, h][rs] for b, h in hs]).astype(np.float64)
    assert np.all(np.abs(got16 - ref) <= np.maximum(1e-2, U.bf16_ulp(ref)) + amb + 1e-12)


@pytest.mark.parametrize("B,H,N", [(2, 96, 128), (2, 24, 1024)])
def test_attention_nvfp4_many_items_per_cta(B, H, N):
    """More work items than SMs: the scale factors of the next item's Q tile
    and first K tile are written while the current item finishes."""
    fqa = _fqa()
    shape = (B, H, N, 128)
    bits = {t: _gen(shape, 70 + i, 2.0) for i, t in enumerate("qkv")}
    qz, qn = _gpu_nvfp4(bits)
    out = fqa.attention_nvfp4(qn, qz, U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    rows = list(range(N)) if N <= 128 else list(range(0, N, 7))
    ref, amb, _ = oracle.attention_nvfp4(_as_oracle(qz, qn), U.SCALE, rows=rows, with_ambiguity=True)
    got = out[:, :, rows].reshape(ref.shape)
    _compare(got, ref, amb)
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK


def test_attention_nvfp4_degenerate_cases():
    """Q all zero: every score 0, so every row is the mean of the V codes
    weighted by the P rule (the oracle's value); V all zero: zero output."""
    fqa = _fqa()
    shape = (1, 2, 256, 128)
    bits = {t: _gen(shape, 50 + i, 1.0) for i, t in enumerate("qkv")}
    bits["q"][:] = 0
    qz, qn = _gpu_nvfp4(bits)
    assert torch.count_nonzero(qn.q4) == 0 and torch.count_nonzero(qn.sq1) == 0
    out = fqa.attention_nvfp4(qn, qz, U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    ref, amb, _ = oracle.attention_nvfp4(_as_oracle(qz, qn), U.SCALE, with_ambiguity=True)
    _compare(out, ref, amb)
    assert np.allclose(out[0, 0, 0], out[0, 0, 255])
    bits["v"][:] = 0
    qz, qn = _gpu_nvfp4(bits)
    out = fqa.attention_nvfp4(qn, qz, U.SCALE, fqa.FQA_OUT_F32)
    assert torch.count_nonzero(out) == 0


def test_attention_nvfp4_deterministic():
    fqa = _fqa()
    g = U.host_inputs(1)
    qz, qn = _gpu_nvfp4(g)
    a = fqa.attention_nvfp4(qn, qz, U.SCALE)
    b = fqa.attention_nvfp4(qn, qz, U.SCALE)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("N", [1, 63, 100, 129, 200, 1000, 4429])
def test_attention_nvfp4_ragged(N):
    """Any sequence length: the short last Q tile and KV tile (keys past N
    take no part; the second 64-key half of the last tile may be empty),
    every row against the oracle on the small cases, sampled rows on 4429."""
    fqa = _fqa()
    shape = (1, 3, N, 128)
    bits = {t: _gen(shape, 30 + i, 2.0) for i, t in enumerate("qkv")}
    qz, qn = _gpu_nvfp4(bits)
    out = fqa.attention_nvfp4(qn, qz, U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    rows = list(range(N)) if N <= 1000 else U.sample_rows(N)
    ref, amb, _ = oracle.attention_nvfp4(_as_oracle(qz, qn), U.SCALE, rows=rows, with_ambiguity=True)
    got = out[:, :, rows].reshape(ref.shape)
    _compare(got, ref, amb)


def test_nvfp4_tracks_fp8_on_workload():
    """The FP4 Q.K variant stays close to the FP8 path on the DiT workload
    (cosine > 0.95 against exact attention on sampled rows, as the oracle
    pins on the small case)."""
    fqa = _fqa()
    w = synth.workload(1)
    g = U.host_inputs(1)
    qz, qn = _gpu_nvfp4(g)
    out = fqa.attention_nvfp4(qn, qz, U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    rows = U.sample_rows(w.N)
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], U.SCALE, heads=[(0, 0)], rows=rows)
    got = out[0, 0][rows].astype(np.float64)
    cos = float((got * ex[0]).sum() / np.sqrt((got * got).sum() * (ex[0] * ex[0]).sum()))
    print(f"\n[{w.name}] nvfp4 cos vs exact (head 0, sampled rows): {cos:.4f}")
    assert cos > 0.9


def test_attention_nvfp4_longest_sequence_sampled():
    """N = 65536 (the maximum), one head, sampled rows against all keys."""
    fqa = _fqa()
    N = 65536
    bits = {t: _gen((1, 1, N, 128), 55 + i) for i, t in enumerate("qkv")}
    qz, qn = _gpu_nvfp4(bits)
    out = fqa.attention_nvfp4(qn, qz, U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    rows = [0, 1, 63, 64, 127, 128, N // 2, N - 129, N - 64, N - 1]
    ref, amb, _ = oracle.attention_nvfp4(_as_oracle(qz, qn), U.SCALE, rows=rows, with_ambiguity=True)
    _compare(out[0, 0][rows][None], ref, amb)
