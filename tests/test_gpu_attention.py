"""fqa_attention_fp8 / fqa_attention_bf16 on the GPU against the oracle.

FP8 path, per workload (full tensors on the GPU, in the launch configuration
the benchmark times; all rows checked on the two small workloads, sampled
heads x rows [0,128) u [N/2,N/2+128) u [N-128,N) against all keys on the
large ones):
  (i)  FP32 verification output vs the oracle's binary64 output:
       mean relative error <= 2e-3 and every element within 1e-2 + amb, where
       amb is the oracle's bound on what P codes lying within binary32
       evaluation error of an E4M3 rounding midpoint can change (such a code
       may round either way; elsewhere amb = 0 and the bound is 1e-2);
  (ii) BF16 output vs the oracle's output rounded once to BF16: mean relative
       error <= 2e-3 and every element within max(1e-2, one BF16 ulp of ref)
       + amb;
  (iii) cosine vs exact unquantized FP64 attention, reported; it must not fall
       more than 1e-3 below the oracle's own (the scheme's ceiling), and must
       reach 0.995 where the oracle does.
BF16 path: vs exact FP64 attention, cos >= 0.9999, mean rel <= 1e-2, FP32
output within 2e-2 + 2^-8 |ref| elementwise.
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


def _rows_heads(w):
    if w.B * w.H * w.N <= 24 * 1280:
        return None, None
    return U.sample_heads(w), U.sample_rows(w.N)


def _pick(a: np.ndarray, heads, rows):
    """[B,H,N,d] -> [n_heads, n_rows, d] in the oracle's order."""
    if heads is None:
        return a.reshape(-1, a.shape[2], a.shape[3])
    return np.stack([a[b, h][rows] for (b, h) in heads])


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
def test_fp8_attention_matches_oracle(idx):
    fqa = _fqa()
    w = synth.workload(idx)
    g = U.host_inputs(idx)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    qz = fqa.quantize(q, k, v)
    out32 = fqa.attention_fp8(qz, U.SCALE, fqa.FQA_OUT_F32)
    out16 = fqa.attention_fp8(qz, U.SCALE, fqa.FQA_OUT_BF16)
    torch.cuda.synchronize()
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    heads, rows = _rows_heads(w)
    ref, amb, namb = oracle.attention_fp8(U.oracle_quant(idx), U.SCALE, heads=heads, rows=rows,
                                          with_ambiguity=True)
    got32 = _pick(out32.cpu().numpy(), heads, rows)
    m = U.metrics(got32, ref)
    err = np.abs(got32 - ref)
    print(f"\n[{w.name}] fp32 out vs oracle: {m}; ambiguous P codes {int(namb.sum())}, "
          f"elements over 1e-2: {int((err > 1e-2).sum())} (all covered: {bool(np.all(err <= 1e-2 + amb))})")
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(err <= 1e-2 + amb), float((err - amb).max())
    # (ii) production BF16 output
    got16 = U.bf16_bits_to_f64(_pick(out16.view(torch.int16).cpu().numpy().view(np.uint16), heads, rows))
    ref16 = U.bf16_bits_to_f64(oracle.bf16_round(ref))
    m16 = U.metrics(got16, ref16)
    print(f"[{w.name}] bf16 out vs oracle(bf16): {m16}")
    assert m16["mean_rel"] <= 2e-3, m16
    assert np.all(np.abs(got16 - ref16) <= np.maximum(1e-2, U.bf16_ulp(ref16)) + amb + 1e-12)
    # the BF16 output is the FP32 output rounded once to nearest even
    b16 = out16.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(b16, oracle.bf16_round(out32.cpu().numpy().astype(np.float64)))
    # (iii) accuracy against exact attention
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], U.SCALE, heads=heads, rows=rows)
    cos_gpu = U.metrics(got32, ex)["cos"]
    cos_orc = U.metrics(ref, ex)["cos"]
    print(f"[{w.name}] cos vs exact FP64: gpu {cos_gpu:.6f}  oracle {cos_orc:.6f}  "
          f"meets 0.995: {cos_gpu >= 0.995}")
    assert cos_gpu >= cos_orc - 1e-3
    if cos_orc >= 0.995:
        assert cos_gpu >= 0.995


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
def test_bf16_attention_matches_exact(idx):
    fqa = _fqa()
    w = synth.workload(idx)
    g = U.host_inputs(idx)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    out32 = fqa.attention_bf16(q, k, v, U.SCALE, fqa.FQA_OUT_F32)
    out16 = fqa.attention_bf16(q, k, v, U.SCALE, fqa.FQA_OUT_BF16)
    torch.cuda.synchronize()
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    heads, rows = _rows_heads(w)
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], U.SCALE, heads=heads, rows=rows)
    got = _pick(out32.cpu().numpy(), heads, rows)
    m = U.metrics(got, ex)
    print(f"\n[{w.name}] bf16 path fp32 out vs exact: {m}")
    assert m["cos"] >= 0.9999 and m["mean_rel"] <= 1e-2, m
    assert np.all(np.abs(got - ex) <= 2e-2 + 2.0 ** -8 * np.abs(ex))
    b16 = out16.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(b16, oracle.bf16_round(out32.cpu().numpy().astype(np.float64)))


# The scheme's own ceiling (the oracle's cos against exact FP64) is below 0.995
# on the four workloads with x20 outlier channels; these cases stay visible as
# expected failures instead of being dropped.
_CEILING = "scheme ceiling: the oracle itself stays below cos 0.995 on x20 outlier channels"


@pytest.mark.parametrize("idx", [0] + [pytest.param(i, marks=pytest.mark.xfail(reason=_CEILING, strict=True))
                                       for i in (1, 2, 3, 4)])
def test_fp8_cos_target_vs_exact(idx):
    """The accuracy target: cos >= 0.995 against exact unquantized FP64
    attention (sampled heads x rows on the large workloads)."""
    fqa = _fqa()
    w = synth.workload(idx)
    g = U.host_inputs(idx)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    out32 = fqa.attention_fp8(fqa.quantize(q, k, v), U.SCALE, fqa.FQA_OUT_F32)
    heads, rows = _rows_heads(w)
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], U.SCALE, heads=heads, rows=rows)
    cos = U.metrics(_pick(out32.cpu().numpy(), heads, rows), ex)["cos"]
    print(f"\n[{w.name}] FP8 cos vs exact FP64: {cos:.6f} (target 0.995)")
    assert cos >= 0.995


def _gen(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return synth.round_to_bf16_bits(rng.standard_normal(shape) * scale)


@pytest.mark.parametrize("N", [128, 256, 384])
def test_fp8_small_sequences_all_rows(N):
    """Single-tile and few-tile sequences, B*H = 3 heads, every row."""
    fqa = _fqa()
    shape = (1, 3, N, 128)
    bits = {t: _gen(shape, 20 + i, 2.0) for i, t in enumerate("qkv")}
    q, k, v = (U.to_device(bits[t]) for t in "qkv")
    out = fqa.attention_fp8(fqa.quantize(q, k, v), U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    ref, amb, _ = oracle.attention_fp8(oracle.quantize(bits["q"], bits["k"], bits["v"]), U.SCALE,
                                       with_ambiguity=True)
    m = U.metrics(out.reshape(ref.shape), ref)
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(np.abs(out.reshape(ref.shape) - ref) <= 1e-2 + amb)


def test_fp8_uniform_scores_give_mean_of_v():
    """Q = 0: every score is 0; with V made of one repeated 64 x 128 block all
    V scales are equal, P = 448 exactly, and the output is the mean of the
    dequantized V rows."""
    fqa = _fqa()
    rng = np.random.default_rng(30)
    blk = rng.standard_normal((64, 128))
    vb = synth.round_to_bf16_bits(np.tile(blk, (4, 1)).reshape(1, 1, 256, 128))
    kb = _gen((1, 1, 256, 128), 31)
    qb = np.zeros_like(kb)
    out = fqa.attention_fp8(fqa.quantize(*(U.to_device(x) for x in (qb, kb, vb))), U.SCALE,
                            fqa.FQA_OUT_F32).cpu().numpy()[0, 0]
    qz = oracle.quantize(qb, kb, vb)
    deq = oracle.e4m3_decode(qz["v8"][0, 0]) * np.repeat(qz["sv"][0, 0].astype(np.float64), 64)[:, None]
    assert np.max(np.abs(out - deq.mean(axis=0)[None, :])) < 1e-5


def test_fp8_zero_v_gives_zero():
    fqa = _fqa()
    qb, kb = _gen((1, 1, 256, 128), 40), _gen((1, 1, 256, 128), 41)
    vb = np.zeros_like(qb)
    out = fqa.attention_fp8(fqa.quantize(*(U.to_device(x) for x in (qb, kb, vb))), U.SCALE,
                            fqa.FQA_OUT_F32)
    assert torch.count_nonzero(out).item() == 0


def test_fp8_longest_sequence_sampled():
    """N = 65536 (the v1 maximum), one head, sampled rows against all keys."""
    fqa = _fqa()
    N = 65536
    bits = {t: _gen((1, 1, N, 128), 50 + i) for i, t in enumerate("qkv")}
    q, k, v = (U.to_device(bits[t]) for t in "qkv")
    out = fqa.attention_fp8(fqa.quantize(q, k, v), U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    rows = [0, 1, 63, 64, 127, 128, N // 2, N - 129, N - 64, N - 1]
    ref, amb, _ = oracle.attention_fp8(oracle.quantize(bits["q"], bits["k"], bits["v"]), U.SCALE,
                                       rows=rows, with_ambiguity=True)
    m = U.metrics(out[0, 0][rows], ref[0])
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(np.abs(out[0, 0][rows] - ref[0]) <= 1e-2 + amb[0])


def test_fp8_deterministic():
    fqa = _fqa()
    g = U.host_inputs(1)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    qz = fqa.quantize(q, k, v)
    a = fqa.attention_fp8(qz, U.SCALE)
    b = fqa.attention_fp8(qz, U.SCALE)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_attention_rejects_bad_arguments():
    fqa = _fqa()
    t = torch.zeros(1, 1, 192, 64, dtype=torch.uint8, device="cuda")    # d != 128
    s = torch.ones(1, 1, 3, device="cuda")
    sm = torch.ones(1, 1, device="cuda")
    out = torch.empty(1, 1, 192, 128, dtype=torch.bfloat16, device="cuda")
    assert fqa.fqa_attention_fp8(t, t, t, s, s, s, sm, U.SCALE, out, 0) == fqa.FQA_ERR_UNSUPPORTED
    t = torch.zeros(1, 1, 128, 128, dtype=torch.uint8, device="cuda")
    out = torch.empty(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    assert fqa.fqa_attention_fp8(t, t, t, s, s, s, sm, float("nan"), out, 0) == fqa.FQA_ERR_INVALID_ARG
    assert fqa.fqa_attention_fp8(t, t, t, s, s, s, sm, U.SCALE, out, 7) == fqa.FQA_ERR_INVALID_ARG
    tb = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    assert fqa.fqa_attention_bf16(tb, tb, tb, -1.0, out, 0) == fqa.FQA_ERR_INVALID_ARG


@pytest.mark.parametrize("B,H,N", [(2, 96, 128), (1, 200, 384)])
def test_fp8_many_items_per_cta(B, H, N):
    """More work items than SMs: with N = 128 every item has one KV tile, so
    the per-item barriers (Q reload, PV completion, the halves' row sums)
    turn over on every tile; with N = 384 the second Q tile of each item's
    last pair lies beyond N.  Every row against the oracle."""
    fqa = _fqa()
    shape = (B, H, N, 128)
    bits = {t: _gen(shape, 60 + i, 2.0) for i, t in enumerate("qkv")}
    q, k, v = (U.to_device(bits[t]) for t in "qkv")
    out = fqa.attention_fp8(fqa.quantize(q, k, v), U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    ref, amb, _ = oracle.attention_fp8(oracle.quantize(bits["q"], bits["k"], bits["v"]), U.SCALE,
                                       with_ambiguity=True)
    got = out.reshape(ref.shape)
    m = U.metrics(got, ref)
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(np.abs(got - ref) <= 1e-2 + amb)
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK


def test_bf16_many_items_per_cta():
    """The BF16 path with more work items than SMs and one KV tile per item."""
    fqa = _fqa()
    shape = (2, 96, 128, 128)
    bits = {t: _gen(shape, 70 + i) for i, t in enumerate("qkv")}
    q, k, v = (U.to_device(bits[t]) for t in "qkv")
    out = fqa.attention_bf16(q, k, v, U.SCALE, fqa.FQA_OUT_F32).cpu().numpy().astype(np.float64)
    ex = oracle.attention_exact(bits["q"], bits["k"], bits["v"], U.SCALE)
    got = out.reshape(ex.shape)
    m = U.metrics(got, ex)
    assert m["cos"] >= 0.9999 and m["mean_rel"] <= 1e-2, m
    assert np.all(np.abs(got - ex) <= 2e-2 + 2.0 ** -8 * np.abs(ex))
