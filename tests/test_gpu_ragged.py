"""Sequences whose length is not a multiple of 64 or 128 (real prompt lengths:
text tokens follow the prompt, so N = n_text + image tokens is ragged), on the
GPU against the oracle.

Readings under test: the last 64-token block of a head holds the remaining
tokens and its scale is their absmax alone; the K mean divides by N; the last
KV tile holds N % 128 keys and keys past N do not exist (no p, no row-sum
term, no P code).  Quantizer outputs must be bit-exact; attention within the
parity tolerances of the full-tile tests; nothing may be written past the end
of any output (canaries)."""

import dataclasses

import numpy as np
import pytest
import torch

import fqa_synth as synth
import oracle
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

RAGGED = [1, 2, 63, 65, 100, 129, 200, 255, 383, 1000]


def _fqa():
    import quantized_fp8_attention_b200 as fqa
    return fqa


def _inputs(B, H, N, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, N, 128)) * 2.0
    k = rng.standard_normal((B, H, N, 128)) * 2.0 + rng.standard_normal((B, H, 1, 128)) * 2.0
    v = rng.standard_normal((B, H, N, 128))
    return {t: synth.round_to_bf16_bits(x) for t, x in zip("qkv", (q, k, v))}


class Guarded:
    """A device buffer with canary regions on both sides of its view."""
    PAD = 4096

    def __init__(self, shape, dtype, fill):
        n = int(np.prod(shape))
        self.base = torch.full((n + 2 * self.PAD,), fill, dtype=dtype, device="cuda")
        self.view = self.base[self.PAD:self.PAD + n].view(*shape)
        self.n, self.fill = n, fill

    def intact(self) -> bool:
        b = self.base
        return bool(torch.all(b[:self.PAD] == self.fill)) and bool(torch.all(b[self.PAD + self.n:] == self.fill))


@pytest.mark.parametrize("N", RAGGED + [8703])
def test_quantize_ragged_bit_exact(N):
    fqa = _fqa()
    B, H = 1, 3
    bits = _inputs(B, H, N, 100 + N)
    nb = fqa.nblocks(N)
    bufs = [Guarded((B, H, N, 128), torch.uint8, 0xA5) for _ in range(3)] + \
           [Guarded((B, H, nb), torch.float32, -7.0) for _ in range(3)] + \
           [Guarded((B, H), torch.float32, -7.0), Guarded((B, H, 128), torch.float32, -7.0)]
    qz = fqa.Quantized(*(g.view for g in bufs))
    fqa.quantize(*(U.to_device(bits[t]) for t in "qkv"), out=qz)
    torch.cuda.synchronize()
    assert all(g.intact() for g in bufs), "a write past the end of an output"
    got = U.to_oracle_quant(qz)
    ref = oracle.quantize(bits["q"], bits["k"], bits["v"])
    for name in ref:
        assert np.array_equal(np.asarray(got[name]).view(np.uint8), np.asarray(ref[name]).view(np.uint8)), name
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK


@pytest.mark.parametrize("N", RAGGED)
def test_fp8_attention_ragged_all_rows(N):
    fqa = _fqa()
    B, H = 1, 3
    bits = _inputs(B, H, N, 200 + N)
    qz = fqa.quantize(*(U.to_device(bits[t]) for t in "qkv"))
    out = Guarded((B, H, N, 128), torch.float32, -9.0)
    out16 = Guarded((B, H, N, 128), torch.bfloat16, -9.0)
    fqa.attention_fp8(qz, U.SCALE, fqa.FQA_OUT_F32, out=out.view)
    fqa.attention_fp8(qz, U.SCALE, fqa.FQA_OUT_BF16, out=out16.view)
    torch.cuda.synchronize()
    assert out.intact() and out16.intact(), "a write past the end of the output"
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    ref, amb, _ = oracle.attention_fp8(oracle.quantize(bits["q"], bits["k"], bits["v"]), U.SCALE,
                                       with_ambiguity=True)
    got = out.view.cpu().numpy().reshape(ref.shape).astype(np.float64)
    m = U.metrics(got, ref)
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(np.abs(got - ref) <= 1e-2 + amb), float((np.abs(got - ref) - amb).max())
    b16 = out16.view.view(torch.int16).cpu().numpy().view(np.uint16).reshape(ref.shape)
    assert np.array_equal(b16, oracle.bf16_round(got))


def _text_length_variant(idx, n_text):
    w = synth.workload(idx)
    return dataclasses.replace(w, name=f"{w.name}_text{n_text}", n_text=n_text)


@pytest.mark.parametrize("idx,n_text", [(1, 77), (2, 333), (3, 301)])
def test_fp8_attention_real_text_lengths(idx, n_text):
    """The DiT workloads with a prompt of n_text tokens instead of a padded
    multiple of 128 (N = 1101, 4429, 8493): sampled heads x rows against all
    keys, within the parity tolerances; cosine against exact FP64 reported."""
    fqa = _fqa()
    w = _text_length_variant(idx, n_text)
    heads = U.sample_heads(w)
    g = synth.generate(w, heads=heads)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    out = fqa.attention_fp8(fqa.quantize(q, k, v), U.SCALE, fqa.FQA_OUT_F32).cpu().numpy()
    rows = U.sample_rows(w.N) + [n_text - 1, n_text, w.N - 1]
    ref, amb, _ = oracle.attention_fp8(oracle.quantize(g["q"], g["k"], g["v"]), U.SCALE,
                                       heads=heads, rows=rows, with_ambiguity=True)
    got = np.stack([out[b, h][rows] for (b, h) in heads]).astype(np.float64)
    m = U.metrics(got, ref)
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], U.SCALE, heads=heads, rows=rows)
    print(f"\n[{w.name} N={w.N}] fp32 out vs oracle: {m}; cos vs exact FP64 {U.metrics(got, ex)['cos']:.6f}")
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(np.abs(got - ref) <= 1e-2 + amb)


@pytest.mark.parametrize("N", [1, 65, 200, 383, 1000, 4429])
def test_bf16_attention_ragged(N):
    fqa = _fqa()
    B, H = 1, 2
    bits = _inputs(B, H, N, 300 + N)
    q, k, v = (U.to_device(bits[t]) for t in "qkv")
    out = Guarded((B, H, N, 128), torch.float32, -9.0)
    fqa.attention_bf16(q, k, v, U.SCALE, fqa.FQA_OUT_F32, out=out.view)
    torch.cuda.synchronize()
    assert out.intact()
    rows = list(range(N)) if N <= 1000 else U.sample_rows(N)
    ex = oracle.attention_exact(bits["q"], bits["k"], bits["v"], U.SCALE, rows=rows)
    got = out.view.cpu().numpy()[:, :, rows].reshape(ex.shape).astype(np.float64)
    m = U.metrics(got, ex)
    assert m["cos"] >= 0.9999 and m["mean_rel"] <= 1e-2, m
    assert np.all(np.abs(got - ex) <= 2e-2 + 2.0 ** -8 * np.abs(ex))
