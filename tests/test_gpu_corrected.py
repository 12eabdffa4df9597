"""Error-corrected FP8 attention on the GPU against the oracle ("FLUX 3 Image
Klein Base: 생성 3.46배, 8장 확장 병목", section "왜 이런 차이가 나나":
VC-Attention FP8 corrects only the tokens with large error, rho = 0.005).

  * the per-key quantization error (fqa_quantize_keyerr) is bit-exact
    against the oracle's pinned-order binary32 sum, on all five workloads;
  * the selection (fqa_select_keys) is bit-exact: the same keys, ties to the
    lower index, the mask words and the ascending index list;
  * the corrected attention matches the oracle's corrected attention within
    the FP8 parity tolerances (FP32 output: mean relative error <= 2e-3 and
    every element within 1e-2 + amb, amb the FP8 part's ambiguity bound
    carried through the merge); its cosine against exact FP64 attention is
    reported next to the plain FP8 path's;
  * rho = 1 (every key exact) matches exact attention like the BF16 path.
"""

import dataclasses

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


def _pick(a, heads, rows):
    if heads is None:
        return a.reshape(-1, a.shape[2], a.shape[3])
    return np.stack([a[b, h][rows] for (b, h) in heads])


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
def test_key_error_and_selection_bit_exact(idx):
    fqa = _fqa()
    g = U.host_inputs(idx)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    qz, k_err = fqa.quantize_keyerr(q, k, v)
    # the quantizer's other outputs are unchanged by the error output
    ref_q = U.oracle_quant(idx)
    got_q = U.to_oracle_quant(qz)
    for name in ref_q:
        assert np.array_equal(np.asarray(got_q[name]).view(np.uint8), np.asarray(ref_q[name]).view(np.uint8)), name
    err = k_err.cpu().numpy()
    ref = oracle.key_error(g["k"], ref_q)
    assert np.array_equal(err.view(np.uint32), ref.view(np.uint32))
    B, H, N = err.shape
    for kc in (1, fqa.fqa_corrected_keys(N, 0.005), fqa.fqa_corrected_keys(N, 0.05)):
        kmask = torch.empty(B, H, (N + 31) // 32, dtype=torch.int32, device="cuda")
        ids = torch.empty(B, H, kc, dtype=torch.int32, device="cuda")
        assert fqa.fqa_select_keys(k_err, kc, kmask, ids) == fqa.FQA_OK
        sel = oracle.select_keys(ref, kc)
        words = kmask.cpu().numpy().view(np.uint32)
        bits = np.unpackbits(words.view(np.uint8), bitorder="little").reshape(B, H, -1)[:, :, :N]
        assert np.array_equal(bits, sel), kc
        want = np.stack([np.stack([np.flatnonzero(sel[b, h]) for h in range(H)]) for b in range(B)])
        assert np.array_equal(ids.cpu().numpy(), want), kc
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK


def test_selection_ties_and_extremes():
    fqa = _fqa()
    rng = np.random.default_rng(50)
    N = 3000
    err = rng.integers(0, 6, size=(2, 3, N)).astype(np.float32)     # many ties
    err[0, 0, :] = 1.0                                               # all equal
    t = torch.from_numpy(err).cuda()
    for kc in (1, 7, 64, 1000, N - 1, N):
        kmask = torch.empty(2, 3, (N + 31) // 32, dtype=torch.int32, device="cuda")
        ids = torch.empty(2, 3, kc, dtype=torch.int32, device="cuda")
        assert fqa.fqa_select_keys(t, kc, kmask, ids) == fqa.FQA_OK
        sel = oracle.select_keys(err, kc)
        bits = np.unpackbits(kmask.cpu().numpy().view(np.uint8), bitorder="little").reshape(2, 3, -1)[:, :, :N]
        assert np.array_equal(bits, sel), kc


def _corrected_case(w, rho, heads, rows):
    fqa = _fqa()
    g = synth.generate(w, heads=heads) if heads is not None else synth.generate(w)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    qz, k_err = fqa.quantize_keyerr(q, k, v)
    out32 = fqa.attention_fp8_corrected(q, k, v, qz, k_err, U.SCALE, rho, fqa.FQA_OUT_F32)
    out16 = fqa.attention_fp8_corrected(q, k, v, qz, k_err, U.SCALE, rho, fqa.FQA_OUT_BF16)
    plain = fqa.attention_fp8(qz, U.SCALE, fqa.FQA_OUT_F32)
    torch.cuda.synchronize()
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    oq = oracle.quantize(g["q"], g["k"], g["v"])
    sel = oracle.select_keys(oracle.key_error(g["k"], oq), oracle.n_corrected(w.N, rho))
    ref, amb = oracle.attention_fp8_corrected(g, oq, sel, U.SCALE, heads=heads, rows=rows, with_ambiguity=True)
    return g, out32, out16, plain, ref, amb


# (1, 0.25): 320 corrected keys per head -- the x3 text keys fill the first
# two KV tiles, so rows start with tiles that have no FP8 key at all, and the
# exact part runs in three 128-key chunks
@pytest.mark.parametrize("idx,rho", [(0, 0.005), (0, 0.05), (1, 0.005), (1, 0.05), (1, 0.25), (2, 0.005),
                                     (3, 0.005), (4, 0.005)])
def test_corrected_attention_matches_oracle(idx, rho):
    w = synth.workload(idx)
    heads, rows = _rows_heads(w)
    g, out32, out16, plain, ref, amb = _corrected_case(w, rho, heads, rows)
    got = _pick(out32.cpu().numpy(), heads, rows).astype(np.float64)
    m = U.metrics(got, ref)
    err = np.abs(got - ref)
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], U.SCALE, heads=heads, rows=rows)
    cos_c = U.metrics(got, ex)["cos"]
    cos_p = U.metrics(_pick(plain.cpu().numpy(), heads, rows), ex)["cos"]
    print(f"\n[{w.name} rho={rho}] corrected vs oracle: {m}; cos vs exact FP64: corrected {cos_c:.6f}, "
          f"plain FP8 {cos_p:.6f}, oracle {U.metrics(ref, ex)['cos']:.6f}; meets 0.995: {cos_c >= 0.995}")
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(err <= 1e-2 + amb), float((err - amb).max())
    assert cos_c >= cos_p - 1e-4
    # the BF16 output is the FP32 output rounded once
    b16 = out16.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(b16, oracle.bf16_round(out32.cpu().numpy().astype(np.float64)))


@pytest.mark.parametrize("N,n_text", [(200, 64), (1000, 77), (4429, 333)])
def test_corrected_attention_ragged(N, n_text):
    w0 = synth.workload(2)
    w = dataclasses.replace(w0, name=f"ragged{N}", n_text=n_text, n_img=N - n_text)
    heads = [(0, 0), (0, 11)]
    rows = list(range(N)) if N <= 1000 else U.sample_rows(N)
    g, out32, _, _, ref, amb = _corrected_case(w, 0.02, heads, rows)
    got = _pick(out32.cpu().numpy(), heads, rows).astype(np.float64)
    m = U.metrics(got, ref)
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(np.abs(got - ref) <= 1e-2 + amb)


def test_every_key_corrected_is_exact_attention():
    fqa = _fqa()
    w = synth.workload(1)
    heads = [(0, 3), (0, 20)]
    g = synth.generate(w, heads=heads)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    qz, k_err = fqa.quantize_keyerr(q, k, v)
    out = fqa.attention_fp8_corrected(q, k, v, qz, k_err, U.SCALE, 1.0, fqa.FQA_OUT_F32).cpu().numpy()
    rows = list(range(0, w.N, 3))
    ex = oracle.attention_exact(g["q"], g["k"], g["v"], U.SCALE, heads=heads, rows=rows)
    got = _pick(out, heads, rows).astype(np.float64)
    m = U.metrics(got, ex)
    print(f"\n[rho=1] vs exact FP64: {m}")
    assert m["cos"] >= 0.99999 and m["mean_rel"] <= 1e-4, m
    assert np.all(np.abs(got - ex) <= 1e-3 + 1e-4 * np.abs(ex))


@pytest.mark.parametrize("layout", ["block_left_with_one_key", "first_and_last_keys_kept"])
def test_patched_tiles_extreme_blocks(layout):
    """The patched FP8 part (fewer than 64 corrected keys per head) at its
    limits, with the key errors chosen by hand (the call takes them as input):
    63 corrected keys in one 64-key block, so its single kept key (the last)
    is copied 63 times; or 63 corrected keys spread over all four blocks, the
    copied key being the block's first, or one in its middle, or after a
    corrected first key.  Against the oracle with the same selection."""
    fqa = _fqa()
    w = dataclasses.replace(synth.workload(0), name="patch_extremes")      # B=1, H=2, N=256
    g = synth.generate(w)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    qz, _ = fqa.quantize_keyerr(q, k, v)
    N = w.N
    err = np.zeros((w.B, w.H, N), np.float32)
    if layout == "block_left_with_one_key":
        err[:, :, 64:127] = 2.0                       # keys 64..126 of block 1; key 127 kept
        rho = 63 / 256
    else:
        err[:, :, 0:16] = 2.0                         # block 0: copies key 16
        err[:, :, 65:80] = 1.5                        # block 1: copies key 64
        err[:, :, 128:144] = 3.0                      # block 2: copies key 144
        err[:, :, 240:256] = 1.0                      # block 3: copies key 192; 16 + 15 + 16 + 16 = 63
        rho = 63 / 256
    kc = fqa.fqa_corrected_keys(N, rho)
    assert kc == 63 and int((err > 0).sum(axis=2).max()) == 63
    k_err = torch.from_numpy(err).cuda()
    out32 = fqa.attention_fp8_corrected(q, k, v, qz, k_err, U.SCALE, rho, fqa.FQA_OUT_F32)
    torch.cuda.synchronize()
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    oq = oracle.quantize(g["q"], g["k"], g["v"])
    sel = oracle.select_keys(err, kc)
    assert np.array_equal(sel.astype(bool), err > 0)
    ref, amb = oracle.attention_fp8_corrected(g, oq, sel, U.SCALE, with_ambiguity=True)
    got = out32.cpu().numpy().reshape(ref.shape).astype(np.float64)
    m = U.metrics(got, ref)
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(np.abs(got - ref) <= 1e-2 + amb), float((np.abs(got - ref) - amb).max())


@pytest.mark.parametrize("rho", [0.0005, 0.005])
def test_corrected_longest_sequence_sampled(rho):
    """N = 65536 (the maximum), one head: 33 corrected keys (patched FP8 part)
    and 328 (key-masked FP8 part, exact part in three chunks); the selection
    reads the errors from global memory at this length.  Sampled rows."""
    fqa = _fqa()
    N = 65536
    rng = np.random.default_rng(77)
    g = {t: synth.round_to_bf16_bits(rng.standard_normal((1, 1, N, 128)) * s)
         for t, s in zip("qkv", (2.0, 2.0, 1.0))}
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    qz, k_err = fqa.quantize_keyerr(q, k, v)
    out32 = fqa.attention_fp8_corrected(q, k, v, qz, k_err, U.SCALE, rho, fqa.FQA_OUT_F32).cpu().numpy()
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    oq = oracle.quantize(g["q"], g["k"], g["v"])
    kc = oracle.n_corrected(N, rho)
    assert kc == fqa.fqa_corrected_keys(N, rho)
    err = oracle.key_error(g["k"], oq)
    assert np.array_equal(err.view(np.uint32), k_err.cpu().numpy().view(np.uint32))
    sel = oracle.select_keys(err, kc)
    rows = [0, 1, 63, 64, 127, 128, N // 2, N - 129, N - 64, N - 1]
    ref, amb = oracle.attention_fp8_corrected(g, oq, sel, U.SCALE, rows=rows, with_ambiguity=True)
    got = out32[0, 0][rows].astype(np.float64)[None]
    m = U.metrics(got, ref)
    assert m["mean_rel"] <= 2e-3, m
    assert np.all(np.abs(got - ref) <= 1e-2 + amb), float((np.abs(got - ref) - amb).max())
