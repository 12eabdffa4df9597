"""fqa_quantize on the GPU against the oracle: codes, scales, K mean and V head
maximum must be bit-identical on all five workloads (full tensors)."""

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


@pytest.mark.parametrize("idx", [0, 1, 2, 3, 4])
def test_quantize_bit_exact(idx):
    fqa = _fqa()
    g = U.host_inputs(idx)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    qz = fqa.quantize(q, k, v)
    torch.cuda.synchronize()
    got = U.to_oracle_quant(qz)
    ref = U.oracle_quant(idx)
    for name in ("k_mean", "sq", "sk", "sv", "sv_max"):
        assert np.array_equal(got[name].view(np.uint32), ref[name].view(np.uint32)), name
    for name in ("q8", "k8", "v8"):
        bad = np.count_nonzero(got[name] != ref[name])
        assert bad == 0, f"{name}: {bad} codes differ"
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK


def test_quantize_deterministic_and_canaries():
    fqa = _fqa()
    w = synth.workload(1)
    g = U.host_inputs(1)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    B, H, N = w.B, w.H, w.N
    pad = 4096
    # outputs carved out of larger buffers whose guard regions must stay untouched

    def guarded(shape, dtype, fill):
        n = int(np.prod(shape))
        base = torch.full((n + 2 * pad,), fill, dtype=dtype, device="cuda")
        return base, base[pad:pad + n].view(*shape)

    outs = []
    for _ in range(2):
        holders = []
        parts = []
        for shape, dt, fill in (((B, H, N, 128), torch.uint8, 0xA5), ((B, H, N, 128), torch.uint8, 0xA5),
                                ((B, H, N, 128), torch.uint8, 0xA5), ((B, H, fqa.nblocks(N)), torch.float32, -7.0),
                                ((B, H, fqa.nblocks(N)), torch.float32, -7.0), ((B, H, fqa.nblocks(N)), torch.float32, -7.0),
                                ((B, H), torch.float32, -7.0), ((B, H, 128), torch.float32, -7.0)):
            base, view = guarded(shape, dt, fill)
            holders.append((base, view.numel(), fill))
            parts.append(view)
        qz = fqa.Quantized(*parts)
        fqa.quantize(q, k, v, out=qz)
        torch.cuda.synchronize()
        for base, n, fill in holders:
            assert torch.all(base[:pad] == fill) and torch.all(base[pad + n:] == fill)
        outs.append([t.clone() for t in qz])
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_quantize_edge_blocks():
    """Zero blocks (scale 0, codes 0), a block whose max is exactly 448, and a
    single-block sequence (N = 64)."""
    fqa = _fqa()
    rng = np.random.default_rng(11)
    x = rng.standard_normal((1, 2, 192, 128)) * 5
    x[0, 0, 64:128] = 0.0                     # a zero block of Q, K and V
    x[0, 1, 0:64] = np.clip(x[0, 1, 0:64], -400, 400)
    x[0, 1, 5, 9] = 448.0
    bits = synth.round_to_bf16_bits(x)
    ref = oracle.quantize(bits, bits, bits)
    t = U.to_device(bits)
    got = U.to_oracle_quant(fqa.quantize(t, t, t))
    for name in ref:
        assert np.array_equal(np.asarray(got[name]).view(np.uint8), np.asarray(ref[name]).view(np.uint8)), name
    bits64 = synth.round_to_bf16_bits(rng.standard_normal((1, 1, 64, 128)))
    ref = oracle.quantize(bits64, bits64, bits64)
    t = U.to_device(bits64)
    got = U.to_oracle_quant(fqa.quantize(t, t, t))
    for name in ref:
        assert np.array_equal(np.asarray(got[name]).view(np.uint8), np.asarray(ref[name]).view(np.uint8)), name


def test_quantize_rejects_bad_arguments():
    fqa = _fqa()
    t = torch.zeros(1, 1, 100, 64, dtype=torch.bfloat16, device="cuda")    # d != 128
    qz = fqa.alloc_quantized(1, 1, 128, "cuda")
    ws = fqa.alloc_workspace(1, 1, 128, "cuda")
    assert fqa.fqa_quantize(t, t, t, *qz, ws) == fqa.FQA_ERR_UNSUPPORTED
    t = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16, device="cuda")
    small = torch.empty(4, dtype=torch.float32, device="cuda")
    assert fqa.fqa_quantize(t, t, t, *qz, small) == fqa.FQA_ERR_INVALID_ARG
    raw = torch.zeros(128 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    mis = raw[1:1 + 128 * 128].view(1, 1, 128, 128)                        # 2-byte offset
    assert fqa.fqa_quantize(mis, t, t, *qz, ws) == fqa.FQA_ERR_MISALIGNED


def test_bounded_wait_times_out_and_context_survives():
    """A wait on a barrier nothing arrives on gives up after its limit, sets the
    timeout bit, and leaves the context usable (no trap, no hang)."""
    fqa = _fqa()
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
    assert fqa.fqa_debug_wait_timeout(20000) == fqa.FQA_OK      # 20 ms
    st, flags = fqa.fqa_debug_status()
    assert st == fqa.FQA_ERR_TIMEOUT and flags & 1
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK              # cleared by the read
    # the context still runs kernels correctly
    g = U.host_inputs(0)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    got = U.to_oracle_quant(fqa.quantize(q, k, v))
    ref = U.oracle_quant(0)
    assert np.array_equal(got["q8"], ref["q8"])


def test_quantize_tiny_blocks():
    """Blocks whose 448/amax overflows binary32 (codes from x / s) and a
    smoothed-K block whose scale underflows (flushed to signed zeros):
    bit-exact against the oracle, and no NaN code (S.1111.111) anywhere."""
    fqa = _fqa()
    N = 1024
    x = np.zeros((1, 2, N, 128))
    x[0, 0, 0, 0] = 2.0 ** -123
    x[0, 0, 1, 5] = -(2.0 ** -123)
    x[0, 0, 2, 9] = 2.0 ** -130
    x[0, 0, 3, 127] = 2.0 ** -133
    x[0, 1, 1000, 0] = 2.0 ** -133          # head 1: K mean 2^-143, blocks 0..14 flushed
    x[0, 0, 64:128] = np.random.default_rng(12).standard_normal((64, 128))   # an ordinary block
    bits = synth.round_to_bf16_bits(x)
    ref = oracle.quantize(bits, bits, bits)
    t = U.to_device(bits)
    got = U.to_oracle_quant(fqa.quantize(t, t, t))
    torch.cuda.synchronize()
    for name in ref:
        assert np.array_equal(np.asarray(got[name]).view(np.uint8), np.asarray(ref[name]).view(np.uint8)), name
    for name in ("q8", "k8", "v8"):
        assert not np.any((got[name] & 0x7F) == 0x7F), name
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
