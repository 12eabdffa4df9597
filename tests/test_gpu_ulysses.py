"""The sequence all-to-all layouts on one GPU ("FLUX 3 Image Klein Base",
sections "결과" and "고를 때 기준": CFG x Ulysses sequence parallel).

fqa_quantize_a2a reads Q, K, V in the layout the forward all-to-all delivers,
[B, P, Hl, Nl, d]; fqa_attention_fp8_a2a writes its output in the layout the
return all-to-all sends.  Both must be bit-identical to the plain calls on the
same tokens.  The last test emulates P ranks on this one GPU: it builds each
rank's receive buffer from the full inputs (the all-to-all as slicing), runs
that rank's kernels, routes the outputs back, and compares the whole result
with single-GPU FP8 attention bit for bit.  No kernel waits on another.
"""

import numpy as np
import pytest
import torch

import fqa_synth as synth
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _fqa():
    import quantized_fp8_attention_b200 as fqa
    return fqa


def _a2a_in(x: torch.Tensor, P: int, r: int) -> torch.Tensor:
    """Rank r's receive buffer [B, P, Hl, Nl, d] from the full [B, H, N, d]:
    chunk p = tokens of rank p for rank r's heads."""
    B, H, N, d = x.shape
    Hl, Nl = H // P, N // P
    heads = x[:, r * Hl:(r + 1) * Hl]                        # [B, Hl, N, d]
    return heads.reshape(B, Hl, P, Nl, d).permute(0, 2, 1, 3, 4).contiguous()


@pytest.mark.parametrize("idx,P", [(1, 2), (2, 4), (3, 8), (4, 4)])
def test_a2a_layout_calls_match_plain_calls(idx, P):
    fqa = _fqa()
    w = synth.workload(idx)
    g = U.host_inputs(idx)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    Hl = w.H // P
    r = P - 1                                                # the last rank's heads
    qa, ka, va = (_a2a_in(t, P, r) for t in (q, k, v))
    qz_a = fqa.quantize_a2a(qa, ka, va)
    sl = slice(r * Hl, (r + 1) * Hl)
    qz = fqa.quantize(*(t[:, sl].contiguous() for t in (q, k, v)))
    for name, a, b in zip(fqa.Quantized._fields, qz_a, qz):
        assert torch.equal(a, b), name
    o_a = fqa.attention_fp8_a2a(qz_a, P, U.SCALE, fqa.FQA_OUT_BF16)          # [B, P, Hl, Nl, d]
    o = fqa.attention_fp8(qz, U.SCALE, fqa.FQA_OUT_BF16)                     # [B, Hl, N, d]
    back = o_a.permute(0, 2, 1, 3, 4).reshape(o.shape)
    assert torch.equal(back.view(torch.int16), o.view(torch.int16))
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK


@pytest.mark.parametrize("idx,P", [(3, 8), (4, 2)])
def test_virtual_ranks_end_to_end_equal_single_gpu(idx, P):
    """P virtual ranks: forward all-to-all as slicing, per-rank kernels, return
    all-to-all as slicing; the assembled output equals single-GPU attention."""
    fqa = _fqa()
    w = synth.workload(idx)
    g = U.host_inputs(idx)
    q, k, v = (U.to_device(g[t]) for t in "qkv")
    B, H, N, d = q.shape
    Hl, Nl = H // P, N // P
    outs = []
    for r in range(P):
        qz = fqa.quantize_a2a(*(_a2a_in(t, P, r) for t in (q, k, v)))
        outs.append(fqa.attention_fp8_a2a(qz, P, U.SCALE, fqa.FQA_OUT_BF16))   # [B, P, Hl, Nl, d]
    # return all-to-all: rank p's shard [B, H, Nl, d] = rank r's chunk p, heads of r
    full = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    for p in range(P):
        shard = torch.cat([outs[r][:, p] for r in range(P)], dim=1)            # [B, H, Nl, d]
        full[:, :, p * Nl:(p + 1) * Nl] = shard
    ref = fqa.attention_fp8(fqa.quantize(q, k, v), U.SCALE, fqa.FQA_OUT_BF16)
    assert torch.equal(full.view(torch.int16), ref.view(torch.int16))


def test_a2a_rejects_bad_shapes():
    fqa = _fqa()
    t = torch.zeros(1, 2, 1, 96, 128, dtype=torch.bfloat16, device="cuda")   # Nl = 96, not a multiple of 64
    qz = fqa.alloc_quantized(1, 1, 192, "cuda")
    ws = fqa.alloc_workspace(1, 1, 192, "cuda")
    assert fqa.fqa_quantize_a2a(t, t, t, *qz, ws) == fqa.FQA_ERR_UNSUPPORTED
