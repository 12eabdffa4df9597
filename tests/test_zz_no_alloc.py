"""fqa_quantize_noalloc through the C ABI against fqa_quantize.

fqa_quantize_noalloc serves callers that cannot allocate device memory at
call time (for example an operator inside a host framework that owns all
device memory): it keeps the K-mean scratch and its counters in a fixed array
(8 MiB + 256 bytes) inside the library instead of taking a workspace.  Its results must equal those of the
workspace entry point bit for bit (the quantizer's tolerance), on two calls in
a row -- the second on a different workload, so stale scratch contents from
the first call cannot leak into it.  This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _outputs(fqa, B, H, N):
    return fqa.alloc_quantized(B, H, N, "cuda")


def test_noalloc_matches_workspace_entry_point_twice():
    import quantized_fp8_attention_b200 as fqa
    L = fqa.lib()
    L.fqa_quantize_noalloc_max_workspace_bytes.restype = ctypes.c_size_t
    assert L.fqa_quantize_noalloc_max_workspace_bytes() == (8 << 20) + 256
    # exactly 16384 blocks of partial sums fit (1 x 16 heads x 65536 tokens)
    assert fqa.fqa_quantize_workspace_bytes(1, 16, 65536) == (8 << 20) + 256
    for idx in (3, 1):                       # two calls in a row, different sizes
        g = U.host_inputs(idx)
        q, k, v = (U.to_device(g[t]) for t in "qkv")
        B, H, N, _ = q.shape
        ref = _outputs(fqa, B, H, N)
        ws = fqa.alloc_workspace(B, H, N, "cuda")
        assert fqa.fqa_quantize(q, k, v, *ref, ws) == fqa.FQA_OK
        got = _outputs(fqa, B, H, N)
        for t in got:
            t.fill_(0x5A if t.dtype == torch.uint8 else -3.0)
        assert fqa.fqa_quantize_noalloc(q, k, v, *got) == fqa.FQA_OK
        torch.cuda.synchronize()
        for name, a, b in zip(ref._fields, ref, got):
            assert torch.equal(a, b), f"workload {idx}: {name} differs"
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import quantized_fp8_attention_b200 as fqa
    # B*H*(N/64)*128*4 bytes = 1*48*1024*512 = 24 MiB > 8 MiB + 256: refused with
    # FQA_ERR_UNSUPPORTED before anything is launched (the pointers below are
    # never dereferenced)
    P = ctypes.c_void_p
    L = fqa.lib()
    L.fqa_quantize_noalloc.restype = ctypes.c_int
    L.fqa_quantize_noalloc.argtypes = [P, P, P] + [ctypes.c_int] * 4 + [P] * 9
    dummy = torch.empty(64, dtype=torch.uint8, device="cuda")
    p = P(dummy.data_ptr())
    st = L.fqa_quantize_noalloc(p, p, p, 1, 48, 65536, 128, p, p, p, p, p, p, p, p, None)
    assert st == fqa.FQA_ERR_UNSUPPORTED
