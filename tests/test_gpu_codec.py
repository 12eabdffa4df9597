"""The GPU's binary32 -> E4M3 conversion (the instruction the quantizer and the
attention kernel use) against the oracle's encoder for all 2^32 inputs."""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def test_e4m3_encode_exhaustive():
    import quantized_fp8_attention_b200 as fqa
    chunk = 1 << 26
    for c in range((1 << 32) // chunk):
        lo = c * chunk
        bits = np.arange(lo, lo + chunk, dtype=np.uint64).astype(np.uint32)
        x = bits.view(np.float32)
        xt = torch.from_numpy(bits.view(np.int32)).cuda().view(torch.float32)
        got = fqa.e4m3_encode(xt).cpu().numpy()
        ref = oracle.e4m3_encode(x)
        nan = np.isnan(x)
        if nan.any():
            # NaN inputs give a NaN code (S.1111.111)
            assert np.all((got[nan] & 0x7F) == 0x7F)
            got, ref = got[~nan], ref[~nan]
        bad = np.count_nonzero(got != ref)
        assert bad == 0, f"chunk {c}: {bad} codes differ"
