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


def test_kernel_exp2_within_the_parity_bound():
    """The exponential of every attention kernel (p = 2^(x - m), the rescale
    factors) against binary64 exp2 at every binary32 x in [-30, 0] -- the
    range where a P code can be nonzero (p * 448 >= 2^-10 needs x - m >= -19)
    and where a term can move the row sum by more than 2^-30 of its largest
    term.  The oracle's ambiguity bound assumes a relative error of at most
    2^-21 for this step; this measures it."""
    import quantized_fp8_attention_b200 as fqa
    err = fqa.exp2_max_rel_error(-30.0, 0.0)
    print(f"\nmax relative error of the kernels' exp2 on [-30, 0]: {err:.3e} (2^{np.log2(err):.2f})")
    assert 0.0 < err <= 2.0 ** -21
    assert fqa.fqa_debug_status()[0] == fqa.FQA_OK
