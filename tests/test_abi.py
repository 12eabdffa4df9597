"""The C ABI without a GPU: the library loads, exports every function that
include/fqa.h declares, and rejects bad arguments on the host before any CUDA
call (only argument sets that fail validation are used here)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from quantized_fp8_attention_b200 import build
    build.build()
    import quantized_fp8_attention_b200 as fqa
    return fqa.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "fqa.h")).read()
    return sorted(set(re.findall(r"FQA_API\s+[\w\s\*]+?\b(fqa_\w+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("fqa_quantize", "fqa_attention_fp8", "fqa_attention_bf16", "fqa_quantize_workspace_bytes",
              "fqa_status_string", "fqa_debug_status"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared_functions():
        assert hasattr(L, n), n


def test_status_strings_and_version(L):
    import quantized_fp8_attention_b200 as fqa
    assert fqa.version() >> 16 == 1
    assert [fqa.status_string(i) for i in range(6)] == [
        "FQA_OK", "FQA_ERR_INVALID_ARG", "FQA_ERR_UNSUPPORTED", "FQA_ERR_MISALIGNED", "FQA_ERR_CUDA",
        "FQA_ERR_TIMEOUT"]


def test_workspace_bytes(L):
    import quantized_fp8_attention_b200 as fqa
    r256 = lambda x: (x + 255) // 256 * 256
    ws = lambda B, H, N: r256(B * H * ((N + 63) // 64) * 128 * 4) + 256
    assert fqa.fqa_quantize_workspace_bytes(1, 24, 8704) == ws(1, 24, 8704) == 1671168 + 256
    assert fqa.fqa_quantize_workspace_bytes(2, 24, 16896) == ws(2, 24, 16896)
    assert fqa.fqa_quantize_workspace_bytes(1, 65535, 64) == ws(1, 65535, 64)
    assert fqa.fqa_quantize_workspace_bytes(1, 1, 100) == ws(1, 1, 100) == 1024 + 256   # short last block
    assert fqa.fqa_quantize_workspace_bytes(1, 1, 1) == 512 + 256
    assert fqa.fqa_quantize_workspace_bytes(1, 1, 0) == 0
    assert fqa.fqa_quantize_workspace_bytes(1, 1, 65537) == 0     # N > 65536
    assert fqa.fqa_quantize_workspace_bytes(1, 1, 128, 64) == 0   # d != 128


P = ctypes.c_void_p


def _p(addr):
    return P(addr)


def test_quantize_validation(L):
    ok = _p(0x10000)
    args = lambda **kw: [kw.get(n, ok) for n in ("q", "k", "v")] + [
        kw.get("B", 1), kw.get("H", 1), kw.get("N", 128), kw.get("d", 128)] + [
        kw.get(n, ok) for n in ("q8", "k8", "v8", "sq", "sk", "sv", "svm", "km", "ws")] + [
        kw.get("wsb", 1 << 20), None]
    assert L.fqa_quantize(*args(q=None)) == 1
    assert L.fqa_quantize(*args(ws=None)) == 1
    assert L.fqa_quantize(*args(B=0)) == 1
    assert L.fqa_quantize(*args(d=64)) == 2
    assert L.fqa_quantize(*args(N=0)) == 1
    assert L.fqa_quantize(*args(N=65600)) == 2
    assert L.fqa_quantize(*args(B=300, H=300)) == 2
    assert L.fqa_quantize(*args(wsb=16)) == 1
    assert L.fqa_quantize(*args(k=_p(0x10008))) == 3
    assert L.fqa_quantize(*args(sq=_p(0x10002))) == 3
    assert L.fqa_quantize(*args(km=_p(0x10004))) == 3      # k_mean: 16-byte aligned


def test_attention_validation(L):
    ok = _p(0x10000)
    f = ctypes.c_float

    def fp8(**kw):
        return L.fqa_attention_fp8(*[kw.get(n, ok) for n in ("q8", "k8", "v8", "sq", "sk", "sv", "svm")],
                                   kw.get("B", 1), kw.get("H", 1), kw.get("N", 128), kw.get("d", 128),
                                   f(kw.get("scale", 0.088)), kw.get("out", ok), kw.get("dt", 0), None)

    assert fp8(q8=None) == 1
    assert fp8(out=None) == 1
    assert fp8(scale=0.0) == 1
    assert fp8(scale=float("inf")) == 1
    assert fp8(dt=5) == 1
    assert fp8(N=65537) == 2
    assert fp8(N=0) == 1
    assert fp8(d=256) == 2
    assert fp8(v8=_p(0x10001)) == 3
    assert fp8(out=_p(0x10004)) == 3
    bf = lambda **kw: L.fqa_attention_bf16(kw.get("q", ok), ok, ok, 1, 1, kw.get("N", 128), 128,
                                           f(kw.get("scale", 0.088)), kw.get("out", ok), 0, None)
    assert bf(q=None) == 1
    assert bf(N=70000) == 2
    assert bf(scale=-1.0) == 1
    assert bf(q=_p(0x10002)) == 3
    assert L.fqa_e4m3_encode(None, ok, 4, None) == 1
    L.fqa_debug_wait_timeout.argtypes = [ctypes.c_uint32, P]
    assert L.fqa_debug_wait_timeout(0, None) == 1
    assert L.fqa_debug_wait_timeout(3000000, None) == 1


def test_corrected_key_count_matches_the_oracle(L):
    """The count of corrected keys per head is a host computation on the
    binary32 rho the ABI takes; it must agree with the oracle's reading."""
    import oracle
    import quantized_fp8_attention_b200 as fqa
    for N in (1, 7, 100, 200, 1000, 1280, 4429, 4608, 8704, 16896, 65536):
        for rho in (0.0, 0.001, 0.005, 0.01, 0.02, 0.05, 0.1, 0.25, 0.5, 1.0):
            assert fqa.fqa_corrected_keys(N, rho) == oracle.n_corrected(N, rho), (N, rho)
    assert fqa.fqa_corrected_keys(0, 0.1) == -1
    assert fqa.fqa_corrected_keys(100, 1.5) == -1
    assert fqa.fqa_corrected_keys(100, float("nan")) == -1
    assert fqa.fqa_attention_fp8_corrected_workspace_bytes(1, 24, 8704, 0.005) > 24 * 8704 * 512
    assert fqa.fqa_attention_fp8_corrected_workspace_bytes(1, 24, 8704, 2.0) == 0


def test_nvfp4_validation(L):
    ok = _p(0x10000)
    f = ctypes.c_float

    def quant(**kw):
        return L.fqa_quantize_nvfp4_qk(kw.get("q", ok), kw.get("k", ok), kw.get("km", ok), kw.get("B", 1),
                                       kw.get("H", 1), kw.get("N", 128), kw.get("d", 128),
                                       *[kw.get(n, ok) for n in ("q4", "k4", "sfq", "sfk", "sq1", "sk1")], None)

    def attn(**kw):
        return L.fqa_attention_nvfp4(*[kw.get(n, ok) for n in ("q4", "k4", "sfq", "sfk", "sq1", "sk1", "v8",
                                                                "sv", "svm")],
                                     kw.get("B", 1), kw.get("H", 1), kw.get("N", 128), kw.get("d", 128),
                                     f(kw.get("scale", 0.088)), kw.get("out", ok), kw.get("dt", 0), None)

    assert quant(q=None) == 1
    assert quant(sk1=None) == 1
    assert quant(N=0) == 1
    assert quant(d=64) == 2
    assert quant(N=65537) == 2
    assert quant(k=_p(0x10008)) == 3            # BF16 inputs: 16-byte aligned
    assert quant(q4=_p(0x10002)) == 3           # packed codes: 4-byte aligned
    assert attn(q4=None) == 1
    assert attn(out=None) == 1
    assert attn(scale=0.0) == 1
    assert attn(dt=3) == 1
    assert attn(N=65537) == 2
    assert attn(d=64) == 2
    assert attn(k4=_p(0x10008)) == 3
    assert attn(sfq=_p(0x10004)) == 3           # group scales: 8-byte aligned
    assert attn(sv=_p(0x10002)) == 3
    assert L.fqa_e2m1_encode(None, ok, 4, None) == 1
    assert L.fqa_e2m1_encode(_p(0x10004), ok, 4, None) == 3


def test_exp2_error_validation(L):
    ok = _p(0x10000)
    f = ctypes.c_float
    L.fqa_exp2_error.argtypes = [f, f, P, P]
    assert L.fqa_exp2_error(f(-30.0), f(0.0), None, None) == 1
    assert L.fqa_exp2_error(f(0.0), f(-30.0), ok, None) == 1        # lo > hi
    assert L.fqa_exp2_error(f(-30.0), f(1.0), ok, None) == 1        # hi > 0
    assert L.fqa_exp2_error(f(-200.0), f(0.0), ok, None) == 1       # lo < -126
    assert L.fqa_exp2_error(f(-30.0), f(0.0), _p(0x10002), None) == 3
