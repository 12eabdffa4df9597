"""CPU checker (the oracle) for the FP8 quantized attention path.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm may import this package; the product
package never does.  It shares no code with the CUDA library.

The arithmetic lives in ``fqa_oracle.c`` (plain C, binary32 in a pinned order
for the quantizer, binary64 for attention); this module only builds it with
gcc, loads it with ctypes and marshals numpy arrays.  Every function states
the passage or reading it follows in the C file.

Parity status (see the tests under tests/test_oracle_*.py for the pins):
  * E4M3 / BF16 codecs: pinned (brute-force nearest-even over the decoded
    code table, torch's float8_e4m3fn / bfloat16 casts where they agree with
    the spec, exhaustive GPU comparison).
  * K mean, block scales, codes: pinned (closed forms on exact inputs, error
    bounds, hand-worked blocks).
  * Tiled attention skeleton: pinned (identity codec == exact softmax
    attention; FP64 brute force; invariants).
  * P rounding rule E4M3(p * 448 * sv_J / sv_max): pinned by hand-worked
    cases and by an independent 40-digit re-evaluation of the whole rule
    (tests/test_oracle_highprec.py); the rule itself is a reading, since the
    pages print no worked example.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fqa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-std=c11", "-Wall", "-Wno-unknown-pragmas"]

_lib = None


def build(force: bool = False) -> str:
    """Compile fqa_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i = ctypes.c_int
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_double]
        L.orc_bf16_round.restype = ctypes.c_uint16
        L.orc_bf16_round.argtypes = [ctypes.c_double]
        L.orc_k_mean.argtypes = [P, i, i, i, i, P]
        L.orc_quantize.argtypes = [P, P, P, i, i, i, i, P, P, P, P, P, P, P, P]
        L.orc_attention_core.argtypes = [P, P, P, P, P, P, ctypes.c_float, i, i,
                                         ctypes.c_double, i, i, P, i, P, P, P]
        L.orc_attention_fp8.argtypes = [P, P, P, P, P, P, P, i, i, i, i, ctypes.c_float, i,
                                        P, i, P, i, P, P, P]
        L.orc_attention_exact.argtypes = [P, P, P, i, i, i, i, ctypes.c_double, P, i, P, i, P]
        L.orc_key_error.argtypes = [P, P, P, P, i, i, i, i, P]
        L.orc_select_keys.argtypes = [P, i, i, i, i, P]
        L.orc_attention_fp8_corrected.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, i, i, i, i,
                                                  ctypes.c_float, i, P, i, P, i, P, P]
        L.orc_attention_fp8_part.argtypes = [P, P, P, P, P, P, P, P, i, i, i, i, ctypes.c_float, P, i, P, i,
                                             P, P, P]
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_e2m1_encode.argtypes = [ctypes.c_double]
        L.orc_quantize_nvfp4_qk.argtypes = [P, P, P, i, i, i, i, P, P, P, P, P, P]
        L.orc_attention_nvfp4.argtypes = [P, P, P, P, P, P, P, P, P, i, i, i, i, ctypes.c_float, P, i, P, i,
                                          P, P, P]
        L.orc_e4m3_encode_f32_array.argtypes = [P, ctypes.c_size_t, P]
        L.orc_bf16_round_array.argtypes = [P, ctypes.c_size_t, P]
        L.orc_num_threads.restype = i
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().orc_num_threads()


# ------------------------------------------------------------------ codecs

def e4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib().orc_e4m3_decode(i) for i in range(256)], dtype=np.float64)
    return table[codes]


def e4m3_encode(x) -> np.ndarray:
    """E4M3 RNE saturating codes of binary32 values (NaN -> 0x7F)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_f32_array(_p(x), x.size, _p(out))
    return out


def e4m3_encode_f64(x: float) -> int:
    return int(lib().orc_e4m3_encode(float(x)))


def bf16_round(x) -> np.ndarray:
    """binary64 -> BF16 bit patterns, one round-to-nearest-even."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    out = np.empty(x.shape, dtype=np.uint16)
    lib().orc_bf16_round_array(_p(x), x.size, _p(out))
    return out


def bf16_to_f32(bits) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------- quantizer

def k_mean(k_bf16: np.ndarray) -> np.ndarray:
    B, H, N, d = k_bf16.shape
    k_bf16 = np.ascontiguousarray(k_bf16, dtype=np.uint16)
    mu = np.empty((B, H, d), dtype=np.float32)
    lib().orc_k_mean(_p(k_bf16), B, H, N, d, _p(mu))
    return mu


def quantize(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> dict:
    """BF16 bit arrays [B,H,N,d], any N >= 1 -> codes (natural layout) and FP32
    scales [B,H,ceil(N/64)]."""
    B, H, N, d = q.shape
    nb = (N + 63) // 64                    # the last block may be short
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    r = dict(
        q8=np.empty((B, H, N, d), np.uint8), k8=np.empty((B, H, N, d), np.uint8),
        v8=np.empty((B, H, N, d), np.uint8),
        sq=np.empty((B, H, nb), np.float32), sk=np.empty((B, H, nb), np.float32),
        sv=np.empty((B, H, nb), np.float32), sv_max=np.empty((B, H), np.float32),
        k_mean=np.empty((B, H, d), np.float32))
    lib().orc_quantize(_p(q), _p(k), _p(v), B, H, N, d, _p(r["q8"]), _p(r["k8"]), _p(r["v8"]),
                       _p(r["sq"]), _p(r["sk"]), _p(r["sv"]), _p(r["sv_max"]), _p(r["k_mean"]))
    return r


# --------------------------------------------------------------- attention

def _heads_rows(B, H, N, heads, rows):
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    if rows is None:
        rows = range(N)
    ha = np.ascontiguousarray(np.array(heads, dtype=np.int32).reshape(-1, 2))
    ra = np.ascontiguousarray(np.array(list(rows), dtype=np.int32))
    return ha, ra


def attention_fp8(qz: dict, softmax_scale: float, heads=None, rows=None, bc: int = 128,
                  with_ambiguity: bool = False):
    """Quantized-math attention on quantize() outputs -> [n_heads, n_rows, d] binary64.

    with_ambiguity: also return (amb [n_heads, n_rows, d], namb [n_heads, n_rows]):
    the output range spanned by P codes that a binary32 evaluation may round
    to the other neighbour of an E4M3 midpoint, and how many such codes."""
    B, H, N, d = qz["q8"].shape
    ha, ra = _heads_rows(B, H, N, heads, rows)
    out = np.empty((len(ha), len(ra), d), dtype=np.float64)
    amb = np.empty_like(out) if with_ambiguity else None
    namb = np.empty((len(ha), len(ra)), dtype=np.int32) if with_ambiguity else None
    lib().orc_attention_fp8(_p(qz["q8"]), _p(qz["k8"]), _p(qz["v8"]), _p(qz["sq"]),
                            _p(qz["sk"]), _p(qz["sv"]), _p(qz["sv_max"]), B, H, N, d,
                            float(np.float32(softmax_scale)), bc, _p(ha), len(ha), _p(ra),
                            len(ra), _p(out), None if amb is None else _p(amb),
                            None if namb is None else _p(namb))
    return (out, amb, namb) if with_ambiguity else out


def attention_core(qc, kc, vc, sq, sk, sv, sv_max, scale, bc=128, quantize_p=True, rows=None,
                   with_ambiguity=False):
    """The tiled core on binary64 operand values for one head ([N,d] each)."""
    qc = np.ascontiguousarray(qc, dtype=np.float64)
    kc = np.ascontiguousarray(kc, dtype=np.float64)
    vc = np.ascontiguousarray(vc, dtype=np.float64)
    N, d = qc.shape
    sq = np.ascontiguousarray(sq, dtype=np.float32)
    sk = np.ascontiguousarray(sk, dtype=np.float32)
    sv = np.ascontiguousarray(sv, dtype=np.float32)
    ra = np.ascontiguousarray(np.array(list(range(N) if rows is None else rows), dtype=np.int32))
    out = np.empty((len(ra), d), dtype=np.float64)
    amb = np.empty_like(out) if with_ambiguity else None
    namb = np.empty(len(ra), dtype=np.int32) if with_ambiguity else None
    lib().orc_attention_core(_p(qc), _p(kc), _p(vc), _p(sq), _p(sk), _p(sv), float(sv_max),
                             N, d, float(scale), bc, int(bool(quantize_p)), _p(ra), len(ra),
                             _p(out), None if amb is None else _p(amb),
                             None if namb is None else _p(namb))
    return (out, amb, namb) if with_ambiguity else out


# ------------------------------------------------------------ NVFP4 Q.K

def e2m1_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib().orc_e2m1_decode(i) for i in range(16)], dtype=np.float64)
    return table[codes & 15]


def e2m1_encode_f64(x: float) -> int:
    return int(lib().orc_e2m1_encode(float(x)))


def quantize_nvfp4(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> dict:
    """The FP8 quantizer's outputs (V codes, scales, k_mean) plus Q and
    smoothed K in NVFP4: q4/k4 [B,H,N,64] packed E2M1 (element 2i in the low
    nibble), sfq/sfk [B,H,N,8] E4M3 group scales, sq1/sk1 [B,H,ceil(N/64)]."""
    r = quantize(q, k, v)
    B, H, N, d = q.shape
    nb = (N + 63) // 64
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    r.update(q4=np.empty((B, H, N, d // 2), np.uint8), k4=np.empty((B, H, N, d // 2), np.uint8),
             sfq=np.empty((B, H, N, d // 16), np.uint8), sfk=np.empty((B, H, N, d // 16), np.uint8),
             sq1=np.empty((B, H, nb), np.float32), sk1=np.empty((B, H, nb), np.float32))
    lib().orc_quantize_nvfp4_qk(_p(q), _p(k), _p(r["k_mean"]), B, H, N, d, _p(r["q4"]), _p(r["k4"]),
                                _p(r["sfq"]), _p(r["sfk"]), _p(r["sq1"]), _p(r["sk1"]))
    return r


def attention_nvfp4(qz: dict, softmax_scale: float, heads=None, rows=None, with_ambiguity: bool = False):
    """NVFP4 Q.K, FP8 P.V attention on quantize_nvfp4() outputs -> [n_heads, n_rows, d]."""
    B, H, N, d = qz["v8"].shape
    ha, ra = _heads_rows(B, H, N, heads, rows)
    out = np.empty((len(ha), len(ra), d), dtype=np.float64)
    amb = np.empty_like(out) if with_ambiguity else None
    namb = np.empty((len(ha), len(ra)), dtype=np.int32) if with_ambiguity else None
    lib().orc_attention_nvfp4(_p(qz["q4"]), _p(qz["k4"]), _p(qz["sfq"]), _p(qz["sfk"]), _p(qz["sq1"]),
                              _p(qz["sk1"]), _p(qz["v8"]), _p(qz["sv"]), _p(qz["sv_max"]), B, H, N, d,
                              float(np.float32(softmax_scale)), _p(ha), len(ha), _p(ra), len(ra), _p(out),
                              None if amb is None else _p(amb), None if namb is None else _p(namb))
    return (out, amb, namb) if with_ambiguity else out


# ------------------------------------------------ error-corrected attention

def key_error(k_bf16: np.ndarray, qz: dict) -> np.ndarray:
    """Per-key quantization error [B,H,N] (binary32, pinned order; see the C file)."""
    B, H, N, d = k_bf16.shape
    k_bf16 = np.ascontiguousarray(k_bf16, dtype=np.uint16)
    err = np.empty((B, H, N), dtype=np.float32)
    lib().orc_key_error(_p(k_bf16), _p(qz["k8"]), _p(qz["sk"]), _p(qz["k_mean"]), B, H, N, d, _p(err))
    return err


def n_corrected(N: int, rho: float) -> int:
    """Keys corrected per head [reading]: ceil(fl32(rho) * N - 0.01), clamped to
    [0, N] -- rho in binary32 as the C ABI takes it; the 0.01 keeps a product
    meant to be an integer (0.05 of 1280 keys) that integer."""
    import math
    return max(0, min(N, math.ceil(float(np.float32(rho)) * N - 0.01)))


def select_keys(err: np.ndarray, kc: int) -> np.ndarray:
    """[B,H,N] 0/1: the kc keys of each head with the largest error (ties to the
    lower index)."""
    B, H, N = err.shape
    err = np.ascontiguousarray(err, dtype=np.float32)
    sel = np.empty((B, H, N), dtype=np.uint8)
    lib().orc_select_keys(_p(err), B, H, N, int(kc), _p(sel))
    return sel


def attention_fp8_part(qz: dict, sel: np.ndarray, softmax_scale: float, heads=None, rows=None):
    """The FP8 rule over the keys with sel = 0 -> (out [n_heads, n_rows, d],
    m [n_heads, n_rows], l [n_heads, n_rows]) in binary64."""
    B, H, N, d = qz["q8"].shape
    ha, ra = _heads_rows(B, H, N, heads, rows)
    out = np.empty((len(ha), len(ra), d), dtype=np.float64)
    m = np.empty((len(ha), len(ra)), dtype=np.float64)
    l = np.empty_like(m)
    sel = np.ascontiguousarray(sel, dtype=np.uint8)
    lib().orc_attention_fp8_part(_p(qz["q8"]), _p(qz["k8"]), _p(qz["v8"]), _p(qz["sq"]), _p(qz["sk"]),
                                 _p(qz["sv"]), _p(qz["sv_max"]), _p(sel), B, H, N, d,
                                 float(np.float32(softmax_scale)), _p(ha), len(ha), _p(ra), len(ra), _p(out),
                                 _p(m), _p(l))
    return out, m, l


def attention_fp8_corrected(g: dict, qz: dict, sel: np.ndarray, softmax_scale: float, heads=None,
                            rows=None, quantize_p: bool = True, with_ambiguity: bool = False):
    """Error-corrected FP8 attention -> [n_heads, n_rows, d] binary64 (and the
    ambiguity bound of its FP8 part when with_ambiguity)."""
    B, H, N, d = qz["q8"].shape
    ha, ra = _heads_rows(B, H, N, heads, rows)
    out = np.empty((len(ha), len(ra), d), dtype=np.float64)
    amb = np.empty_like(out) if with_ambiguity else None
    q, k, v = (np.ascontiguousarray(g[t], dtype=np.uint16) for t in "qkv")
    sel = np.ascontiguousarray(sel, dtype=np.uint8)
    lib().orc_attention_fp8_corrected(
        _p(q), _p(k), _p(v), _p(qz["q8"]), _p(qz["k8"]), _p(qz["v8"]), _p(qz["sq"]), _p(qz["sk"]),
        _p(qz["sv"]), _p(qz["sv_max"]), _p(qz["k_mean"]), _p(sel), B, H, N, d,
        float(np.float32(softmax_scale)), int(bool(quantize_p)), _p(ha), len(ha), _p(ra), len(ra),
        _p(out), None if amb is None else _p(amb))
    return (out, amb) if with_ambiguity else out


def attention_exact(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                    heads=None, rows=None) -> np.ndarray:
    """softmax(Q K^T * scale) V in binary64 on BF16 inputs -> [n_heads, n_rows, d]."""
    B, H, N, d = q.shape
    assert d <= 512
    ha, ra = _heads_rows(B, H, N, heads, rows)
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    out = np.empty((len(ha), len(ra), d), dtype=np.float64)
    lib().orc_attention_exact(_p(q), _p(k), _p(v), B, H, N, d, float(scale), _p(ha), len(ha),
                              _p(ra), len(ra), _p(out))
    return out


def softmax_scale(d: int = 128) -> float:
    """fl32(1/sqrt(d)), the FP32 softmax scale the workloads use."""
    return float(np.float32(1.0) / np.sqrt(np.float32(d)))
