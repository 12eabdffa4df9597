"""Python binding of libfqa.so, the B200 FP8 quantized attention library.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  The C ABI
is declared (and documented) in include/fqa.h; the functions below carry the
same names and pass ``tensor.data_ptr()`` and the stream handle through.

The library must have been built (``python -m quantized_fp8_attention_b200.build``
or ``__graft_entry__.build()``); every call raises ImportError without it.
"""

from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfqa.so")

FQA_OK, FQA_ERR_INVALID_ARG, FQA_ERR_UNSUPPORTED, FQA_ERR_MISALIGNED, FQA_ERR_CUDA, FQA_ERR_TIMEOUT = range(6)
FQA_OUT_BF16, FQA_OUT_F32 = 0, 1
HEAD_DIM = 128

_lib = None


def _load():
    """Load libfqa.so and declare the C signatures.  Raises if it is not built:
    there is no fallback implementation."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libfqa.so is not built ({LIB_PATH}); run `python -m quantized_fp8_attention_b200.build`. "
            "There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    P, I = ctypes.c_void_p, ctypes.c_int
    L.fqa_version.restype = I
    L.fqa_status_string.restype = ctypes.c_char_p
    L.fqa_status_string.argtypes = [I]
    L.fqa_quantize_workspace_bytes.restype = ctypes.c_size_t
    L.fqa_quantize_workspace_bytes.argtypes = [I, I, I, I]
    L.fqa_quantize.restype = I
    L.fqa_quantize.argtypes = [P, P, P, I, I, I, I, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.fqa_attention_fp8.restype = I
    L.fqa_attention_fp8.argtypes = [P, P, P, P, P, P, P, I, I, I, I, ctypes.c_float, P, I, P]
    L.fqa_attention_bf16.restype = I
    L.fqa_attention_bf16.argtypes = [P, P, P, I, I, I, I, ctypes.c_float, P, I, P]
    L.fqa_e4m3_encode.restype = I
    L.fqa_e4m3_encode.argtypes = [P, P, ctypes.c_size_t, P]
    L.fqa_debug_status.restype = I
    L.fqa_debug_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    L.fqa_quantize_a2a.restype = I
    L.fqa_quantize_a2a.argtypes = [P, P, P, I, I, I, I, I, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.fqa_attention_fp8_a2a.restype = I
    L.fqa_attention_fp8_a2a.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, ctypes.c_float, P, I, P]
    L.fqa_quantize_keyerr.restype = I
    L.fqa_quantize_keyerr.argtypes = [P, P, P, I, I, I, I, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    L.fqa_corrected_keys.restype = I
    L.fqa_corrected_keys.argtypes = [I, ctypes.c_float]
    L.fqa_select_keys.restype = I
    L.fqa_select_keys.argtypes = [P, I, I, I, I, P, P, P]
    L.fqa_attention_fp8_corrected_workspace_bytes.restype = ctypes.c_size_t
    L.fqa_attention_fp8_corrected_workspace_bytes.argtypes = [I, I, I, I, ctypes.c_float]
    L.fqa_attention_fp8_corrected.restype = I
    L.fqa_attention_fp8_corrected.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, ctypes.c_float,
                                              ctypes.c_float, P, I, P, ctypes.c_size_t, P]
    L.fqa_quantize_nvfp4_qk.restype = I
    L.fqa_quantize_nvfp4_qk.argtypes = [P, P, P, I, I, I, I, P, P, P, P, P, P, P]
    L.fqa_attention_nvfp4.restype = I
    L.fqa_attention_nvfp4.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, ctypes.c_float, P, I, P]
    L.fqa_e2m1_encode.restype = I
    L.fqa_e2m1_encode.argtypes = [P, P, ctypes.c_size_t, P]
    L.fqa_exp2_error.restype = I
    L.fqa_exp2_error.argtypes = [ctypes.c_float, ctypes.c_float, P, P]
    _lib = L
    return L


class FqaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib():
    """The loaded ctypes library (for tests that call the ABI directly)."""
    return _load()


def status_string(status: int) -> str:
    return _load().fqa_status_string(int(status)).decode()


def version() -> int:
    return _load().fqa_version()


def _check(status: int, where: str):
    if status != FQA_OK:
        raise FqaError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------- raw ABI

def fqa_quantize_workspace_bytes(B: int, H: int, N: int, d: int = HEAD_DIM) -> int:
    return int(_load().fqa_quantize_workspace_bytes(B, H, N, d))


def fqa_quantize(q, k, v, q8, k8, v8, sq, sk, sv, sv_max, k_mean, workspace, stream=None) -> int:
    """The C call with tensors; returns the fqa_status code."""
    B, H, N, d = q.shape
    return _load().fqa_quantize(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(q8), _ptr(k8), _ptr(v8),
                             _ptr(sq), _ptr(sk), _ptr(sv), _ptr(sv_max), _ptr(k_mean),
                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream))


def fqa_quantize_noalloc(q, k, v, q8, k8, v8, sq, sk, sv, sv_max, k_mean, stream=None) -> int:
    """fqa_quantize without a workspace (for callers that cannot allocate
    device memory when they call): the library keeps the scratch in a fixed
    8 MiB array per GPU.  Returns the fqa_status code."""
    L = _load()
    f = L.fqa_quantize_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.restype = I
    f.argtypes = [P, P, P, I, I, I, I, P, P, P, P, P, P, P, P, P]
    B, H, N, d = q.shape
    return f(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq),
             _ptr(sk), _ptr(sv), _ptr(sv_max), _ptr(k_mean), _stream(stream))


def fqa_attention_fp8(q8, k8, v8, sq, sk, sv, sv_max, softmax_scale, out, out_dtype, stream=None) -> int:
    B, H, N, d = q8.shape
    return _load().fqa_attention_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv),
                                  _ptr(sv_max), B, H, N, d, float(softmax_scale), _ptr(out),
                                  int(out_dtype), _stream(stream))


def fqa_attention_bf16(q, k, v, softmax_scale, out, out_dtype, stream=None) -> int:
    B, H, N, d = q.shape
    return _load().fqa_attention_bf16(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, float(softmax_scale),
                                   _ptr(out), int(out_dtype), _stream(stream))


def fqa_quantize_a2a(q, k, v, q8, k8, v8, sq, sk, sv, sv_max, k_mean, workspace, stream=None) -> int:
    """fqa_quantize on inputs in the sequence all-to-all layout [B, P, Hl, Nl, d]."""
    B, P, Hl, Nl, d = q.shape
    return _load().fqa_quantize_a2a(_ptr(q), _ptr(k), _ptr(v), B, Hl, P, Nl, d, _ptr(q8), _ptr(k8), _ptr(v8),
                                 _ptr(sq), _ptr(sk), _ptr(sv), _ptr(sv_max), _ptr(k_mean), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))


def fqa_attention_fp8_a2a(q8, k8, v8, sq, sk, sv, sv_max, P: int, softmax_scale, out, out_dtype,
                          stream=None) -> int:
    """fqa_attention_fp8 writing out in the layout [B, P, Hl, N / P, d]."""
    B, Hl, N, d = q8.shape
    return _load().fqa_attention_fp8_a2a(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv),
                                      _ptr(sv_max), B, Hl, int(P), N // int(P), d, float(softmax_scale),
                                      _ptr(out), int(out_dtype), _stream(stream))


def fqa_quantize_keyerr(q, k, v, q8, k8, v8, sq, sk, sv, sv_max, k_mean, k_err, workspace,
                        stream=None) -> int:
    """fqa_quantize plus each key's quantization error k_err [B,H,N] FP32."""
    B, H, N, d = q.shape
    return _load().fqa_quantize_keyerr(_ptr(q), _ptr(k), _ptr(v), B, H, N, d, _ptr(q8), _ptr(k8), _ptr(v8),
                                    _ptr(sq), _ptr(sk), _ptr(sv), _ptr(sv_max), _ptr(k_mean), _ptr(k_err),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream))


def fqa_corrected_keys(N: int, rho: float) -> int:
    return int(_load().fqa_corrected_keys(int(N), float(rho)))


def fqa_select_keys(k_err, kc: int, kmask, idx, stream=None) -> int:
    B, H, N = k_err.shape
    return _load().fqa_select_keys(_ptr(k_err), B, H, N, int(kc), _ptr(kmask), _ptr(idx), _stream(stream))


def fqa_attention_fp8_corrected_workspace_bytes(B: int, H: int, N: int, rho: float, d: int = HEAD_DIM) -> int:
    return int(_load().fqa_attention_fp8_corrected_workspace_bytes(B, H, N, d, float(rho)))


def fqa_attention_fp8_corrected(q, k, v, q8, k8, v8, sq, sk, sv, sv_max, k_mean, k_err, softmax_scale, rho,
                                out, out_dtype, workspace, stream=None) -> int:
    B, H, N, d = q.shape
    return _load().fqa_attention_fp8_corrected(
        _ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk), _ptr(sv), _ptr(sv_max),
        _ptr(k_mean), _ptr(k_err), B, H, N, d, float(softmax_scale), float(rho), _ptr(out), int(out_dtype),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))


def fqa_e4m3_encode(x, out, stream=None) -> int:
    return _load().fqa_e4m3_encode(_ptr(x), _ptr(out), x.numel(), _stream(stream))


def fqa_quantize_nvfp4_qk(q, k, k_mean, q4, k4, sfq, sfk, sq1, sk1, stream=None) -> int:
    B, H, N, d = q.shape
    return _load().fqa_quantize_nvfp4_qk(_ptr(q), _ptr(k), _ptr(k_mean), B, H, N, d, _ptr(q4), _ptr(k4),
                                         _ptr(sfq), _ptr(sfk), _ptr(sq1), _ptr(sk1), _stream(stream))


def fqa_attention_nvfp4(q4, k4, sfq, sfk, sq1, sk1, v8, sv, sv_max, softmax_scale, out, out_dtype,
                        stream=None) -> int:
    B, H, N, d = v8.shape
    return _load().fqa_attention_nvfp4(_ptr(q4), _ptr(k4), _ptr(sfq), _ptr(sfk), _ptr(sq1), _ptr(sk1), _ptr(v8),
                                       _ptr(sv), _ptr(sv_max), B, H, N, d, float(softmax_scale), _ptr(out),
                                       int(out_dtype), _stream(stream))


def fqa_e2m1_encode(x, out, stream=None) -> int:
    return _load().fqa_e2m1_encode(_ptr(x), _ptr(out), x.numel() // 2, _stream(stream))


def fqa_exp2_error(lo: float, hi: float, max_rel_bits, stream=None) -> int:
    return _load().fqa_exp2_error(float(lo), float(hi), _ptr(max_rel_bits), _stream(stream))


def exp2_max_rel_error(lo: float, hi: float, device="cuda") -> float:
    """Largest relative error of the kernels' exp2 over every binary32 in [lo, hi]."""
    bits = torch.zeros(1, dtype=torch.int32, device=device)
    _check(fqa_exp2_error(lo, hi, bits), "fqa_exp2_error")
    return float(bits.cpu().view(torch.float32)[0])


def fqa_debug_wait_timeout(limit_us: int, stream=None) -> int:
    """Launch a bounded wait that is bound to give up after limit_us (tests the
    timeout path; the next fqa_debug_status() reports FQA_ERR_TIMEOUT)."""
    L = _load()
    L.fqa_debug_wait_timeout.restype = ctypes.c_int
    L.fqa_debug_wait_timeout.argtypes = [ctypes.c_uint32, ctypes.c_void_p]
    return L.fqa_debug_wait_timeout(int(limit_us), _stream(stream))


def fqa_debug_status(stream=None):
    """(status, raw flag bits) of the current device's status word; clears it."""
    flags = ctypes.c_uint32(0)
    st = _load().fqa_debug_status(_stream(stream), ctypes.byref(flags))
    return st, flags.value


# ----------------------------------------------------- tensor-level API

def _require(t, dtype: torch.dtype, name: str, shape=None) -> None:
    """The C ABI takes contiguous device buffers of a fixed element type and
    shape; anything else is refused here, before a pointer is passed on."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device.type != "cuda":
        raise ValueError(f"{name}: expected a CUDA tensor, got one on {t.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _require_qkv(q, k, v, dtype: torch.dtype):
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q: expected a [B, H, N, 128] tensor")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require(t, dtype, name, q.shape)
    if q.device != k.device or q.device != v.device:
        raise ValueError("q, k and v must be on the same device")
    return tuple(q.shape)


def nblocks(N: int) -> int:
    """64-token blocks per head: ceil(N / 64) (the last one may be short)."""
    return (N + 63) // 64


def _require_quantized(qz: "Quantized", B: int, H: int, N: int) -> None:
    nb = nblocks(N)
    shapes = ((B, H, N, HEAD_DIM),) * 3 + ((B, H, nb),) * 3 + ((B, H), (B, H, HEAD_DIM))
    for name, t, shape in zip(Quantized._fields, qz, shapes):
        _require(t, torch.uint8 if name.endswith("8") else torch.float32, name, shape)


class Quantized(NamedTuple):
    q8: torch.Tensor       # uint8 E4M3 codes [B,H,N,128]
    k8: torch.Tensor
    v8: torch.Tensor
    sq: torch.Tensor       # float32 [B,H,ceil(N/64)]
    sk: torch.Tensor
    sv: torch.Tensor
    sv_max: torch.Tensor   # float32 [B,H]
    k_mean: torch.Tensor   # float32 [B,H,128]


def alloc_quantized(B: int, H: int, N: int, device) -> Quantized:
    u8 = dict(dtype=torch.uint8, device=device)
    f32 = dict(dtype=torch.float32, device=device)
    nb = nblocks(N)
    return Quantized(torch.empty(B, H, N, HEAD_DIM, **u8), torch.empty(B, H, N, HEAD_DIM, **u8),
                     torch.empty(B, H, N, HEAD_DIM, **u8), torch.empty(B, H, nb, **f32),
                     torch.empty(B, H, nb, **f32), torch.empty(B, H, nb, **f32),
                     torch.empty(B, H, **f32), torch.empty(B, H, HEAD_DIM, **f32))


def alloc_workspace(B: int, H: int, N: int, device) -> torch.Tensor:
    nbytes = fqa_quantize_workspace_bytes(B, H, N)
    return torch.empty(max(nbytes, 16) // 4, dtype=torch.float32, device=device)


def quantize(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[Quantized] = None,
             workspace: Optional[torch.Tensor] = None, stream=None) -> Quantized:
    """BF16 [B,H,N,128] Q, K, V (CUDA, contiguous) -> Quantized."""
    B, H, N, _ = _require_qkv(q, k, v, torch.bfloat16)
    if out is None:
        out = alloc_quantized(B, H, N, q.device)
    _require_quantized(out, B, H, N)
    if workspace is None:
        workspace = alloc_workspace(B, H, N, q.device)
    _require(workspace, workspace.dtype, "workspace")
    _check(fqa_quantize(q, k, v, *out, workspace, stream=stream), "fqa_quantize")
    return out


def attention_fp8(qz: Quantized, softmax_scale: float, out_dtype: int = FQA_OUT_BF16,
                  out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    if not isinstance(qz.q8, torch.Tensor) or qz.q8.dim() != 4:
        raise ValueError("qz.q8: expected a [B, H, N, 128] tensor")
    B, H, N, d = qz.q8.shape
    _require_quantized(qz, B, H, N)
    dt = torch.float32 if out_dtype == FQA_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(B, H, N, d, dtype=dt, device=qz.q8.device)
    _require(out, dt, "out", (B, H, N, d))
    _check(fqa_attention_fp8(qz.q8, qz.k8, qz.v8, qz.sq, qz.sk, qz.sv, qz.sv_max, softmax_scale,
                             out, out_dtype, stream=stream), "fqa_attention_fp8")
    return out


def attention_bf16(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, softmax_scale: float,
                   out_dtype: int = FQA_OUT_BF16, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    B, H, N, d = _require_qkv(q, k, v, torch.bfloat16)
    dt = torch.float32 if out_dtype == FQA_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(B, H, N, d, dtype=dt, device=q.device)
    _require(out, dt, "out", (B, H, N, d))
    _check(fqa_attention_bf16(q, k, v, softmax_scale, out, out_dtype, stream=stream),
           "fqa_attention_bf16")
    return out


def quantize_keyerr(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[Quantized] = None,
                    k_err: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream=None):
    """quantize() plus the per-key quantization error: (Quantized, k_err [B,H,N] float32)."""
    B, H, N, _ = _require_qkv(q, k, v, torch.bfloat16)
    if out is None:
        out = alloc_quantized(B, H, N, q.device)
    _require_quantized(out, B, H, N)
    if k_err is None:
        k_err = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    _require(k_err, torch.float32, "k_err", (B, H, N))
    if workspace is None:
        workspace = alloc_workspace(B, H, N, q.device)
    _require(workspace, workspace.dtype, "workspace")
    _check(fqa_quantize_keyerr(q, k, v, *out, k_err, workspace, stream=stream), "fqa_quantize_keyerr")
    return out, k_err


def quantize_a2a(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: Optional[Quantized] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> Quantized:
    """Q, K, V in the sequence all-to-all layout [B, P, Hl, Nl, 128] (BF16,
    CUDA, contiguous; Nl a multiple of 64) -> Quantized for B, Hl heads and
    N = P * Nl tokens in the usual layouts."""
    if not isinstance(q, torch.Tensor) or q.dim() != 5:
        raise ValueError("q: expected a [B, P, Hl, Nl, 128] tensor")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require(t, torch.bfloat16, name, q.shape)
    B, P, Hl, Nl, _ = q.shape
    N = P * Nl
    if out is None:
        out = alloc_quantized(B, Hl, N, q.device)
    _require_quantized(out, B, Hl, N)
    if workspace is None:
        workspace = alloc_workspace(B, Hl, N, q.device)
    _require(workspace, workspace.dtype, "workspace")
    _check(fqa_quantize_a2a(q, k, v, *out, workspace, stream=stream), "fqa_quantize_a2a")
    return out


def attention_fp8_a2a(qz: Quantized, P: int, softmax_scale: float, out_dtype: int = FQA_OUT_BF16,
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """fqa_attention_fp8 with the output in the layout [B, P, Hl, N / P, 128]."""
    B, Hl, N, d = qz.q8.shape
    _require_quantized(qz, B, Hl, N)
    if N % P:
        raise ValueError(f"N = {N} is not a multiple of P = {P}")
    dt = torch.float32 if out_dtype == FQA_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(B, P, Hl, N // P, d, dtype=dt, device=qz.q8.device)
    _require(out, dt, "out", (B, P, Hl, N // P, d))
    _check(fqa_attention_fp8_a2a(*qz[:7], P, softmax_scale, out, out_dtype, stream=stream),
           "fqa_attention_fp8_a2a")
    return out


def alloc_corrected_workspace(B: int, H: int, N: int, rho: float, device) -> torch.Tensor:
    nbytes = fqa_attention_fp8_corrected_workspace_bytes(B, H, N, rho)
    if nbytes == 0:
        raise ValueError("invalid sizes or rho for the corrected path")
    return torch.empty((nbytes + 15) // 16 * 4, dtype=torch.float32, device=device)


def attention_fp8_corrected(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, qz: Quantized,
                            k_err: torch.Tensor, softmax_scale: float, rho: float = 0.005,
                            out_dtype: int = FQA_OUT_BF16, out: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Error-corrected FP8 attention: the ceil(rho * N) keys per head with the
    largest quantization error are handled exactly, the rest by the FP8 rule."""
    B, H, N, d = _require_qkv(q, k, v, torch.bfloat16)
    _require_quantized(qz, B, H, N)
    _require(k_err, torch.float32, "k_err", (B, H, N))
    dt = torch.float32 if out_dtype == FQA_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(B, H, N, d, dtype=dt, device=q.device)
    _require(out, dt, "out", (B, H, N, d))
    if workspace is None:
        workspace = alloc_corrected_workspace(B, H, N, rho, q.device)
    _require(workspace, workspace.dtype, "workspace")
    _check(fqa_attention_fp8_corrected(q, k, v, *qz[:7], qz.k_mean, k_err, softmax_scale, rho, out, out_dtype,
                                       workspace, stream=stream), "fqa_attention_fp8_corrected")
    return out


def fp8_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, softmax_scale: float,
                  out_dtype: int = FQA_OUT_BF16, stream=None) -> torch.Tensor:
    """The whole FP8 path: quantize, then fused FP8 attention."""
    return attention_fp8(quantize(q, k, v, stream=stream), softmax_scale, out_dtype, stream=stream)


def e4m3_encode(x: torch.Tensor, stream=None) -> torch.Tensor:
    _require(x, torch.float32, "x")
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(fqa_e4m3_encode(x, out, stream=stream), "fqa_e4m3_encode")
    return out


# ------------------------------------------------ NVFP4 Q.K variant

class QuantizedNvfp4(NamedTuple):
    q4: torch.Tensor       # uint8 [B,H,N,64]: E2M1 codes, element 2i in the low nibble
    k4: torch.Tensor       # of K - k_mean
    sfq: torch.Tensor      # uint8 [B,H,N,8]: E4M3 scale per 16 channels
    sfk: torch.Tensor
    sq1: torch.Tensor      # float32 [B,H,ceil(N/64)]
    sk1: torch.Tensor


def alloc_quantized_nvfp4(B: int, H: int, N: int, device) -> QuantizedNvfp4:
    u8 = dict(dtype=torch.uint8, device=device)
    f32 = dict(dtype=torch.float32, device=device)
    nb = nblocks(N)
    return QuantizedNvfp4(torch.empty(B, H, N, HEAD_DIM // 2, **u8), torch.empty(B, H, N, HEAD_DIM // 2, **u8),
                          torch.empty(B, H, N, HEAD_DIM // 16, **u8), torch.empty(B, H, N, HEAD_DIM // 16, **u8),
                          torch.empty(B, H, nb, **f32), torch.empty(B, H, nb, **f32))


def _require_nvfp4(qn: QuantizedNvfp4, B: int, H: int, N: int) -> None:
    nb = nblocks(N)
    shapes = ((B, H, N, HEAD_DIM // 2),) * 2 + ((B, H, N, HEAD_DIM // 16),) * 2 + ((B, H, nb),) * 2
    for name, t, shape in zip(QuantizedNvfp4._fields, qn, shapes):
        _require(t, torch.float32 if name.endswith("1") else torch.uint8, name, shape)


def quantize_nvfp4_qk(q: torch.Tensor, k: torch.Tensor, k_mean: torch.Tensor,
                      out: Optional[QuantizedNvfp4] = None, stream=None) -> QuantizedNvfp4:
    """BF16 Q, K [B,H,N,128] and the K channel means of quantize() -> NVFP4 Q and
    smoothed K."""
    B, H, N, _ = _require_qkv(q, k, k, torch.bfloat16)
    _require(k_mean, torch.float32, "k_mean", (B, H, HEAD_DIM))
    if out is None:
        out = alloc_quantized_nvfp4(B, H, N, q.device)
    _require_nvfp4(out, B, H, N)
    _check(fqa_quantize_nvfp4_qk(q, k, k_mean, *out, stream=stream), "fqa_quantize_nvfp4_qk")
    return out


def attention_nvfp4(qn: QuantizedNvfp4, qz: Quantized, softmax_scale: float, out_dtype: int = FQA_OUT_BF16,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """NVFP4 Q.K^T, FP8 P.V: qn from quantize_nvfp4_qk(), V (v8, sv, sv_max) from qz."""
    if not isinstance(qz.v8, torch.Tensor) or qz.v8.dim() != 4:
        raise ValueError("qz.v8: expected a [B, H, N, 128] tensor")
    B, H, N, d = qz.v8.shape
    _require_quantized(qz, B, H, N)
    _require_nvfp4(qn, B, H, N)
    dt = torch.float32 if out_dtype == FQA_OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty(B, H, N, d, dtype=dt, device=qz.v8.device)
    _require(out, dt, "out", (B, H, N, d))
    _check(fqa_attention_nvfp4(*qn, qz.v8, qz.sv, qz.sv_max, softmax_scale, out, out_dtype, stream=stream),
           "fqa_attention_nvfp4")
    return out


def nvfp4_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, softmax_scale: float,
                    out_dtype: int = FQA_OUT_BF16, stream=None) -> torch.Tensor:
    """The whole FP4 Q.K path: quantize (V codes and the K mean), NVFP4 Q and
    K, then the attention."""
    qz = quantize(q, k, v, stream=stream)
    return attention_nvfp4(quantize_nvfp4_qk(q, k, qz.k_mean, stream=stream), qz, softmax_scale, out_dtype,
                           stream=stream)


def e2m1_encode(x: torch.Tensor, stream=None) -> torch.Tensor:
    """FP32 [..., 2n] -> uint8 [..., n]: two E2M1 codes per byte, x[2i] in the low nibble."""
    _require(x, torch.float32, "x")
    if x.numel() % 2:
        raise ValueError("x: expected an even number of elements")
    out = torch.empty(x.numel() // 2, dtype=torch.uint8, device=x.device)
    _check(fqa_e2m1_encode(x, out, stream=stream), "fqa_e2m1_encode")
    return out


def softmax_scale(d: int = HEAD_DIM) -> float:
    """fl32(1/sqrt(d))."""
    return float(torch.tensor(1.0, dtype=torch.float32) / torch.sqrt(torch.tensor(float(d), dtype=torch.float32)))
