"""Shared helpers for the GPU parity tests: seeded inputs on the device, the
oracle's results on the same inputs, and the comparison metrics."""

from __future__ import annotations

import functools

import numpy as np
import torch

import fqa_synth as synth
import oracle

SCALE = oracle.softmax_scale()


@functools.lru_cache(maxsize=2)
def host_inputs(idx: int):
    """BF16 bit arrays (uint16) for workload idx."""
    return synth.generate(synth.workload(idx))


def to_device(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda().contiguous()


@functools.lru_cache(maxsize=2)
def oracle_quant(idx: int):
    g = host_inputs(idx)
    return oracle.quantize(g["q"], g["k"], g["v"])


def sample_rows(N: int):
    """Rows checked on the large workloads: [0,128), [N/2, N/2+128), [N-128, N)."""
    return list(range(0, 128)) + list(range(N // 2, N // 2 + 128)) + list(range(N - 128, N))


def sample_heads(w):
    heads = [(0, 0), (0, w.H - 1)]
    if w.B > 1:
        heads += [(1, 0), (1, w.H - 1)]
    return heads


def to_oracle_quant(qz) -> dict:
    """GPU Quantized -> numpy dict in the oracle's naming (codes in [B,H,N,d])."""
    return dict(q8=qz.q8.cpu().numpy(), k8=qz.k8.cpu().numpy(), v8=qz.v8.cpu().numpy(),
                sq=qz.sq.cpu().numpy(), sk=qz.sk.cpu().numpy(), sv=qz.sv.cpu().numpy(),
                sv_max=qz.sv_max.cpu().numpy(), k_mean=qz.k_mean.cpu().numpy())


def metrics(gpu: np.ndarray, ref: np.ndarray) -> dict:
    gpu = gpu.astype(np.float64)
    ref = ref.astype(np.float64)
    err = np.abs(gpu - ref)
    return dict(max_abs=float(err.max()),
                mean_rel=float(err.sum() / max(np.abs(ref).sum(), 1e-300)),
                cos=float((gpu * ref).sum() / np.sqrt((gpu * gpu).sum() * (ref * ref).sum() + 1e-300)))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_to_f32(bits).astype(np.float64)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """One BF16 ulp at |x| (8 significant bits)."""
    a = np.abs(x).astype(np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)
