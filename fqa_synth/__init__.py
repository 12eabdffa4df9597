"""Seeded synthetic Q/K/V for the FLUX-style DiT attention workloads.

This module is shared by the tests, the benchmark and the CPU checker. It holds
none of the attention method's arithmetic: only a counter-based random number
generator, Box-Muller normals, the five workload recipes, and the rounding of
the drawn FP64 values to BF16 storage.

Random numbers
--------------
Every (seed, batch b, stream t, head h) has its own splitmix64 stream
(Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014): state_0 = key, state_{i+1} = state_i + 0x9E3779B97F4A7C15,
output_i = mix64(state_{i+1}), where mix64 is the splitmix64 finaliser.
The key is mix64(mix64(mix64(mix64(seed) ^ (b+1)) ^ (t+1)) ^ (h+1)).
Uniforms are u = (output >> 11) * 2^-53 in [0, 1).  Standard normals come in
pairs from Box-Muller: r = sqrt(-2 ln(1 - u0)), z0 = r cos(2 pi u1),
z1 = r sin(2 pi u1).  Streams: t = 0 (Q), 1 (K), 2 (V), 3 (outlier-channel
choice), 4 (K per-channel offsets).  Element (n, c) of a head's [N, 128]
matrix is normal number n*128 + c of its stream.

Workloads
---------
The token sequence is [text | context image | output image] (FLUX.1 Kontext
concatenates the context-image tokens to the output-image tokens, "NVIDIA RTX
AI optimiert FLUX.1", the model-structure paragraph).  Per element, in FP64:
draw z; x1.5 on context-image tokens; x3 on text tokens (Q, K and V); x20 on
the head's 4 outlier channels (Q and K only); + offset[c] (K only, offset
~ N(0, sd 2) per (b, h, c)); then one round-to-nearest-even to BF16.
"""

from __future__ import annotations

import dataclasses
import hashlib

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_Q, STREAM_K, STREAM_V, STREAM_OUTLIER, STREAM_OFFSET = 0, 1, 2, 3, 4
HEAD_DIM = 128
N_OUTLIERS = 4


def mix64(x):
    """splitmix64 finaliser on uint64 scalars or arrays (wrapping arithmetic)."""
    x = np.asarray(x, dtype=np.uint64)
    with np.errstate(over="ignore"):
        x = (x ^ (x >> np.uint64(30))) * _M1
        x = (x ^ (x >> np.uint64(27))) * _M2
        x = x ^ (x >> np.uint64(31))
    return x


def stream_key(seed: int, b: int, t: int, h: int) -> np.uint64:
    k = mix64(np.uint64(seed))
    k = mix64(k ^ np.uint64(b + 1))
    k = mix64(k ^ np.uint64(t + 1))
    k = mix64(k ^ np.uint64(h + 1))
    return np.uint64(k)


def uniforms(key: np.uint64, start: int, count: int) -> np.ndarray:
    """Uniforms number start .. start+count-1 of the stream with this key."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = np.uint64(key) + idx * GAMMA
    bits = mix64(state)
    return (bits >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normals(key: np.uint64, count: int) -> np.ndarray:
    """The first `count` standard normals of a stream (Box-Muller pairs)."""
    pairs = (count + 1) // 2
    u = uniforms(key, 0, 2 * pairs)
    u0, u1 = u[0::2], u[1::2]
    r = np.sqrt(-2.0 * np.log1p(-u0))
    th = 2.0 * np.pi * u1
    z = np.empty(2 * pairs, dtype=np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    return z[:count]


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """FP64 -> BF16 bit patterns, one round-to-nearest-even (normal range)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2^e, 0.5 <= |m| < 1
    q = np.rint(m * 256.0)                  # 8 significant bits, ties to even
    y = np.ldexp(q, e - 8).astype(np.float32)   # exact: 8-bit significand
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    n_text: int
    n_ctx: int
    n_img: int
    seed: int
    text_scale: float       # multiplies text tokens of Q, K and V
    ctx_scale: float        # multiplies context-image tokens
    outliers: bool          # 4 channels x20 in Q and K
    k_offset: bool          # K + per-channel N(0, sd 2) offset
    d: int = HEAD_DIM

    @property
    def N(self) -> int:
        return self.n_text + self.n_ctx + self.n_img

    @property
    def flops(self) -> int:
        return 4 * self.B * self.H * self.N * self.N * self.d


# The five attention workloads (FLUX-style DiT sequence lengths for 512^2,
# 1024^2 and 2048^2 images at 16x latent downsampling with 2x2 patches, plus
# text tokens; the Kontext editing case doubles the image tokens).
WORKLOADS = [
    Workload("tiny_n256", 1, 2, 64, 0, 192, 1000, 1.0, 1.0, False, True),
    Workload("dit512_n1280", 1, 24, 256, 0, 1024, 1001, 3.0, 1.0, True, False),
    Workload("dit1024_n4608", 1, 24, 512, 0, 4096, 1002, 3.0, 1.0, True, True),
    Workload("kontext_n8704", 1, 24, 512, 4096, 4096, 1003, 3.0, 1.5, True, True),
    Workload("dit2048_cfg_n16896", 2, 24, 512, 0, 16384, 1004, 3.0, 1.0, True, True),
]


def workload(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[name_or_index]
    for w in WORKLOADS:
        if w.name == name_or_index:
            return w
    raise KeyError(name_or_index)


def outlier_channels(seed: int, b: int, h: int, d: int = HEAD_DIM) -> np.ndarray:
    """4 distinct channels per (b, h): partial Fisher-Yates on stream 3."""
    u = uniforms(stream_key(seed, b, STREAM_OUTLIER, h), 0, N_OUTLIERS)
    perm = list(range(d))
    for k in range(N_OUTLIERS):
        j = k + int(np.floor(u[k] * (d - k)))
        perm[k], perm[j] = perm[j], perm[k]
    return np.array(perm[:N_OUTLIERS], dtype=np.int64)


def head_fp64(w: Workload, b: int, h: int, which: str) -> np.ndarray:
    """One head's [N, d] FP64 values before BF16 rounding. which in 'qkv'."""
    t = {"q": STREAM_Q, "k": STREAM_K, "v": STREAM_V}[which]
    N, d = w.N, w.d
    x = normals(stream_key(w.seed, b, t, h), N * d).reshape(N, d)
    if w.n_ctx and w.ctx_scale != 1.0:
        x[w.n_text:w.n_text + w.n_ctx] *= w.ctx_scale
    if w.text_scale != 1.0:
        x[:w.n_text] *= w.text_scale
    if w.outliers and which in "qk":
        x[:, outlier_channels(w.seed, b, h, d)] *= 20.0
    if w.k_offset and which == "k":
        off = 2.0 * normals(stream_key(w.seed, b, STREAM_OFFSET, h), d)
        x += off[None, :]
    return x


def generate(w: Workload, which: str = "qkv", heads=None):
    """BF16 bit patterns (uint16) of shape [B, H, N, d] for each tensor in `which`.

    heads: optional list of (b, h) to fill; the rest stays zero (for partial
    CPU checks on the largest workloads)."""
    out = {}
    for t in which:
        a = np.zeros((w.B, w.H, w.N, w.d), dtype=np.uint16)
        todo = heads if heads is not None else [(b, h) for b in range(w.B) for h in range(w.H)]
        for (b, h) in todo:
            a[b, h] = round_to_bf16_bits(head_fp64(w, b, h, t))
        out[t] = a
    return out


def sha256(a: np.ndarray) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()
