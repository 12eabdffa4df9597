"""The Ulysses / CFG-parallel wrapper on CPU gloo ranks ("FLUX 3 Image Klein
Base: 생성 3.46배, 8장 확장 병목", sections "결과" and "고를 때 기준": CFG
groups times Ulysses sequence parallel on a DGX B200).

Each rank holds a sequence shard of the seeded inputs and runs the wrapper's
real collectives (torch.distributed all_to_all_single on gloo); only the two
library calls between them, which need a B200, are replaced by an emulation
of the same layouts on the CPU oracle.  Every rank's output shard must equal
the oracle's FP8 attention on the whole sequence, bit for bit: this pins the
routing (which rank gets which heads and tokens, in which order) and the
all-to-all layout [B, P, Hl, Nl, d] both ways.  The GPU side of the layouts
is checked on one GPU in tests/test_gpu_ulysses.py.
"""

import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, H, N, seed):
    sys.path.insert(0, ROOT)
    import fqa_synth as synth
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, N, 128)) * 2
    k = rng.standard_normal((B, H, N, 128)) * 2 + rng.standard_normal((B, H, 1, 128))
    v = rng.standard_normal((B, H, N, 128))
    return {t: synth.round_to_bf16_bits(x) for t, x in zip("qkv", (q, k, v))}


class OracleOps:
    """The wrapper's two library calls, emulated on the oracle with the same
    input and output layouts (test infrastructure)."""

    def empty(self, shape, dtype, like):
        return torch.empty(shape, dtype=dtype)

    def quantize_a2a(self, q, k, v):
        import oracle

        def std(t):                              # [B, P, Hl, Nl, d] -> [B, Hl, P * Nl, d]
            bits = t.contiguous().view(torch.int16).numpy().view(np.uint16)
            B, P, Hl, Nl, d = bits.shape
            return np.ascontiguousarray(bits.transpose(0, 2, 1, 3, 4).reshape(B, Hl, P * Nl, d))
        return oracle.quantize(std(q), std(k), std(v))

    def attention_fp8_a2a(self, qz, P, scale, out_dtype):
        import oracle
        B, Hl, N, d = qz["q8"].shape
        o = oracle.attention_fp8(qz, scale).reshape(B, Hl, P, N // P, d).transpose(0, 2, 1, 3, 4)
        return torch.from_numpy(np.ascontiguousarray(o.astype(np.float32)))


def _worker(rank, world, port, cfg, shape, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        from quantized_fp8_attention_b200 import ulysses
        B, H, N = shape
        g = _inputs(B, H, N, 77)
        if cfg > 1:
            group, c, P = ulysses.cfg_ulysses_groups(cfg)
            bsl = slice(c * (B // cfg), (c + 1) * (B // cfg))
        else:
            group, P, bsl = None, world, slice(0, B)
        r = rank % P
        Nl = N // P

        def shard(bits):
            x = np.ascontiguousarray(bits[bsl, :, r * Nl:(r + 1) * Nl])
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)

        out = ulysses.ulysses_fp8_attention(shard(g["q"]), shard(g["k"]), shard(g["v"]), oracle.softmax_scale(),
                                            group=group, ops=OracleOps())
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), out.numpy())
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"P": P, "r": r, "b0": bsl.start, "b1": bsl.stop}, f)
    finally:
        dist.destroy_process_group()


def _run(world, cfg, shape, tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, cfg, shape, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    import oracle
    B, H, N = shape
    g = _inputs(B, H, N, 77)
    ref = oracle.attention_fp8(oracle.quantize(g["q"], g["k"], g["v"]), oracle.softmax_scale())
    ref = ref.reshape(B, H, N, 128).astype(np.float32)
    for rank in range(world):
        meta = json.load(open(tmp_path / f"rank{rank}.json"))
        got = np.load(tmp_path / f"rank{rank}.npy")
        Nl = N // meta["P"]
        want = ref[meta["b0"]:meta["b1"], :, meta["r"] * Nl:(meta["r"] + 1) * Nl]
        assert got.shape == want.shape, (rank, got.shape, want.shape)
        assert np.array_equal(got, want), f"rank {rank}: max diff {np.abs(got - want).max()}"


def test_ulysses_two_ranks(tmp_path):
    """Ulysses degree 2: B=1, 4 heads (2 per rank), N=256 (128 tokens per rank)."""
    _run(2, 1, (1, 4, 256), tmp_path)


def test_cfg_times_ulysses_four_ranks(tmp_path):
    """CFG 2 groups x Ulysses 2: the batched guidance pair (B=2) split across
    the groups, 6 heads and N=384 sharded inside each group."""
    _run(4, 2, (2, 6, 384), tmp_path)


def test_ulysses_four_ranks_one_group(tmp_path):
    """Ulysses degree 4 on one group: 8 heads, N=512 (128 tokens per rank)."""
    _run(4, 1, (1, 8, 512), tmp_path)
