"""Sequence-parallel (Ulysses) FP8 attention with the CFG pair split across
GPU groups.

"FLUX 3 Image Klein Base: 생성 3.46배, 8장 확장 병목", sections "결과" and
"고를 때 기준": on 8 B200s the Base model runs CFG parallel (the positive and
negative prompts on separate GPU groups) times Ulysses sequence parallel of
degree 4, the step-reduced model Ulysses of degree 8.  Ulysses shards the
sequence over the P ranks of a group; before attention an all-to-all turns a
rank's sequence shard (all heads, tokens [r Nl, (r+1) Nl)) into a head shard
(H / P heads, all tokens), and after attention a second all-to-all turns it
back.

The collectives are torch.distributed all_to_all_single calls (NCCL over
NVLink / NVSwitch on GPUs), one per batch element.  Their buffers need no
pack or unpack pass: the receive buffer's layout [B, P, Hl, Nl, d] is read
directly by fqa_quantize_a2a, and fqa_attention_fp8_a2a writes its output in
that layout, which is the send buffer of the return all-to-all.
"""

from __future__ import annotations

from typing import Optional

import torch
import torch.distributed as dist


class GpuOps:
    """The library's CUDA calls the wrapper runs between the collectives."""

    def __init__(self, fqa_module=None):
        if fqa_module is None:
            import quantized_fp8_attention_b200 as fqa_module
        self.fqa = fqa_module

    def empty(self, shape, dtype, like: torch.Tensor) -> torch.Tensor:
        return torch.empty(shape, dtype=dtype, device=like.device)

    def quantize_a2a(self, q, k, v):
        return self.fqa.quantize_a2a(q, k, v)

    def attention_fp8_a2a(self, qz, P: int, softmax_scale: float, out_dtype: int):
        return self.fqa.attention_fp8_a2a(qz, P, softmax_scale, out_dtype)

    def out_dtype(self, out_dtype: int) -> torch.dtype:
        return torch.float32 if out_dtype == self.fqa.FQA_OUT_F32 else torch.bfloat16


def _seq_to_heads(x: torch.Tensor, P: int, group, ops) -> torch.Tensor:
    """[B, H, Nl, d] sequence shard -> [B, P, Hl, Nl, d] head shard (chunk p:
    rank p's tokens) by one all-to-all per batch element."""
    B, H, Nl, d = x.shape
    recv = ops.empty((B, P, H // P, Nl, d), x.dtype, x)
    for b in range(B):
        # x[b] is [H, Nl, d] = P chunks of Hl heads: chunk p goes to rank p
        dist.all_to_all_single(recv[b], x[b].contiguous(), group=group)
    return recv


def _heads_to_seq(o: torch.Tensor, group, ops) -> torch.Tensor:
    """[B, P, Hl, Nl, d] (chunk p: rank p's tokens of this rank's heads) ->
    [B, H, Nl, d] sequence shard."""
    B, P, Hl, Nl, d = o.shape
    out = ops.empty((B, P * Hl, Nl, d), o.dtype, o)
    for b in range(B):
        dist.all_to_all_single(out[b], o[b].contiguous(), group=group)
    return out


def ulysses_fp8_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, softmax_scale: float,
                          group=None, out_dtype: Optional[int] = None, ops=None) -> torch.Tensor:
    """FP8 attention over a sequence sharded across the ranks of `group`.

    q, k, v: this rank's shard [B, H, Nl, d] (BF16): rank r of the group holds
    tokens [r Nl, (r+1) Nl) of every head; H must be a multiple of the group
    size P and Nl of 64.  Returns this rank's shard of the output [B, H, Nl, d].
    Every rank runs the same two all-to-alls per batch element, in order."""
    ops = ops if ops is not None else GpuOps()
    if out_dtype is None:
        out_dtype = 0
    P = dist.get_world_size(group)
    B, H, Nl, d = q.shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k and v must have the same shape")
    rq, rk, rv = (_seq_to_heads(t, P, group, ops) for t in (q, k, v))
    qz = ops.quantize_a2a(rq, rk, rv)
    o = ops.attention_fp8_a2a(qz, P, softmax_scale, out_dtype)
    return _heads_to_seq(o, group, ops)


def cfg_ulysses_groups(cfg: int):
    """Split the world into `cfg` consecutive groups of P = world / cfg ranks
    (CFG parallel: group c handles batch slice c).  Every rank must call this,
    in the same order.  Returns (this rank's group, its index c, P)."""
    world, rank = dist.get_world_size(), dist.get_rank()
    if world % cfg:
        raise ValueError(f"world size {world} does not split into {cfg} CFG groups")
    P = world // cfg
    mine = None
    for c in range(cfg):
        g = dist.new_group(list(range(c * P, (c + 1) * P)))
        if rank // P == c:
            mine = g
    return mine, rank // P, P


def cfg_ulysses_fp8_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, softmax_scale: float,
                              group, out_dtype: Optional[int] = None, ops=None) -> torch.Tensor:
    """CFG parallel x Ulysses: this rank holds its CFG group's batch slice and
    its sequence shard, [B / cfg, H, Nl, d]; attention runs over the group
    (cfg_ulysses_groups) exactly as ulysses_fp8_attention."""
    return ulysses_fp8_attention(q, k, v, softmax_scale, group=group, out_dtype=out_dtype, ops=ops)
