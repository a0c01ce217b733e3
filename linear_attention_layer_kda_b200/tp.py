"""Tensor parallelism by heads: one rank per GPU owns a contiguous group of heads.

The pages run the model tensor-parallel over many cores (the TrnRT listing; the Kiln post,
"How was Kiln measured against vLLM on H200?") and move a blocking collective into the
kernel (the TrnRT story's third rule).  For this layer half the head split needs exactly one
exchange: rank g owns heads [g*nh/G, (g+1)*nh/G) -- the rows of W_q, W_k, W_v, W_a_up and
W_b for them, those heads' state, and the matching column block of W_o -- and computes a
partial out = W_o[:, its columns] o_its_heads.  W_a_down is small and replicated (every
rank forms t = W_a_down x).  The job's out is the sum of the partials over ranks: one
all-reduce of B x H fp32 per step, done here with torch.distributed (NCCL on GPUs).

Host-side sharding only: each rank then runs the ordinary single-GPU step on its shard.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from .inputs import KdaInputs


def head_range(num_heads: int, rank: int, world: int):
    """Heads [h0, h1) of `rank`; requires an even split."""
    if world < 1 or num_heads % world:
        raise ValueError(f"{num_heads} heads do not split evenly over {world} ranks")
    n = num_heads // world
    return rank * n, (rank + 1) * n


def check_shardable(shape, world: int) -> None:
    """Each rank's q/k and v row blocks and W_o column block must be whole 128-wide scale blocks."""
    h0, h1 = head_range(shape.num_heads, 0, world)
    n = h1 - h0
    if (n * shape.head_dk) % 128 or (n * shape.head_dv) % 128:
        raise ValueError(f"{n} heads per rank of {shape.head_dk} x {shape.head_dv} do not fill 128-wide blocks")


def shard_inputs(inp: KdaInputs, rank: int, world: int) -> KdaInputs:
    """The inputs of one rank: its heads' weights, scales and state; x and W_a_down whole."""
    s = inp.shape
    check_shardable(s, world)
    h0, h1 = head_range(s.num_heads, rank, world)
    dk, dv = s.head_dk, s.head_dv
    qk = slice(h0 * dk, h1 * dk)
    vv = slice(h0 * dv, h1 * dv)
    qk_b = slice(h0 * dk // 128, h1 * dk // 128)
    vv_b = slice(h0 * dv // 128, h1 * dv // 128)
    c = np.ascontiguousarray
    return KdaInputs(
        shape=dataclasses.replace(s, num_heads=h1 - h0, name=f"{s.name}_tp{rank}of{world}"),
        x=inp.x,
        wq=c(inp.wq[qk]), sq=c(inp.sq[qk_b]),
        wk=c(inp.wk[qk]), sk=c(inp.sk[qk_b]),
        wv=c(inp.wv[vv]), sv=c(inp.sv[vv_b]),
        wo=c(inp.wo[:, vv]), so=c(inp.so[:, vv_b]),
        wa_down=inp.wa_down,
        wa_up=c(inp.wa_up[qk]),
        wb=c(inp.wb[h0:h1]),
        state0=c(inp.state0[:, h0:h1]),
    )


class TensorParallelDecoder:
    """One rank of a head-parallel decode step: the local step, then a sum of out over ranks.

    `group` is a torch.distributed process group (NCCL for GPUs); every rank calls step()
    the same number of times, in the same order.
    """

    def __init__(self, shard: KdaInputs, max_batch: int, group=None):
        import torch
        import torch.distributed as dist

        from . import binding
        s = shard.shape
        self.dec = binding.KdaDecoder(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank, max_batch)
        self.group = group
        self._dist = dist
        self._torch = torch

    def step(self, x, weights, state_shard, out) -> None:
        """out (fp32 [B, H]) becomes the whole layer half's output on every rank."""
        self.dec.step(x, weights, state_shard, out)
        self._dist.all_reduce(out, op=self._dist.ReduceOp.SUM, group=self.group)

    def sync(self) -> None:
        self.dec.sync()

    def close(self) -> None:
        self.dec.close()
