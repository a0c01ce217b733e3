"""Tensor parallelism by heads: one rank per GPU owns a contiguous group of heads.

The pages run the model tensor-parallel over many cores (the TrnRT listing; the Kiln post,
"How was Kiln measured against vLLM on H200?") and move a blocking collective into the
kernel (the TrnRT story's third rule).  For this layer half the head split needs exactly one
exchange: rank g owns heads [g*nh/G, (g+1)*nh/G) -- the rows of W_q, W_k, W_v, W_a_up and
W_b for them, those heads' state, and the matching column block of W_o -- and computes a
partial out = W_o[:, its columns] o_its_heads.  W_a_down is small and replicated (every
rank forms t = W_a_down x).  The job's out is the sum of the partials over ranks: one
all-reduce of B x H fp32 per step.  By default that sum runs inside the fused kernel over
peer memory (kda_tp_configure / kda_tp_set_peer); torch.distributed.all_reduce (NCCL on
GPUs) is the other choice.
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


def exchange_handles(dec, rank: int, world: int, group=None) -> None:
    """Connects the exchange regions of a head-parallel group (every rank calls it, in order).

    Each rank configures its handle (an exchange region on its GPU), the ranks trade the
    regions' IPC handles with all_gather_object, and each maps its peers' regions.  A rank
    whose configuration fails sends None instead of a handle; then every rank raises, so no
    rank is left waiting in a later step for a peer that will never run one.
    """
    import torch.distributed as dist
    err = None
    try:
        mine = dec.tp_configure(rank, world)
    except Exception as e:  # noqa: BLE001 -- reported to every rank below
        mine, err = None, e
    handles = [None] * world
    if world > 1:
        dist.all_gather_object(handles, mine, group=group)
    else:
        handles[0] = mine
    bad = [r for r, h in enumerate(handles) if h is None]
    if bad:
        raise RuntimeError(f"tensor-parallel exchange regions failed on ranks {bad}") from err
    for peer, h in enumerate(handles):
        if peer != rank:
            dec.tp_set_peer(peer, h)


class TensorParallelDecoder:
    """One rank of a head-parallel decode step whose out is the sum over ranks.

    reduce = "fused" (the default): the sum runs inside the step's own kernel over peer
    memory (kda_tp_configure); every step must take the fused engine.  reduce = "nccl": the
    local step, then torch.distributed.all_reduce of out (any engine, any backend).
    `group` is a torch.distributed process group; every rank calls step() the same number of
    times, in the same order.
    """

    def __init__(self, shard: KdaInputs, max_batch: int, group=None, reduce: str = "fused", out_dtype=None):
        import torch
        import torch.distributed as dist

        from . import binding
        if reduce not in ("fused", "nccl"):
            raise ValueError(f"reduce must be 'fused' or 'nccl', got {reduce!r}")
        s = shard.shape
        kw = {} if out_dtype is None else {"out_dtype": out_dtype}
        self.dec = binding.KdaDecoder(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank, max_batch, **kw)
        self.group = group
        self.reduce = reduce
        self._dist = dist
        self._torch = torch
        if reduce == "fused":
            rank = dist.get_rank(group) if dist.is_initialized() else 0
            world = dist.get_world_size(group) if dist.is_initialized() else 1
            try:
                exchange_handles(self.dec, rank, world, group)
            except Exception:
                self.dec.close()
                raise

    def step(self, x, weights, state_shard, out, batch=None) -> None:
        """out ([B, H]) becomes the whole layer half's output on every rank."""
        self.dec.step(x, weights, state_shard, out, batch)
        if self.reduce == "nccl":
            self._dist.all_reduce(out, op=self._dist.ReduceOp.SUM, group=self.group)

    def step_tokens(self, x, weights, state_shard, out, batch: int, tokens: int) -> None:
        self.dec.step_tokens(x, weights, state_shard, out, batch, tokens)
        if self.reduce == "nccl":
            self._dist.all_reduce(out, op=self._dist.ReduceOp.SUM, group=self.group)

    def prefill(self, x, weights, state_shard, out, batch: int, tokens: int, chunk: int = 0) -> None:
        """A prompt through the chunked form on this rank's heads; out ([batch * tokens, H], fp32)
        becomes the whole layer's output on every rank (the partial outs summed with
        torch.distributed.all_reduce in either mode: the prefill kernels do not exchange)."""
        self.dec.prefill(x, weights, state_shard, out, batch, tokens, chunk)
        if self._dist.is_initialized() and self._dist.get_world_size(self.group) > 1:
            self._dist.all_reduce(out, op=self._dist.ReduceOp.SUM, group=self.group)

    def sync(self) -> None:
        self.dec.sync()

    def close(self) -> None:
        self.dec.close()
