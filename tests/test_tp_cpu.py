"""Tensor parallelism by heads, host side: the shards of two gloo ranks reproduce the whole step.

Each rank takes its heads' weights and state (linear_attention_layer_kda_b200.tp), steps
them through the oracle and all-reduces its partial out over gloo.  The heads' states must
equal the whole-layer oracle's bit for bit (heads are independent); the summed out equals
the whole layer's out up to the order of the final additions.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SHAPE_ARGS = dict(name="tp_b2_h256_4x64", batch=2, hidden=256, num_heads=4, head_dk=64, head_dv=64,
                  alpha_rank=32, steps=2, seed=17)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from linear_attention_layer_kda_b200 import inputs as I, tp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = I.generate(I.KdaShape(**SHAPE_ARGS))
        sh = tp.shard_inputs(inp, rank, world)
        m = oracle.OracleModel(sh, batch=sh.shape.batch)
        S = sh.state0.astype(np.float64).copy()
        for t in range(SHAPE_ARGS["steps"]):
            part = torch.from_numpy(m.step(inp.x[t], S).copy())
            dist.all_reduce(part, op=dist.ReduceOp.SUM)
            np.save(os.path.join(outdir, f"out{rank}_{t}.npy"), part.numpy())
        m.close()
        np.save(os.path.join(outdir, f"state{rank}.npy"), S)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_heads_exactly(tmp_path):
    import oracle
    from linear_attention_layer_kda_b200 import inputs as I
    oracle.build()
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    inp = I.generate(I.KdaShape(**SHAPE_ARGS))
    m = oracle.OracleModel(inp, batch=inp.shape.batch)
    S = inp.state0.astype(np.float64).copy()
    for t in range(SHAPE_ARGS["steps"]):
        ref = m.step(inp.x[t], S)
        for r in range(world):
            got = np.load(tmp_path / f"out{r}_{t}.npy")
            assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()
    m.close()
    hpr = SHAPE_ARGS["num_heads"] // world
    for r in range(world):
        np.testing.assert_array_equal(np.load(tmp_path / f"state{r}.npy"), S[:, r * hpr:(r + 1) * hpr])


def test_shard_layout():
    from linear_attention_layer_kda_b200 import inputs as I, tp
    inp = I.generate(I.CONFIGS[1].replace(steps=1))
    sh = tp.shard_inputs(inp, 1, 4)  # heads 8..15
    assert sh.shape.num_heads == 8
    np.testing.assert_array_equal(sh.wq, inp.wq[1024:2048])
    np.testing.assert_array_equal(sh.sq, inp.sq[8:16])
    np.testing.assert_array_equal(sh.wo, inp.wo[:, 1024:2048])
    np.testing.assert_array_equal(sh.so, inp.so[:, 8:16])
    np.testing.assert_array_equal(sh.wb, inp.wb[8:16])
    np.testing.assert_array_equal(sh.wa_up, inp.wa_up[1024:2048])
    assert sh.wa_down is inp.wa_down
    np.testing.assert_array_equal(sh.state0, inp.state0[:, 8:16])
    assert sh.wo.flags["C_CONTIGUOUS"] and sh.state0.flags["C_CONTIGUOUS"]
    with pytest.raises(ValueError):
        tp.head_range(32, 0, 3)
    with pytest.raises(ValueError):  # 1 head of 64 per rank: not a whole 128-wide block
        tp.check_shardable(I.CONFIGS[0], 2)


class _FakeHandle:
    """Stands in for a KdaDecoder's tensor-parallel calls (no GPU): records what it was given."""

    def __init__(self, rank, fail_rank=None):
        self.rank, self.fail_rank = rank, fail_rank
        self.configured, self.peers = None, {}

    def tp_configure(self, rank, world):
        if rank == self.fail_rank:
            raise RuntimeError("no exchange region")
        self.configured = (rank, world)
        return bytes([rank + 1]) * 64

    def tp_set_peer(self, peer, handle):
        self.peers[peer] = handle


def _exchange_main(rank, world, port, outdir, fail_rank):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from linear_attention_layer_kda_b200 import tp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        fake = _FakeHandle(rank, fail_rank)
        try:
            tp.exchange_handles(fake, rank, world)
            result = {"configured": fake.configured, "peers": {p: h[0] for p, h in fake.peers.items()}}
        except RuntimeError as e:
            result = {"error": str(e), "peers": {p: h[0] for p, h in fake.peers.items()}}
        np.save(os.path.join(outdir, f"x{rank}.npy"), np.array([repr(result)]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,fail_rank", [(2, None), (3, None), (3, 1)])
def test_exchange_handles_over_gloo(tmp_path, world, fail_rank):
    """Every rank maps every other rank's region with that rank's handle; a failed rank fails all."""
    import ast
    mp.start_processes(_exchange_main, args=(world, _free_port(), str(tmp_path), fail_rank), nprocs=world,
                       join=True, start_method="spawn")
    for r in range(world):
        res = ast.literal_eval(str(np.load(tmp_path / f"x{r}.npy")[0]))
        if fail_rank is None:
            assert res["configured"] == (r, world)
            assert res["peers"] == {p: p + 1 for p in range(world) if p != r}
        else:
            assert f"ranks [{fail_rank}]" in res["error"]
            assert res["peers"] == {}  # nobody maps anything
