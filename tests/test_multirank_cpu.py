"""The N > 1 path on the CPU: two gloo ranks, data parallel over sequences.

bench.py gives each rank its own sequences (rank r holds rows r*B .. r*B + B - 1 of the
job's counter-based input streams) and shares nothing on the data path; the only
collectives are the timing barrier and the max over ranks.  Here each rank steps its shard
through the oracle, and the union of the shards must equal, bit for bit, the oracle run on
the whole job batch at once; the max-over-ranks reduction and the job rate are checked too.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    import oracle
    from linear_attention_layer_kda_b200 import inputs as I

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        shape = I.CONFIGS[0].replace(batch=2)
        inp = bench.rank_inputs(shape, rank, world)
        m = oracle.OracleModel(inp, batch=shape.batch)
        S = inp.state0.astype(np.float64).copy()
        out = m.step(inp.x[0], S)
        m.close()
        np.save(os.path.join(outdir, f"out{rank}.npy"), out)
        np.save(os.path.join(outdir, f"state{rank}.npy"), S)
        np.save(os.path.join(outdir, f"x{rank}.npy"), inp.x[0])
        worst = bench.max_over_ranks(1.5 + rank, world)
        np.save(os.path.join(outdir, f"max{rank}.npy"), np.array([worst]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_the_batch_exactly(tmp_path):
    import bench
    import oracle
    from linear_attention_layer_kda_b200 import inputs as I

    oracle.build()
    mp.start_processes(_rank_main, args=(WORLD, _free_port(), str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    shape = I.CONFIGS[0].replace(batch=2)
    job = I.generate(shape.replace(batch=2 * WORLD, steps=1))
    m = oracle.OracleModel(job, batch=2 * WORLD)
    S = job.state0.astype(np.float64).copy()
    ref = m.step(job.x[0], S)
    m.close()
    for r in range(WORLD):
        rows = slice(2 * r, 2 * r + 2)
        np.testing.assert_array_equal(np.load(tmp_path / f"x{r}.npy"), job.x[0][rows])
        np.testing.assert_array_equal(np.load(tmp_path / f"out{r}.npy"), ref[rows])
        np.testing.assert_array_equal(np.load(tmp_path / f"state{r}.npy"), S[rows])
        assert float(np.load(tmp_path / f"max{r}.npy")[0]) == 1.5 + (WORLD - 1)
    assert bench.job_steps_per_s(0.05, WORLD) == pytest.approx(WORLD * 20000.0)


def test_single_rank_needs_no_process_group():
    import bench
    from linear_attention_layer_kda_b200 import inputs as I
    assert bench.max_over_ranks(3.25, 1) == 3.25
    shape = I.CONFIGS[0]
    a, b = bench.rank_inputs(shape, 0, 1), I.generate(shape.replace(steps=1))
    np.testing.assert_array_equal(a.x[0], b.x[0])
    np.testing.assert_array_equal(a.state0, b.state0)
