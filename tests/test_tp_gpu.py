"""Tensor parallelism by heads on one GPU: the ranks' shards run one after another.

Every shard is an ordinary step of the library on its heads (linear_attention_layer_kda_b200.tp);
the partial outs are added on the device in place of the all-reduce.  No kernel waits on
another rank's kernel.  The sum must match the whole-layer oracle within the decode
tolerances, and every shard's state the oracle's state of its heads.
"""
import numpy as np
import pytest

from linear_attention_layer_kda_b200 import binding, inputs as I

from gpu_util import OUT_TOL, STATE_TOL, maxrel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4])
def test_head_shards_sum_to_the_whole_step(world):
    import torch

    import oracle
    from linear_attention_layer_kda_b200 import tensors, tp
    shape = I.CONFIGS[1].replace(steps=2)
    inp = I.generate(shape)
    B, H = shape.batch, shape.hidden
    shards = [tp.shard_inputs(inp, r, world) for r in range(world)]
    decs, ws, sts = [], [], []
    for sh in shards:
        s = sh.shape
        decs.append(binding.KdaDecoder(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank, B))
        ws.append(tensors.weights_struct(tensors.to_device_weights(sh)))
        sts.append(tensors.state_tensor(sh.state0))
    model = oracle.OracleModel(inp, batch=B)
    S = inp.state0.astype(np.float64).copy()
    try:
        part = torch.empty(B, H, device="cuda")
        for t in range(shape.steps):
            x = tensors.bf16_tensor(inp.x[t])
            total = torch.zeros(B, H, device="cuda")
            for d, w, st in zip(decs, ws, sts):
                d.step(x, w, st, part)
                total += part
            for d in decs:
                d.sync()
            ref = model.step(inp.x[t], S)
            eo = maxrel(total.double().cpu().numpy(), ref)
            assert eo <= OUT_TOL, f"step {t}: out error {eo:.3e}"
        hpr = shape.num_heads // world
        for r, st in enumerate(sts):
            es = maxrel(st.double().cpu().numpy(), S[:, r * hpr:(r + 1) * hpr])
            assert es <= STATE_TOL, f"rank {r}: state error {es:.3e}"
        assert decs[0].engine(B) == binding.KDA_ENGINE_FUSED
    finally:
        for d in decs:
            d.close()
        model.close()
