"""The in-kernel out reduction of a head-parallel group, on one GPU (a group of one rank).

A configured handle pushes its partial out into the exchange region, raises the blocks'
flags and adds the ranks' partials in rank order inside the fused kernel.  With one rank the
sum is 0 + partial, so the out must equal the plain fused step's bit for bit, for fp32 and
bf16 out, one and several tokens, and over many steps (the exchange flips parity every
step).  Groups of two or more ranks need one GPU per rank: their host logic is covered on
CPU (test_tp_cpu.py); no kernel here waits on another rank's kernel.
"""
import numpy as np
import pytest

from linear_attention_layer_kda_b200 import binding, inputs as I

from gpu_util import OUT_TOL, STATE_TOL, maxrel

pytestmark = pytest.mark.gpu


def _setup(shape, out_dtype=binding.KDA_OUT_F32):
    import torch
    from linear_attention_layer_kda_b200 import tensors
    inp = I.generate(shape)
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    tdt = torch.float32 if out_dtype == binding.KDA_OUT_F32 else torch.bfloat16
    return inp, w, tdt


def _decoder(shape, max_batch=None, out_dtype=binding.KDA_OUT_F32):
    s = shape
    return binding.KdaDecoder(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank,
                              max_batch or s.batch, out_dtype=out_dtype)


@pytest.mark.parametrize("out_dtype", [binding.KDA_OUT_F32, binding.KDA_OUT_BF16], ids=["f32", "bf16"])
def test_group_of_one_equals_the_plain_step(out_dtype):
    import torch
    from linear_attention_layer_kda_b200 import tensors, tp
    shape = I.CONFIGS[1].replace(steps=6)
    inp, w, tdt = _setup(shape, out_dtype)
    B, H = shape.batch, shape.hidden
    plain = _decoder(shape, out_dtype=out_dtype)
    group = tp.TensorParallelDecoder(inp, B, reduce="fused", out_dtype=out_dtype)
    try:
        assert group.dec.engine(B) == binding.KDA_ENGINE_FUSED
        s1, s2 = tensors.state_tensor(inp.state0), tensors.state_tensor(inp.state0)
        o1 = torch.empty(B, H, device="cuda", dtype=tdt)
        o2 = torch.full((B, H), float("nan"), device="cuda", dtype=tdt)
        for t in range(shape.steps):
            x = tensors.bf16_tensor(inp.x[t])
            plain.step(x, w, s1, o1)
            group.step(x, w, s2, o2)
            plain.sync()
            group.sync()
            assert torch.equal(o1, o2), f"step {t}: out differs from the plain step"
        assert torch.equal(s1, s2)
    finally:
        group.close()
        plain.close()


def test_group_of_one_matches_the_oracle_with_tokens():
    import torch

    import oracle
    from linear_attention_layer_kda_b200 import tensors, tp
    T = 3
    shape = I.CONFIGS[1].replace(steps=T)
    inp, w, _ = _setup(shape)
    B, H = shape.batch, shape.hidden
    group = tp.TensorParallelDecoder(inp, B * T)
    model = oracle.OracleModel(inp, batch=B)
    try:
        assert group.dec.tokens_engine(B, T) == binding.KDA_ENGINE_FUSED
        st = tensors.state_tensor(inp.state0)
        xs = tensors.bf16_tensor(np.stack([inp.x[t] for t in range(T)], axis=1).reshape(B * T, H))
        out = torch.full((B * T, H), float("nan"), device="cuda")
        group.step_tokens(xs, w, st, out, B, T)
        group.sync()
        S = inp.state0.astype(np.float64).copy()
        got = out.view(B, T, H).double().cpu().numpy()
        for t in range(T):
            ref = model.step(inp.x[t], S)
            assert maxrel(got[:, t], ref) <= OUT_TOL
        assert maxrel(st.double().cpu().numpy(), S) <= STATE_TOL
    finally:
        group.close()
        model.close()


def test_configuration_errors_enqueue_nothing():
    import torch
    from linear_attention_layer_kda_b200 import tensors
    shape = I.CONFIGS[1]
    inp, w, _ = _setup(shape)
    B, H = shape.batch, shape.hidden
    dec = _decoder(shape, max_batch=80)
    try:
        for rank, world in [(0, 0), (1, 1), (-1, 2), (0, 9)]:
            with pytest.raises(binding.KdaError):
                dec.tp_configure(rank, world)
        with pytest.raises(binding.KdaError):
            dec.tp_set_peer(1, bytes(binding.KDA_TP_HANDLE_BYTES))  # not configured
        handle = dec.tp_configure(0, 2)
        assert len(handle) == binding.KDA_TP_HANDLE_BYTES
        with pytest.raises(binding.KdaError):
            dec.tp_configure(0, 2)  # once per handle
        for peer in (0, 2, -1):  # itself, out of range
            with pytest.raises(binding.KdaError):
                dec.tp_set_peer(peer, handle)
        st = tensors.state_tensor(inp.state0)
        out = torch.zeros(B, H, device="cuda")
        x = tensors.bf16_tensor(inp.x[0])
        with pytest.raises(binding.KdaError, match="not all mapped"):
            dec.step(x, w, st, out)  # peer 1 is not mapped
        big = torch.zeros(80, H, device="cuda", dtype=torch.bfloat16)
        st_big = torch.zeros(80, *st.shape[1:], device="cuda")
        assert dec.engine(80) == binding.KDA_ENGINE_SIMPLE
        with pytest.raises(binding.KdaError, match="fused engine"):
            dec.step(big, w, st_big, torch.zeros(80, H, device="cuda"))
        dec.sync()
        assert torch.count_nonzero(out) == 0  # nothing ran
        assert torch.equal(st, tensors.state_tensor(inp.state0))
    finally:
        dec.close()


def test_prefill_on_a_configured_handle():
    """kda_prefill on a tensor-parallel handle returns the rank's partial out: with one rank,
    the plain prefill's bits."""
    import torch
    from linear_attention_layer_kda_b200 import tensors, tp
    shape = I.CONFIGS[1].replace(steps=48)
    inp, w, _ = _setup(shape)
    B, H, T = shape.batch, shape.hidden, 48
    xs = tensors.bf16_tensor(np.stack([inp.x[t] for t in range(T)], axis=1).reshape(B * T, H))
    plain = _decoder(shape)
    group = tp.TensorParallelDecoder(inp, B)
    try:
        s1, s2 = tensors.state_tensor(inp.state0), tensors.state_tensor(inp.state0)
        o1 = torch.empty(B * T, H, device="cuda")
        o2 = torch.full((B * T, H), float("nan"), device="cuda")
        plain.prefill(xs, w, s1, o1, B, T, 16)
        group.prefill(xs, w, s2, o2, B, T, 16)
        plain.sync()
        group.sync()
        assert torch.equal(o1, o2) and torch.equal(s1, s2)
    finally:
        group.close()
        plain.close()


def test_nccl_reduce_mode_at_one_rank(tmp_path):
    """reduce="nccl": the local step, then torch.distributed.all_reduce of out over NCCL.  With
    one rank the sum is the rank's own out, so it must equal the plain step bit for bit."""
    import datetime

    import torch
    import torch.distributed as dist
    from linear_attention_layer_kda_b200 import tensors, tp
    if dist.is_initialized():
        pytest.skip("a process group is already initialised in this process")
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        shape = I.CONFIGS[1].replace(steps=3)
        inp, w, _ = _setup(shape)
        B, H = shape.batch, shape.hidden
        plain = _decoder(shape)
        group = tp.TensorParallelDecoder(inp, B, reduce="nccl")
        try:
            s1, s2 = tensors.state_tensor(inp.state0), tensors.state_tensor(inp.state0)
            o1 = torch.empty(B, H, device="cuda")
            o2 = torch.full((B, H), float("nan"), device="cuda")
            for t in range(shape.steps):
                x = tensors.bf16_tensor(inp.x[t])
                plain.step(x, w, s1, o1)
                group.step(x, w, s2, o2)
                plain.sync()
                group.sync()
                torch.cuda.synchronize()
                assert torch.equal(o1, o2), f"step {t}: out differs from the plain step"
            assert torch.equal(s1, s2)
        finally:
            group.close()
            plain.close()
    finally:
        dist.destroy_process_group()
