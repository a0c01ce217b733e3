"""Multi-token decode and state checkpoint / restore, through the C ABI.

kda_decode_step_tokens(batch, tokens) must match the fp64 oracle applied token by token
within the decode tolerances on both engines; on the five-kernel engine it must also equal
`tokens` successive single-token steps bit for bit, and on the fused engine (one kernel, the
tokens applied in order by each state unit) two runs must agree bit for bit.  kda_state_checkpoint / kda_state_restore are ordered on the handle's
stream with the steps around them: a checkpoint taken right after an enqueued step (no
synchronisation in between) holds that step's state, and restoring it replays the
following steps bit for bit.
"""
import numpy as np
import pytest

from linear_attention_layer_kda_b200 import binding, inputs as I

from gpu_util import OUT_TOL, STATE_TOL, maxrel

pytestmark = pytest.mark.gpu

RAGGED = I.KdaShape("ragged_b2_h384_2x128x64", batch=2, hidden=384, num_heads=2, head_dk=128, head_dv=64,
                    alpha_rank=32, steps=3, seed=41)
CASES = [(I.CONFIGS[0], 4), (I.CONFIGS[1].replace(batch=2), 4), (RAGGED, 3)]


def _bits(t):
    import torch
    return t.view(torch.int32)


ENGINES = [binding.KDA_ENGINE_SIMPLE, binding.KDA_ENGINE_AUTO]
FUSED_CASES = [(I.CONFIGS[1], 2), (I.CONFIGS[1], 4), (I.CONFIGS[1].replace(batch=2), 8), (I.CONFIGS[0], 8),
               (RAGGED, 3)]


def _tokens_run(shape, T, engine, runs=1):
    import torch
    from linear_attention_layer_kda_b200 import tensors
    B, H = shape.batch, shape.hidden
    inp = I.generate(shape.replace(steps=T))
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    # token t of sequence b is row b*T + t
    xs = tensors.bf16_tensor(np.stack([inp.x[t] for t in range(T)], axis=1).reshape(B * T, H))
    multi = binding.KdaDecoder(H, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B * T,
                               engine=engine)
    res = []
    try:
        used = multi.tokens_engine(B, T)
        for _ in range(runs):
            st = tensors.state_tensor(inp.state0)
            out = torch.full((B * T, H), float("nan"), device="cuda")
            multi.step_tokens(xs, w, st, out, B, T)
            multi.sync()
            res.append((out, st))
    finally:
        multi.close()
    return inp, w, res, used


def _check_oracle(inp, shape, T, out_m, st_m):
    import oracle
    B, H = shape.batch, shape.hidden
    model = oracle.OracleModel(inp, batch=B)
    try:
        S = inp.state0.astype(np.float64).copy()
        for t in range(T):
            ref = model.step(inp.x[t], S)
            eo = maxrel(out_m.view(B, T, H)[:, t].double().cpu().numpy(), ref)
            assert eo <= OUT_TOL, f"token {t}: out error {eo:.3e}"
        es = maxrel(st_m.double().cpu().numpy(), S)
        assert es <= STATE_TOL, f"state error {es:.3e}"
    finally:
        model.close()


@pytest.mark.parametrize("shape,T", CASES, ids=[f"{s.name}_T{t}" for s, t in CASES])
def test_tokens_equal_single_steps_and_the_oracle(shape, T):
    """Five-kernel engine: bit for bit the same as T single steps, and the oracle."""
    import torch
    from linear_attention_layer_kda_b200 import tensors
    B, H = shape.batch, shape.hidden
    inp, w, [(out_m, st_m)], used = _tokens_run(shape, T, binding.KDA_ENGINE_SIMPLE)
    assert used == binding.KDA_ENGINE_SIMPLE
    single = binding.KdaDecoder(H, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B,
                                engine=binding.KDA_ENGINE_SIMPLE)
    try:
        st_s = tensors.state_tensor(inp.state0)
        out_s = torch.empty(B, H, device="cuda")
        for t in range(T):
            single.step(tensors.bf16_tensor(inp.x[t]), w, st_s, out_s)
            single.sync()
            rows = out_m.view(B, T, H)[:, t]
            assert torch.equal(_bits(rows.contiguous()), _bits(out_s)), f"token {t}: out differs from a single step"
        assert torch.equal(_bits(st_m), _bits(st_s)), "state differs from single steps"
    finally:
        single.close()
    _check_oracle(inp, shape, T, out_m, st_m)


@pytest.mark.parametrize("shape,T", FUSED_CASES, ids=[f"{s.name}_T{t}" for s, t in FUSED_CASES])
def test_tokens_fused_engine_matches_the_oracle(shape, T):
    """Fused engine (one kernel per multi-token step): the oracle token by token, and two runs
    bit for bit."""
    import torch
    inp, _, res, used = _tokens_run(shape, T, binding.KDA_ENGINE_AUTO, runs=2)
    assert used == binding.KDA_ENGINE_FUSED
    (o1, s1), (o2, s2) = res
    assert torch.equal(_bits(o1), _bits(o2)) and torch.equal(_bits(s1), _bits(s2))
    _check_oracle(inp, shape, T, o1, s1)


def test_tokens_engine_choice():
    s = I.CONFIGS[1]
    dec = binding.KdaDecoder(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank, 128)
    try:
        assert dec.tokens_engine(8, 4) == binding.KDA_ENGINE_FUSED   # 32 rows
        assert dec.tokens_engine(8, 8) == binding.KDA_ENGINE_FUSED   # 64 rows
        assert dec.tokens_engine(16, 8) == binding.KDA_ENGINE_SIMPLE  # 128 rows
        assert dec.tokens_engine(1, 16) == binding.KDA_ENGINE_SIMPLE  # more than 8 tokens
        assert dec.tokens_engine(8, 1) == dec.engine(8)
    finally:
        dec.close()


def test_tokens_argument_errors():
    s = I.CONFIGS[0]
    dec = binding.KdaDecoder(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank, 4)
    try:
        lib = binding.load()
        w = binding.kda_weights()
        for n in binding.WEIGHT_FIELDS:
            setattr(w, n, 1 << 40)
        import ctypes
        assert lib.kda_decode_step_tokens(dec.h, 1 << 41, ctypes.byref(w), 1 << 42, 1 << 43, 1, 0) == \
            binding.KDA_ERR_INVALID_ARG
        assert lib.kda_decode_step_tokens(dec.h, 1 << 41, ctypes.byref(w), 1 << 42, 1 << 43, 2, 3) == \
            binding.KDA_ERR_INVALID_ARG  # 6 rows > max_batch 4
        assert lib.kda_state_checkpoint(dec.h, 1 << 42, 3, 2, 1 << 44) == binding.KDA_ERR_INVALID_ARG
        assert lib.kda_state_restore(dec.h, 1 << 44, 1 << 42, -1, 1) == binding.KDA_ERR_INVALID_ARG
    finally:
        dec.close()


def test_checkpoint_restore_is_stream_ordered_and_replays_bitwise():
    import torch

    import oracle
    from linear_attention_layer_kda_b200 import tensors
    shape = I.CONFIGS[1]  # batch 8, hidden 4096, 32 heads of 128 x 128 (fused engine)
    B, H, K = shape.batch, shape.hidden, 4
    inp = I.generate(shape.replace(steps=2 * K))
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    dec = binding.KdaDecoder(H, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B)
    xs = [tensors.bf16_tensor(inp.x[t]) for t in range(2 * K)]
    try:
        st = tensors.state_tensor(inp.state0)
        out = torch.empty(B, H, device="cuda")
        per_seq = shape.num_heads * shape.head_dk * shape.head_dv
        ck = torch.empty(B, per_seq, dtype=torch.float32).pin_memory()
        part = torch.empty(3, per_seq, dtype=torch.float32).pin_memory()
        outs_a, outs_b = [], []
        for t in range(K):
            dec.step(xs[t], w, st, out)
        dec.checkpoint(st, ck)             # right behind the queued steps, no sync
        dec.checkpoint(st, part, 2, 3)     # sequences 2..4 only
        for t in range(K, 2 * K):
            dec.step(xs[t], w, st, out)
            outs_a.append(out.clone())
        st_a = st.clone()
        st.zero_()
        dec.restore(ck, st)                # the next step must read the restored state
        for t in range(K, 2 * K):
            dec.step(xs[t], w, st, out)
            outs_b.append(out.clone())
        dec.sync()
        torch.cuda.synchronize()
        assert torch.equal(_bits(st), _bits(st_a)), "replay from the checkpoint differs"
        for a, b in zip(outs_a, outs_b):
            assert torch.equal(_bits(a), _bits(b))
        np.testing.assert_array_equal(part.numpy(), ck.numpy()[2:5])
        model = oracle.OracleModel(inp, batch=B)
        S = inp.state0.astype(np.float64).copy()
        for t in range(K):
            model.step(inp.x[t], S)
        model.close()
        es = maxrel(ck.numpy().astype(np.float64).reshape(S.shape), S)
        assert es <= STATE_TOL, f"checkpoint error {es:.3e}"
        # a partial restore touches only its sequences
        before = st.clone()
        fill = torch.full((2, per_seq), 0.5, dtype=torch.float32).pin_memory()
        dec.restore(fill, st, 5, 2)
        dec.sync()
        after = st.view(B, per_seq)
        assert torch.equal(after[5:7], torch.full((2, per_seq), 0.5, device="cuda"))
        assert torch.equal(after[:5], before.view(B, per_seq)[:5])
        assert torch.equal(after[7:], before.view(B, per_seq)[7:])
    finally:
        dec.close()
