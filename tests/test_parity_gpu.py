"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances are the decode benchmark's: max-norm relative error <= 2e-3 on
out and <= 1e-3 on the updated state, every checked step.
"""
import dataclasses

import numpy as np
import pytest

from linear_attention_layer_kda_b200 import binding, inputs as I

from gpu_util import OUT_TOL, STATE_TOL, run_parity
from helpers import gate_weights

pytestmark = pytest.mark.gpu

ENGINES = [binding.KDA_ENGINE_SIMPLE, binding.KDA_ENGINE_AUTO]

# dk != dv, hidden of three 128-blocks, ragged batch of 5
RAGGED = I.KdaShape("ragged_b5_h384_2x128x64", batch=5, hidden=384, num_heads=2, head_dk=128, head_dv=64,
                    alpha_rank=32, steps=3, seed=21)


def _assert_ok(errs, tag):
    for t, eo, es in errs:
        assert eo <= OUT_TOL and es <= STATE_TOL, f"{tag} step {t}: out {eo:.3e} state {es:.3e}"


@pytest.mark.parametrize("engine", ENGINES)
def test_tiny_16_steps(engine):
    shape = I.CONFIGS[0]
    errs, _ = run_parity(I.generate(shape), shape.steps, engine=engine)
    assert len(errs) == 16
    _assert_ok(errs, "tiny")


@pytest.mark.parametrize("engine", ENGINES)
def test_ragged_dk_ne_dv(engine):
    errs, _ = run_parity(I.generate(RAGGED), RAGGED.steps, engine=engine)
    _assert_ok(errs, "ragged")


# dk < dv: 64 key channels, 128 value columns per head (the remaining head shape)
WIDE_V = I.KdaShape("wide_v_b3_h256_2x64x128", batch=3, hidden=256, num_heads=2, head_dk=64, head_dv=128,
                    alpha_rank=32, steps=4, seed=23)


@pytest.mark.parametrize("engine", ENGINES)
def test_dk_lt_dv(engine):
    inp = I.generate(WIDE_V)
    errs, _ = run_parity(inp, WIDE_V.steps, engine=engine)
    _assert_ok(errs, "wide_v")


@pytest.mark.parametrize("cfg", [1, 2])
@pytest.mark.parametrize("engine", ENGINES)
def test_full_size_single_step(cfg, engine):
    shape = I.CONFIGS[cfg]
    errs, _ = run_parity(I.generate(shape), 1, engine=engine)
    _assert_ok(errs, shape.name)


@pytest.mark.parametrize("engine", ENGINES)
def test_batch12_64_steps_in_place(engine):
    shape = I.CONFIGS[3]
    errs, _ = run_parity(I.generate(shape), shape.steps, engine=engine, check_every=8)
    assert len(errs) == 8
    _assert_ok(errs, shape.name)


def test_batch64_hidden6144():
    shape = I.CONFIGS[4]
    errs, _ = run_parity(I.generate(shape), 1)
    _assert_ok(errs, shape.name)


def test_bf16_output():
    shape = I.CONFIGS[1]
    errs, _ = run_parity(I.generate(shape), 1, out_dtype=binding.KDA_OUT_BF16)
    for t, eo, es in errs:
        assert eo <= OUT_TOL + 2.0 ** -9 and es <= STATE_TOL


def test_batch_below_max_batch_leaves_other_rows_untouched():
    import torch
    from linear_attention_layer_kda_b200 import tensors
    shape = I.CONFIGS[1].replace(batch=3)
    inp = I.generate(shape)
    dec = binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, 8)
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    state = torch.full((8, shape.num_heads, shape.head_dk, shape.head_dv), 7.25, device="cuda")
    state[:3] = tensors.state_tensor(inp.state0)
    out = torch.full((8, shape.hidden), -3.5, device="cuda")
    x = torch.zeros(8, shape.hidden, dtype=torch.bfloat16, device="cuda")
    x[:3] = tensors.bf16_tensor(inp.x[0])
    dec.step(x, w, state, out, batch=3)
    dec.sync()
    assert bool((state[3:] == 7.25).all()) and bool((out[3:] == -3.5).all())
    assert not bool((out[:3] == -3.5).any())
    dec.close()


def test_replays_are_bitwise_identical():
    import torch
    from linear_attention_layer_kda_b200 import tensors
    shape = I.CONFIGS[1]
    inp = I.generate(shape)
    dec = binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, 8)
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    x = tensors.bf16_tensor(inp.x[0])
    s0 = tensors.state_tensor(inp.state0)
    out = torch.empty(8, shape.hidden, device="cuda")
    ref_out = ref_state = None
    for _ in range(1000):
        st = s0.clone()
        dec.step(x, w, st, out)
        dec.sync()
        if ref_out is None:
            ref_out, ref_state = out.clone(), st.clone()
        else:
            assert torch.equal(out, ref_out) and torch.equal(st, ref_state)
    dec.close()


def test_pipelined_host_steps_match_device_steps():
    """kda_decode_step_host_async: six steps fed from pinned host buffers without waiting, each
    out copied to its own host buffer, give the device steps' bits (out of every step, state)."""
    import torch
    from linear_attention_layer_kda_b200 import tensors
    shape = I.CONFIGS[1].replace(steps=6)
    inp = I.generate(shape)
    B, H = shape.batch, shape.hidden
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    dec = binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B)
    try:
        s_dev, s_host = tensors.state_tensor(inp.state0), tensors.state_tensor(inp.state0)
        ref = []
        for t in range(shape.steps):
            out = torch.empty(B, H, device="cuda")
            dec.step(tensors.bf16_tensor(inp.x[t]), w, s_dev, out)
            ref.append(out)
        dec.sync()
        xh = [torch.from_numpy(inp.x[t].view(np.int16)).view(torch.bfloat16).pin_memory() for t in range(shape.steps)]
        oh = [torch.full((B, H), float("nan")).pin_memory() for _ in range(shape.steps)]
        for t in range(shape.steps):
            dec.step_host_async(xh[t], w, s_host, oh[t])
        dec.sync()
        for t in range(shape.steps):
            assert torch.equal(oh[t], ref[t].cpu()), f"step {t}"
        assert torch.equal(s_host, s_dev)
    finally:
        dec.close()


def test_host_buffer_entry_point_matches_device_entry_point():
    import torch
    from linear_attention_layer_kda_b200 import tensors
    shape = I.CONFIGS[1]
    inp = I.generate(shape)
    dec = binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, 8)
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    s_dev = tensors.state_tensor(inp.state0)
    s_host = s_dev.clone()
    out = torch.empty(8, shape.hidden, device="cuda")
    dec.step(tensors.bf16_tensor(inp.x[0]), w, s_dev, out)
    dec.sync()
    xh = torch.from_numpy(inp.x[0].view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.empty(8, shape.hidden, dtype=torch.float32).pin_memory()
    dec.step_host(xh, w, s_host, oh)
    assert torch.equal(oh, out.cpu()) and torch.equal(s_host, s_dev)
    dec.close()


def test_invalid_arguments_rejected_before_launch():
    import torch
    from linear_attention_layer_kda_b200 import tensors
    shape = I.CONFIGS[0]
    inp = I.generate(shape, steps=1)
    dec = binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, 1)
    wt = tensors.to_device_weights(inp)
    w = tensors.weights_struct(wt)
    st = tensors.state_tensor(inp.state0)
    out = torch.empty(1, shape.hidden, device="cuda")
    x = tensors.bf16_tensor(inp.x[0])
    with pytest.raises(binding.KdaError) as ei:
        binding.kda_decode_step(dec.h, x.data_ptr(), w, st.data_ptr(), out.data_ptr(), 2)  # batch > max_batch
    assert ei.value.status == binding.KDA_ERR_INVALID_ARG
    with pytest.raises(binding.KdaError):
        binding.kda_decode_step(dec.h, x.data_ptr() + 2, w, st.data_ptr(), out.data_ptr(), 1)  # misaligned x
    with pytest.raises(binding.KdaError):
        binding.kda_decode_step(dec.h, x.data_ptr(), w, st.data_ptr(), st.data_ptr(), 1)  # out aliases state
    w2 = tensors.weights_struct(wt)
    w2.wq = None
    with pytest.raises(binding.KdaError):
        binding.kda_decode_step(dec.h, x.data_ptr(), w2, st.data_ptr(), out.data_ptr(), 1)
    dec.close()


@pytest.mark.parametrize("engine", ENGINES)
def test_stage_intermediates_match_oracle(engine):
    """Block-by-block check of the projection stage: q, k, v, W_b x and W_a_down x."""
    import oracle
    import torch
    from linear_attention_layer_kda_b200 import tensors
    shape = I.CONFIGS[1]
    inp = I.generate(shape)
    dec = binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, 8,
                             engine=engine)
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    st = tensors.state_tensor(inp.state0)
    out = torch.empty(8, shape.hidden, device="cuda")
    dec.step(tensors.bf16_tensor(inp.x[0]), w, st, out)
    dec.sync()
    m = oracle.OracleModel(inp)
    S = inp.state0.astype(np.float64).copy()
    _, dbg = m.step(inp.x[0], S, debug=True)
    bpre_ref = np.log(dbg["beta"] / (1.0 - dbg["beta"]))
    checks = [(binding.KDA_DEBUG_Q, dbg["q"]), (binding.KDA_DEBUG_K, dbg["k"]), (binding.KDA_DEBUG_V, dbg["v"]),
              (binding.KDA_DEBUG_BETA_PRE, bpre_ref), (binding.KDA_DEBUG_T, dbg["t"])]
    for which, ref in checks:
        got = dec.debug_tensor(which, 8).double().cpu().numpy()
        # per 128-row block error, reported on failure
        err = np.abs(got - ref).max() / np.abs(ref).max()
        blocks = [np.abs(got[:, i:i + 128] - ref[:, i:i + 128]).max() for i in range(0, ref.shape[1], 128)]
        assert err < 1e-4, f"debug tensor {which}: max rel err {err:.3e}; per-block abs err {blocks}"
    dec.close()


# ------------------------------------------------------------------ the method's edge cases

def _one_x(inp, steps):
    """Every step and every sequence sees x row 0 of step 0 (the gate weights below saturate
    beta or alpha for that one row); the states of the sequences still differ."""
    x0 = inp.x[0][:1]
    return dataclasses.replace(inp, x=[np.repeat(x0, inp.shape.batch, axis=0) for _ in range(steps)])


def _wide_x(shape, steps):
    """x whose every 128-wide block mixes magnitudes 2^20 apart (odd positions scaled by
    2^-20): the small half falls below the two E4M3 planes' floor, 2^-10 of the block scale."""
    xs = []
    for t in range(steps):
        v = I.bf16_bits_to_f64(I.gen_x(shape, t))
        v[:, 1::2] *= 2.0 ** -20
        xs.append(I.round_to_bf16_bits(v))
    return xs


EDGE_CASES = ["beta0_alpha1", "alpha0", "wk0", "wide_x"]


def _edge_inputs(shape, steps, case):
    inp = I.generate(shape, steps=steps)
    if case == "beta0_alpha1":
        inp = _one_x(inp, steps)
        wb, wd, wu = gate_weights(shape, inp.x[0][0], beta_mode="zero", alpha_mode="one", base=inp)
        return dataclasses.replace(inp, wb=wb, wa_down=wd, wa_up=wu)
    if case == "alpha0":
        inp = _one_x(inp, steps)
        _, wd, wu = gate_weights(shape, inp.x[0][0], alpha_mode="zero", base=inp)
        return dataclasses.replace(inp, wa_down=wd, wa_up=wu)
    if case == "wk0":
        return dataclasses.replace(inp, wk=np.zeros_like(inp.wk))
    return dataclasses.replace(inp, x=_wide_x(shape, steps))


@pytest.mark.parametrize("case", EDGE_CASES)
@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("cfg", [0, 1])
def test_edge_cases_match_oracle(cfg, engine, case):
    """Saturated gates (beta = 0 with alpha = 1; alpha -> 0 at z ~ +3e5), a zero key (W_k = 0,
    so k^ = 0) and wide-range x blocks, through the CUDA path against the oracle."""
    shape = I.CONFIGS[cfg]
    steps = 3 if cfg == 0 else 1
    inp = _edge_inputs(shape, steps, case)
    errs, used, final = run_parity(inp, steps, engine=engine, return_state=True)
    _assert_ok(errs, f"{shape.name} {case}")
    if case == "beta0_alpha1":  # S' = S: the state must come back unchanged
        s0 = inp.state0.astype(np.float64)
        assert np.abs(final - s0).max() <= 1e-6 * np.abs(s0).max()
