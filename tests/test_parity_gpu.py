"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances are the decode benchmark's: max-norm relative error <= 2e-3 on
out and <= 1e-3 on the updated state, every checked step.
"""
import numpy as np
import pytest

from linear_attention_layer_kda_b200 import binding, inputs as I

from gpu_util import OUT_TOL, STATE_TOL, run_parity

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
    for _ in range(50):
        st = s0.clone()
        dec.step(x, w, st, out)
        dec.sync()
        if ref_out is None:
            ref_out, ref_state = out.clone(), st.clone()
        else:
            assert torch.equal(out, ref_out) and torch.equal(st, ref_state)
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
