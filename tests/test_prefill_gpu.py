"""Chunked prefill (kda_prefill) against the fp64 oracle applied token by token.

The chunked form must reproduce the recurrence: every token's output within the decode
tolerance (max-norm relative error <= 2e-3 over each token's outputs) and the final state
within 1e-3, for prompts of 64 to 4096 tokens, chunks of 16, 32 and 64, a last chunk that
is only partly filled, dk != dv, and saturated decay (alpha = 0, the state forgotten at every
token), which the kernel's log-space decays must handle without overflow.
"""
import dataclasses

import numpy as np
import pytest

from linear_attention_layer_kda_b200 import binding, inputs as I

from gpu_util import OUT_TOL, STATE_TOL, maxrel
from helpers import gate_weights

pytestmark = pytest.mark.gpu

RAGGED = I.KdaShape("ragged_b2_h384_2x128x64", batch=2, hidden=384, num_heads=2, head_dk=128, head_dv=64,
                    alpha_rank=32, steps=1, seed=51)
FULL = I.CONFIGS[2]  # hidden 4096, 32 heads of 128 x 128, one sequence


def _prefill(inp, shape, T, chunk):
    import torch
    from linear_attention_layer_kda_b200 import tensors
    B, H = shape.batch, shape.hidden
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    xs = tensors.bf16_tensor(np.stack([inp.x[t] for t in range(T)], axis=1).reshape(B * T, H))
    dec = binding.KdaDecoder(H, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B)
    try:
        st = tensors.state_tensor(inp.state0)
        out = torch.full((B * T, H), float("nan"), device="cuda")
        dec.prefill(xs, w, st, out, B, T, chunk)
        dec.sync()
        return out.view(B, T, H).double().cpu().numpy(), st.double().cpu().numpy()
    finally:
        dec.close()


def _oracle(inp, shape, T):
    import oracle
    B = shape.batch
    m = oracle.OracleModel(inp, batch=B)
    try:
        S = inp.state0.astype(np.float64).copy()
        outs = np.stack([m.step(inp.x[t], S) for t in range(T)], axis=1)  # [B, T, H]
        return outs, S
    finally:
        m.close()


def _check(got_out, got_state, ref_out, ref_state, T):
    worst = max(maxrel(got_out[:, t], ref_out[:, t]) for t in range(T))
    es = maxrel(got_state, ref_state)
    assert worst <= OUT_TOL, f"out error {worst:.3e}"
    assert es <= STATE_TOL, f"state error {es:.3e}"


WIDE_V = I.KdaShape("wide_v_b3_h256_2x64x128", batch=3, hidden=256, num_heads=2, head_dk=64, head_dv=128,
                    alpha_rank=32, steps=1, seed=53)
CASES = [(I.CONFIGS[0], 64, 16), (I.CONFIGS[0], 64, 64), (I.CONFIGS[0], 4096, 64), (I.CONFIGS[0], 1000, 32),
         (RAGGED, 100, 32), (RAGGED, 77, 16), (WIDE_V, 90, 16), (WIDE_V, 90, 64), (FULL, 256, 32), (FULL, 2048, 64)]


@pytest.mark.parametrize("shape,T,chunk", CASES, ids=[f"{s.name}_T{t}_C{c}" for s, t, c in CASES])
def test_prefill_matches_the_recurrence(shape, T, chunk):
    inp = I.generate(shape.replace(steps=T))
    got_out, got_state = _prefill(inp, shape, T, chunk)
    ref_out, ref_state = _oracle(inp, shape, T)
    _check(got_out, got_state, ref_out, ref_state, T)


def test_prefill_with_alpha_zero_forgets_at_every_token():
    """z = +3e5 on every channel: log alpha is clamped, gamma(t, i) is 0 across tokens."""
    shape = I.CONFIGS[0]
    T = 48
    inp = I.generate(shape.replace(steps=T))
    x0 = inp.x[0][:1]
    inp = dataclasses.replace(inp, x=[x0.copy() for _ in range(T)])
    _, wd, wu = gate_weights(shape, x0[0], alpha_mode="zero", base=inp)
    inp = dataclasses.replace(inp, wa_down=wd, wa_up=wu)
    got_out, got_state = _prefill(inp, shape, T, 16)
    ref_out, ref_state = _oracle(inp, shape, T)
    _check(got_out, got_state, ref_out, ref_state, T)


def test_chunk_sizes_agree():
    shape = RAGGED
    T = 96
    inp = I.generate(shape.replace(steps=T))
    res = [_prefill(inp, shape, T, c) for c in (16, 32, 64)]
    for o, s in res[1:]:
        assert maxrel(o, res[0][0]) <= 1e-4 and maxrel(s, res[0][1]) <= 1e-4


def test_prefill_bf16_out_and_growing_workspace():
    """bf16 out (the output GEMMs sum in fp32, then one rounding) and one handle whose workspace
    grows between calls: a short prompt, then a longer one continuing the same state."""
    import torch
    from linear_attention_layer_kda_b200 import tensors
    shape = RAGGED
    T1, T2 = 40, 200
    inp = I.generate(shape.replace(steps=T1 + T2))
    B, H = shape.batch, shape.hidden
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    dec = binding.KdaDecoder(H, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B,
                             out_dtype=binding.KDA_OUT_BF16)
    ref_out, ref_state = _oracle(inp, shape, T1 + T2)
    try:
        st = tensors.state_tensor(inp.state0)
        got = []
        for t0, T in ((0, T1), (T1, T2)):
            xs = tensors.bf16_tensor(np.stack([inp.x[t] for t in range(t0, t0 + T)], axis=1).reshape(B * T, H))
            out = torch.full((B * T, H), float("nan"), device="cuda", dtype=torch.bfloat16)
            dec.prefill(xs, w, st, out, B, T, 32)
            dec.sync()
            got.append(out.view(B, T, H).double().cpu().numpy())
        got_out = np.concatenate(got, axis=1)
        worst = max(maxrel(got_out[:, t], ref_out[:, t]) for t in range(T1 + T2))
        assert worst <= OUT_TOL + 2.0 ** -9, f"out error {worst:.3e}"
        assert maxrel(st.double().cpu().numpy(), ref_state) <= STATE_TOL
    finally:
        dec.close()


def test_prefill_argument_errors():
    import ctypes
    s = I.CONFIGS[0]
    dec = binding.KdaDecoder(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank, 1)
    try:
        lib = binding.load()
        w = binding.kda_weights()
        for n in binding.WEIGHT_FIELDS:
            setattr(w, n, 1 << 40)
        bad = [(1, 0, 16), (0, 4, 16), (1, 4, 8), (1, 4, 128)]
        for batch, tokens, chunk in bad:
            assert lib.kda_prefill(dec.h, 1 << 41, ctypes.byref(w), 1 << 42, 1 << 43, batch, tokens, chunk) == \
                binding.KDA_ERR_INVALID_ARG
    finally:
        dec.close()
