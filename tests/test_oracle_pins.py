"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
the FP8 E4M3 format definition and torch's float8 cast, library special
functions, exact special cases, and the invariants of the gated delta rule.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from linear_attention_layer_kda_b200 import inputs as I

from helpers import SMALL, bf16, gate_weights, maxnorm_rel, permuted_fp8, small_inputs


# ------------------------------------------------------------------ FP8 / bf16 decode

def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_decode_format_landmarks():
    # OCP 8-bit floating point spec, E4M3: max finite 448 (S.1111.110), min
    # normal 2^-6 (S.0001.000), min subnormal 2^-9 (S.0000.001), 1.0 = 0.0111.000.
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0xFE) == -448.0
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_decode(0x38) == 1.0 and oracle.e4m3_decode(0xB8) == -1.0
    assert oracle.e4m3_decode(0x00) == 0.0 and math.copysign(1, oracle.e4m3_decode(0x80)) < 0
    pos = [oracle.e4m3_decode(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(pos, pos[1:]))  # strictly increasing magnitudes


def test_bf16_widening_all_patterns():
    b = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    sample = np.r_[0:70000:97, 0x3F80, 0x7F7F, 0x0001, 0x8001][:800] % 65536
    for s in sample:
        got = oracle.bf16_to_f64(int(s))
        assert (np.isnan(got) and np.isnan(ref[s])) or got == ref[s]


def test_quantiser_round_trip_bound():
    rng = np.random.default_rng(5)
    w = rng.standard_normal((256, 256)) * 10.0 ** rng.uniform(-4, 1, (256, 256))
    codes, scales = I.quantize_fp8_blocks(w)
    deq = oracle.dequant_fp8(codes, scales)
    s = np.repeat(np.repeat(scales.astype(np.float64), 128, 0), 128, 1)
    err = np.abs(deq - w)
    normal = np.abs(w) / s >= 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(w[normal]) * (1 + 1e-12))
    assert np.all(err[~normal] <= 2.0 ** -10 * s[~normal] * (1 + 1e-12))


def test_quantiser_448_identity_is_exact():
    w = 448.0 * np.eye(256)
    codes, scales = I.quantize_fp8_blocks(w)
    assert np.all(scales[np.eye(2, dtype=bool)] == 1.0)
    assert np.array_equal(oracle.dequant_fp8(codes, scales), w)


# ------------------------------------------------------------------ gates

def test_gate_special_values_and_identity():
    assert oracle.sigmoid(0.0) == 0.5 and oracle.alpha(0.0) == 0.5
    assert oracle.sigmoid(-2e4) == 0.0 and oracle.sigmoid(2e4) == 1.0
    assert oracle.alpha(-2e4) == 1.0 and oracle.alpha(2e4) == 0.0
    for z in np.linspace(-60, 60, 241):
        # exp(-softplus(z)) = 1 / (1 + e^z) = sigmoid(-z)
        assert abs(oracle.alpha(z) - scipy.special.expit(-z)) <= 1e-15 * max(1.0, scipy.special.expit(-z)) + 1e-300
        assert abs(oracle.softplus(z) - np.logaddexp(0.0, z)) <= 1e-14 * max(1.0, abs(z))
        assert abs(oracle.sigmoid(z) - scipy.special.expit(z)) <= 1e-15


# ------------------------------------------------------------------ projections

def _run(inp, shape, x=None, state=None, literal=False):
    m = oracle.OracleModel(inp, batch=shape.batch)
    S = (inp.state0 if state is None else state).astype(np.float64).copy()
    out, dbg = m.step(inp.x[0] if x is None else x, S, literal=literal, debug=True)
    return out, dbg, S


def test_projections_on_scaled_permutations():
    """W = 448 * P with pow2 block scales: every projection is an exact gather of x."""
    shape = SMALL
    base = small_inputs(shape)
    H, Dk, Dv = shape.hidden, shape.dk_total, shape.dv_total
    wq, sq, pq, mq = permuted_fp8(Dk, H, 1)
    wk, sk, pk, mk = permuted_fp8(Dk, H, 2)
    wv, sv, pv, mv = permuted_fp8(Dv, H, 3)
    wo, so, po, mo = permuted_fp8(H, Dv, 4)
    inp = small_inputs(shape, wq=wq, sq=sq, wk=wk, sk=sk, wv=wv, sv=sv, wo=wo, so=so)
    out, dbg, _ = _run(inp, shape)
    x = I.bf16_bits_to_f64(base.x[0])
    assert np.array_equal(dbg["q"], mq * x[:, pq])
    assert np.array_equal(dbg["k"], mk * x[:, pk])
    assert np.array_equal(dbg["v"], mv * x[:, pv])
    assert np.array_equal(out, mo * dbg["o"][:, po])


def test_low_rank_alpha_projection_on_unit_vectors():
    """W_a_down = e_j rows and W_a_up = e_0 columns: t and z are exact copies of x."""
    shape = SMALL.replace(batch=1)
    base = small_inputs(shape)
    r, H, Dk = shape.alpha_rank, shape.hidden, shape.dk_total
    down = np.zeros((r, H)); down[np.arange(r), 3 * np.arange(r) + 1] = 1.0
    up = np.zeros((Dk, r)); up[:, 5] = 0.25
    inp = small_inputs(shape, wa_down=bf16(down), wa_up=bf16(up))
    _, dbg, _ = _run(inp, shape)
    x = I.bf16_bits_to_f64(base.x[0])[0]
    assert np.array_equal(dbg["t"][0], x[3 * np.arange(r) + 1])
    z = 0.25 * x[16]
    assert np.allclose(dbg["alpha"][0], scipy.special.expit(-z), rtol=1e-15, atol=0)


def test_beta_is_sigmoid_of_wb_x():
    shape = SMALL.replace(batch=1)
    base = small_inputs(shape)
    x = I.bf16_bits_to_f64(base.x[0])[0]
    wb = np.zeros((shape.num_heads, shape.hidden)); wb[np.arange(shape.num_heads), [0, 7, 9, 200]] = 1.0
    inp = small_inputs(shape, wb=bf16(wb))
    _, dbg, _ = _run(inp, shape)
    assert np.allclose(dbg["beta"][0], scipy.special.expit(x[[0, 7, 9, 200]]), rtol=1e-15, atol=0)


def test_key_normalisation_and_zero_key():
    shape = SMALL
    inp = small_inputs(shape)
    _, dbg, _ = _run(inp, shape)
    kh = dbg["khat"].reshape(shape.batch, shape.num_heads, shape.head_dk)
    assert np.allclose(np.linalg.norm(kh, axis=-1), 1.0, atol=1e-14)
    k = dbg["k"].reshape(kh.shape)
    assert np.allclose(kh * np.linalg.norm(k, axis=-1, keepdims=True), k, rtol=1e-14, atol=0)
    # W_k = 0: k^ = 0, the update term vanishes and S' = diag(alpha) S exactly
    inp0 = small_inputs(shape, wk=np.zeros_like(inp.wk))
    _, dbg0, S1 = _run(inp0, shape)
    assert np.all(dbg0["khat"] == 0.0)
    a = dbg0["alpha"].reshape(shape.batch, shape.num_heads, shape.head_dk, 1)
    assert np.array_equal(S1, a * inp.state0.astype(np.float64))


# ------------------------------------------------------------------ state update invariants

@pytest.mark.parametrize("literal", [False, True])
def test_invariant_beta0_alpha1_keeps_state(literal):
    shape = SMALL.replace(batch=1)
    base = small_inputs(shape)
    wb, wd, wu = gate_weights(shape, base.x[0][0], beta_mode="zero", alpha_mode="one", base=base)
    inp = small_inputs(shape, wb=wb, wa_down=wd, wa_up=wu)
    out, dbg, S1 = _run(inp, shape, literal=literal)
    assert np.all(dbg["beta"] == 0.0) and np.all(dbg["alpha"] == 1.0)
    S0 = inp.state0.astype(np.float64)
    assert np.array_equal(S1, S0)
    # readout o = S^T q (contracts the key index)
    q = dbg["q"].reshape(shape.num_heads, shape.head_dk)
    o = np.einsum("hij,hi->hj", S0[0], q).reshape(-1)
    assert np.allclose(dbg["o"][0], o, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("literal", [False, True])
def test_invariant_beta1_unit_key_stores_value(literal):
    shape = SMALL.replace(batch=1)
    base = small_inputs(shape)
    wb, _, _ = gate_weights(shape, base.x[0][0], beta_mode="one", base=base)
    inp = small_inputs(shape, wb=wb)
    _, dbg, S1 = _run(inp, shape, literal=literal)
    assert np.all(dbg["beta"] == 1.0)
    assert 0.0 < dbg["alpha"].min() and dbg["alpha"].max() < 1.0
    kh = dbg["khat"].reshape(shape.num_heads, shape.head_dk)
    v = dbg["v"].reshape(shape.num_heads, shape.head_dv)
    Stk = np.einsum("hij,hi->hj", S1[0], kh)
    assert np.allclose(Stk, v, rtol=0, atol=1e-13 * np.abs(v).max())
    # the readout contracts the UPDATED state with q: o = S'^T q.  A readout taken before the
    # update (o = S^T q) differs from it by beta (v - S~^T k^)(k^ . q), which is large here.
    q = dbg["q"].reshape(shape.num_heads, shape.head_dk)
    o = dbg["o"][0].reshape(shape.num_heads, shape.head_dv)
    after = np.einsum("hij,hi->hj", S1[0], q)
    before = np.einsum("hij,hi->hj", inp.state0[0].astype(np.float64), q)
    assert np.allclose(o, after, rtol=0, atol=1e-13 * np.abs(after).max())
    assert np.abs(o - before).max() > 1e-3 * np.abs(after).max()


@pytest.mark.parametrize("literal", [False, True])
def test_invariant_alpha0_forgets_state(literal):
    shape = SMALL.replace(batch=1)
    base = small_inputs(shape)
    _, wd, wu = gate_weights(shape, base.x[0][0], alpha_mode="zero", base=base)
    inp = small_inputs(shape, wa_down=wd, wa_up=wu)
    _, dbg, S1 = _run(inp, shape, literal=literal)
    assert np.all(dbg["alpha"] == 0.0)
    beta = dbg["beta"][0]
    kh = dbg["khat"].reshape(shape.num_heads, shape.head_dk)
    v = dbg["v"].reshape(shape.num_heads, shape.head_dv)
    want = beta[:, None, None] * kh[:, :, None] * v[:, None, :]
    assert np.allclose(S1[0], want, rtol=1e-14, atol=1e-300)
    # with the old state forgotten, the readout after the update is o_h = beta_h v_h (k^_h . q_h)
    # in closed form; a readout before the update would give S_0^T q instead
    q = dbg["q"].reshape(shape.num_heads, shape.head_dk)
    o = dbg["o"][0].reshape(shape.num_heads, shape.head_dv)
    kq = np.einsum("hi,hi->h", kh, q)
    want_o = beta[:, None] * v * kq[:, None]
    assert np.allclose(o, want_o, rtol=0, atol=1e-13 * np.abs(want_o).max())
    before = np.einsum("hij,hi->hj", inp.state0[0].astype(np.float64), q)
    assert np.abs(o - before).max() > 1e-3 * np.abs(want_o).max()


def test_invariant_idempotent_repeat():
    shape = SMALL.replace(batch=1)
    base = small_inputs(shape)
    wb, wd, wu = gate_weights(shape, base.x[0][0], beta_mode="one", alpha_mode="one", base=base)
    inp = small_inputs(shape, wb=wb, wa_down=wd, wa_up=wu)
    m = oracle.OracleModel(inp, batch=1)
    S = inp.state0.astype(np.float64).copy()
    m.step(inp.x[0], S)
    S1 = S.copy()
    m.step(inp.x[0], S)
    assert np.allclose(S, S1, rtol=0, atol=1e-13 * np.abs(S1).max())


def test_invariant_contraction_without_values():
    shape = SMALL
    inp = small_inputs(shape, wv=np.zeros_like(small_inputs(shape).wv))
    out, dbg, S1 = _run(inp, shape)
    S0 = inp.state0.astype(np.float64)
    a = dbg["alpha"].reshape(shape.batch, shape.num_heads, shape.head_dk, 1)
    n1 = np.linalg.norm(S1, axis=(2, 3))
    assert np.all(n1 <= np.linalg.norm(a * S0, axis=(2, 3)) * (1 + 1e-14))
    assert np.all(n1 < np.linalg.norm(S0, axis=(2, 3)))


def test_invariant_scale_x_by_two():
    shape = SMALL
    inp = small_inputs(shape)
    _, d1, _ = _run(inp, shape)
    x2 = bf16(2.0 * I.bf16_bits_to_f64(inp.x[0]))
    _, d2, _ = _run(inp, shape, x=x2)
    for n in ("q", "k", "v", "t"):
        assert np.array_equal(d2[n], 2.0 * d1[n])
    assert np.allclose(d2["khat"], d1["khat"], rtol=0, atol=1e-15)


def test_invariant_unrolled_product_matches_steps():
    """S_T = (prod A_t) S_0 + sum_t (prod_{s>t} A_s) beta_t k^_t v_t^T, A_t = (I - beta_t k^ k^T) diag(alpha_t)."""
    shape = SMALL.replace(batch=1, steps=16)
    inp = small_inputs(shape)
    m = oracle.OracleModel(inp, batch=1)
    S = inp.state0.astype(np.float64).copy()
    S0 = S.copy()
    nh, dk, dv = shape.num_heads, shape.head_dk, shape.head_dv
    As, Us = [], []
    for t in range(shape.steps):
        _, dbg = m.step(inp.x[t], S, debug=True)
        kh = dbg["khat"].reshape(nh, dk)
        b = dbg["beta"][0]
        al = dbg["alpha"].reshape(nh, dk)
        v = dbg["v"].reshape(nh, dv)
        As.append([(np.eye(dk) - b[h] * np.outer(kh[h], kh[h])) @ np.diag(al[h]) for h in range(nh)])
        Us.append([b[h] * np.outer(kh[h], v[h]) for h in range(nh)])
    for h in range(nh):
        P = np.eye(dk)
        acc = np.zeros((dk, dv))
        for t in reversed(range(shape.steps)):
            acc += P @ Us[t][h]
            P = P @ As[t][h]
        ST = P @ S0[0, h] + acc
        assert np.allclose(S[0, h], ST, rtol=0, atol=1e-12 * np.abs(ST).max())


@pytest.mark.parametrize("cfg", [0, 1])
def test_literal_and_rank1_forms_agree(cfg):
    shape = I.CONFIGS[cfg]
    steps = min(shape.steps, 4)
    inp = I.generate(shape, steps=steps)
    m = oracle.OracleModel(inp)
    Sa = inp.state0.astype(np.float64).copy()
    Sb = Sa.copy()
    for t in range(steps):
        oa = m.step(inp.x[t], Sa, literal=True)
        ob = m.step(inp.x[t], Sb, literal=False)
        assert maxnorm_rel(ob, oa) < 1e-12
        assert maxnorm_rel(Sb, Sa) < 1e-12


def test_oracle_golden_tiny():
    """Regression pin of the oracle on the tiny workload (tests/golden/make_golden.py writes the file)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle_out.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    shape = I.CONFIGS[0]
    inp = I.generate(shape)
    m = oracle.OracleModel(inp)
    S = inp.state0.astype(np.float64).copy()
    outs = [m.step(inp.x[t], S) for t in range(shape.steps)]
    for step, idx, val in rows:
        if step == "state_sum":
            assert abs(S.sum() - float(val)) <= 1e-12 * abs(float(val)) + 1e-15
        else:
            got = outs[int(step)][0, int(idx)]
            assert abs(got - float(val)) <= 1e-13 * max(1.0, abs(float(val)))
