"""The chunked (parallel-in-time) form of the gated delta rule equals the token-by-token
recurrence of the oracle.  Groundwork for a chunked prefill, where a chunk of C tokens is
processed with dense C x C and C x dk products instead of C sequential rank-1 updates.

Per head, inside a chunk that starts from state S0 (dk x dv), with g_t the running product
of alpha over the chunk's tokens 1..t (a diagonal over key channels):
    S_t = diag(g_t) S0 + sum_{i<=t} diag(g_t / g_i) k_i u_i^T
    u_t = beta_t (v_t - S0^T (g_t k_t) - sum_{i<t} u_i (k_i^T diag(g_t / g_i) k_t))
so (I + A) U = diag(beta) (V - (G K) S0) with A strictly lower triangular,
A[t, i] = beta_t k_i^T diag(g_t / g_i) k_t, and the readout after token t is
    o_t = S0^T (g_t q_t) + sum_{i<=t} u_i (k_i^T diag(g_t / g_i) q_t).
(k is the L2-normalised key.)  Derived from the recurrence by unrolling it over the chunk.
"""
import numpy as np
import pytest

import oracle
from linear_attention_layer_kda_b200 import inputs as I


def chunk_step(S0, q, k, v, beta, alpha):
    """One chunk for one head: q, k, alpha [C, dk]; v [C, dv]; beta [C]. Returns (O [C, dv], S_C)."""
    C = q.shape[0]
    g = np.cumprod(alpha, axis=0)                      # g_t, [C, dk]
    ratio = g[:, None, :] / g[None, :, :]              # g_t / g_i, [t, i, dk] (used for i <= t)
    kk = np.einsum("id,tid,td->ti", k, ratio, k)       # k_i^T diag(g_t/g_i) k_t
    kq = np.einsum("id,tid,td->ti", k, ratio, q)       # k_i^T diag(g_t/g_i) q_t
    A = np.tril(beta[:, None] * kk, -1)
    rhs = beta[:, None] * (v - (g * k) @ S0)
    U = np.linalg.solve(np.eye(C) + A, rhs)            # unit lower triangular system
    O = (g * q) @ S0 + np.tril(kq) @ U
    S = g[-1][:, None] * S0 + (k * (g[-1][None, :] / g)).T @ U
    return O, S


SHAPES = [I.CONFIGS[0],  # batch 1, hidden 256, 2 heads of 64 x 64, 16 steps
          I.KdaShape("chunk_dk_lt_dv", batch=1, hidden=256, num_heads=2, head_dk=64, head_dv=128,
                     alpha_rank=32, steps=12, seed=31),
          I.KdaShape("chunk_dk_gt_dv", batch=1, hidden=384, num_heads=2, head_dk=128, head_dv=64,
                     alpha_rank=32, steps=12, seed=32)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
@pytest.mark.parametrize("C", [1, 4, 5, 16])
def test_chunked_form_matches_the_recurrence(C, shape):
    T, nh, dk, dv = shape.steps, shape.num_heads, shape.head_dk, shape.head_dv
    inp = I.generate(shape)
    m = oracle.OracleModel(inp, batch=1)
    S = inp.state0.astype(np.float64).copy()
    S_init = S.copy()
    rec = {n: [] for n in ("q", "khat", "v", "beta", "alpha", "o")}
    for t in range(T):
        _, d = m.step(inp.x[t], S, debug=True)
        for n in rec:
            rec[n].append(d[n][0])
    m.close()
    for h in range(nh):
        q = np.array([a[h * dk:(h + 1) * dk] for a in rec["q"]])
        k = np.array([a[h * dk:(h + 1) * dk] for a in rec["khat"]])
        al = np.array([a[h * dk:(h + 1) * dk] for a in rec["alpha"]])
        v = np.array([a[h * dv:(h + 1) * dv] for a in rec["v"]])
        o_ref = np.array([a[h * dv:(h + 1) * dv] for a in rec["o"]])
        beta = np.array([a[h] for a in rec["beta"]])
        Sh = S_init[0, h].copy()
        outs = []
        for c0 in range(0, T, C):
            c1 = min(T, c0 + C)
            O, Sh = chunk_step(Sh, q[c0:c1], k[c0:c1], v[c0:c1], beta[c0:c1], al[c0:c1])
            outs.append(O)
        O = np.concatenate(outs)
        assert np.abs(O - o_ref).max() <= 1e-11 * np.abs(o_ref).max()
        assert np.abs(Sh - S[0, h]).max() <= 1e-11 * np.abs(S[0, h]).max()
