"""Shared test helpers: special-case inputs and error metrics (no method arithmetic)."""
import dataclasses

import numpy as np

from linear_attention_layer_kda_b200 import inputs as I

# A small shape with dk != dv and several 128 x 128 scale blocks in every
# direction, so that a transposed operand or a wrong block index shows up.
SMALL = I.KdaShape("small_b2_h256_4x64x32", batch=2, hidden=256, num_heads=4, head_dk=64, head_dv=32,
                   alpha_rank=16, steps=4, seed=11)


def small_inputs(shape=SMALL, **over):
    inp = I.generate(shape)
    return dataclasses.replace(inp, **over) if over else inp


def bf16(v):
    return I.round_to_bf16_bits(np.asarray(v, dtype=np.float64))


def sign_row(x_bits, c):
    """bf16 row c * sign(x): dotted with x gives c * sum |x|."""
    x = I.bf16_bits_to_f64(x_bits)
    return bf16(c * np.sign(x))


def gate_weights(shape, x_bits, beta_mode=None, alpha_mode=None, base=None):
    """(wb, wa_down, wa_up) that drive beta / alpha to exact 0 or 1 for the single x row given.

    beta_mode 'zero' | 'one' | None (keep base), alpha_mode 'one' | 'zero' | None.
    Saturation: sigmoid(-2e4) == 0 and exp(-softplus(-2e4)) == 1 exactly in fp64.
    """
    wb, wa_down, wa_up = (base.wb.copy(), base.wa_down.copy(), base.wa_up.copy()) if base is not None else (None,) * 3
    nh, H, r, Dk = shape.num_heads, shape.hidden, shape.alpha_rank, shape.dk_total
    if beta_mode is not None:
        c = -100.0 if beta_mode == "zero" else 100.0
        wb = np.tile(sign_row(x_bits, c), (nh, 1))
    if alpha_mode is not None:
        wa_down = np.zeros((r, H), dtype=np.uint16)
        wa_down[0] = sign_row(x_bits, 100.0)  # t_0 = 100 * sum|x| > 0
        up = np.zeros((Dk, r))
        up[:, 0] = -1.0 if alpha_mode == "one" else 1.0
        wa_up = bf16(up)
    return wb, wa_down, wa_up


def permuted_fp8(rows, cols, seed):
    """FP8 codes of 448 * P (P a rows x cols partial permutation) with pow2 block scales.

    Returns (codes, scales, perm, mult): row n has its single non-zero in
    column perm[n], with dequantised value mult[n] (exact).
    """
    rng = np.random.default_rng(seed)
    perm = rng.permutation(cols)[:rows] if rows <= cols else rng.integers(0, cols, rows)
    codes = np.zeros((rows, cols), dtype=np.uint8)
    nbr, nbc = -(-rows // 128), -(-cols // 128)
    scales = np.zeros((nbr, nbc), dtype=np.float32)
    for i in range(nbr):
        for j in range(nbc):
            scales[i, j] = 2.0 ** (i + 2 * j - 3)
    codes[np.arange(rows), perm] = 0x7E  # 448
    mult = 448.0 * scales[np.arange(rows) // 128, perm // 128].astype(np.float64)
    return codes, scales, perm, mult


def maxnorm_rel(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / (den if den > 0 else 1.0))
