"""Pins of the seeded input generator (no GPU, no oracle arithmetic)."""
from fractions import Fraction
import hashlib
import math
import struct

import numpy as np
import pytest
import torch

from linear_attention_layer_kda_b200 import inputs as I


def test_splitmix64_published_vector():
    # splitmix64 (Steele, Lea & Flood 2014) from raw state 1234567: the first
    # five outputs of the reference C implementation.
    key = 1234567
    i = np.arange(5, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (i + np.uint64(1)) * I._GAMMA
        got = [int(v) for v in I._mix64(z)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_streams_deterministic_and_independent():
    a = I.normal(I.stream_key(7, I.TAG_X), 0, 1000)
    b = I.normal(I.stream_key(7, I.TAG_X), 0, 1000)
    c = I.normal(I.stream_key(7, I.TAG_WQ), 0, 1000)
    d = I.normal(I.stream_key(8, I.TAG_X), 0, 1000)
    assert np.array_equal(a, b)
    assert not np.array_equal(a, c) and not np.array_equal(a, d)
    # counter-based: any window regenerates the same values
    assert np.array_equal(I.normal(I.stream_key(7, I.TAG_X), 300, 200), a[300:500])


def test_normal_moments():
    v = I.normal(I.stream_key(3, I.TAG_STATE), 0, 1 << 20)
    assert abs(v.mean()) < 5e-3
    assert abs(v.std() - 1.0) < 5e-3
    # fraction beyond 2 sigma of a standard normal: 0.0455
    assert abs(np.mean(np.abs(v) > 2.0) - 0.0455) < 2e-3


def _bf16_exact_rne(v: float) -> float:
    """Round v to bf16 by exhaustive neighbour search on exact rationals."""
    if v == 0.0:
        return 0.0
    f = Fraction(v)
    e = math.floor(math.log2(abs(v)))
    q = Fraction(2) ** (max(e, -126) - 7)
    n = f / q
    lo = math.floor(n)
    r = n - lo
    k = lo + (1 if (r > Fraction(1, 2) or (r == Fraction(1, 2) and lo % 2 == 1)) else 0)
    return float(k * q)


def test_bf16_rounding_is_single_rne():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000), [1.0, -2.5, 3.0e38]])
    bits = I.round_to_bf16_bits(v)
    got = I.bf16_bits_to_f64(bits)
    want = np.array([_bf16_exact_rne(float(a)) for a in v])
    assert np.array_equal(got, want)
    # ties go to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    assert I.round_to_bf16_bits(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80
    assert I.round_to_bf16_bits(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 0x3F82


def test_e4m3_encode_matches_torch_cast_on_fp32_values():
    # torch's fp32 -> float8_e4m3fn cast is RNE; on fp32-exact inputs inside
    # the finite range both must give the same code.
    rng = np.random.default_rng(1)
    v = np.concatenate([np.linspace(-448, 448, 40001), rng.standard_normal(20000) * 1e-2,
                        rng.standard_normal(20000) * 30.0]).astype(np.float32).astype(np.float64)
    ours = I.e4m3_encode(v)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)
    assert I.e4m3_encode(np.array([1e6, -1e6]))[0] == 0x7E  # saturates
    assert I.e4m3_encode(np.array([-1e6]))[0] == 0xFE


def test_block_quantiser_scales():
    w = np.zeros((256, 384))
    w[:128, :128] = 3.0
    w[130, 200] = -448.0 * 4.0
    codes, scales = I.quantize_fp8_blocks(w)
    assert scales.shape == (2, 3)
    assert scales[0, 0] == np.float32(3.0 / 448.0)
    assert scales[1, 1] == np.float32(4.0)
    assert scales[0, 2] == 1.0  # all-zero block
    assert codes[130, 200] == 0xFE and codes[0, 0] == 0x7E


def test_config_shapes_and_distributions():
    s = I.CONFIGS[0]
    inp = I.generate(s)
    assert inp.x.shape == (16, 1, 256) and inp.x.dtype == np.uint16
    assert inp.wq.shape == (128, 256) and inp.sq.shape == (1, 2)
    assert inp.wo.shape == (256, 128) and inp.so.shape == (2, 1)
    assert inp.wa_down.shape == (64, 256) and inp.wa_up.shape == (128, 64) and inp.wb.shape == (2, 256)
    assert inp.state0.shape == (1, 2, 64, 64) and inp.state0.dtype == np.float32
    assert abs(inp.state0.std() - 0.02) < 2e-3
    wb = I.bf16_bits_to_f64(inp.wb)
    assert abs(wb.std() - 1 / 16) < 8e-3
    # per-step x draws are fresh and reproducible row by row
    assert not np.array_equal(inp.x[0], inp.x[1])
    assert np.array_equal(I.gen_x(s, 3), inp.x[3])


def test_generator_golden_hash():
    """Regression pin: SHA-256 of the tiny workload's bytes (written by tests/golden/make_golden.py)."""
    inp = I.generate(I.CONFIGS[0])
    h = hashlib.sha256()
    for a in (inp.x, inp.wq, inp.sq, inp.wk, inp.sk, inp.wv, inp.sv, inp.wo, inp.so, inp.wa_down, inp.wa_up,
              inp.wb, inp.state0):
        h.update(np.ascontiguousarray(a).tobytes())
    with open(__file__.replace("test_inputs.py", "golden/tiny_inputs.sha256")) as f:
        want = [ln.split()[0] for ln in f if ln.strip() and not ln.startswith("#")][0]
    assert h.hexdigest() == want
