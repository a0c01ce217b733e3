"""Seeded synthetic inputs for the KDA decode step.

This module only *makes* inputs: a counter-based random generator, rounding of
fp64 draws to bf16 / fp32, and the FP8 E4M3 block quantiser that turns fp64
weight draws into (codes, fp32 block scales).  It holds none of the decode
step's arithmetic (no FP8 decoding, no projections, gates or state update), so
both the fp64 oracle and the CUDA path can consume the same bytes without
sharing any of the method's code.

Workloads follow the decode regime the pages describe (Kiln, "The decode
kernels, and why they are opt-in": a per-sequence recurrent state updated in
place; TrnRT story: batch-8 decode step; TrnRT listing: batch-12 serving
point) with the distributions the workload table fixes:

* x ~ N(0, 1) rounded to bf16 (round-to-nearest-even; Kiln, "The
  hyper-connection arithmetic ..." uses RNE for bf16),
* every weight matrix ~ N(0, std = 1/sqrt(fan_in)),
* q/k/v/out weights quantised to FP8 E4M3 with one fp32 scale per 128x128
  block (Kiln, "How was Kiln measured": FP8 weights in 128 x 128 blocks),
  scale = amax / 448, code = RNE(w / scale) saturated to +-448,
* alpha (low rank) and beta gate weights in bf16,
* initial state ~ N(0, std 0.02) rounded to fp32.

Random numbers: splitmix64 (Steele, Lea & Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) used as a counter-based
generator.  Value i of a stream with key K is mix64(K + (i + 1) * gamma); the
key of tensor ``tag`` under ``seed`` is mix64(seed * gamma + tag).  Uniform
doubles take the top 53 bits; normals use Box-Muller on the uniform pair
(2i, 2i + 1), keeping the cosine branch, so element i of any tensor can be
regenerated on its own.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1

# tensor tags: one independent stream per tensor
TAG_X, TAG_WQ, TAG_WK, TAG_WV, TAG_WO, TAG_WA_DOWN, TAG_WA_UP, TAG_WB, TAG_STATE = range(1, 10)

FP8_E4M3_MAX = 448.0
SCALE_BLOCK = 128


@dataclasses.dataclass(frozen=True)
class KdaShape:
    """Dimensions of one KDA decode workload."""

    name: str
    batch: int
    hidden: int
    num_heads: int
    head_dk: int
    head_dv: int
    alpha_rank: int
    steps: int
    seed: int

    @property
    def dk_total(self) -> int:  # rows of W_q, W_k, W_a_up
        return self.num_heads * self.head_dk

    @property
    def dv_total(self) -> int:  # rows of W_v, columns of W_o
        return self.num_heads * self.head_dv

    def replace(self, **kw) -> "KdaShape":
        return dataclasses.replace(self, **kw)


# The five workloads of the decode benchmark (tiny parity case, batch 8,
# batch 1 latency, batch 12 with 64 in-place steps, batch 64 at hidden 6144).
CONFIGS: Dict[int, KdaShape] = {
    0: KdaShape("tiny_b1_h256_2x64_16steps", 1, 256, 2, 64, 64, 64, 16, 0),
    1: KdaShape("b8_h4096_32x128", 8, 4096, 32, 128, 128, 64, 1, 1),
    2: KdaShape("b1_h4096_32x128", 1, 4096, 32, 128, 128, 64, 1, 2),
    3: KdaShape("b12_h4096_32x128_64steps", 12, 4096, 32, 128, 128, 64, 64, 3),
    4: KdaShape("b64_h6144_48x128", 64, 6144, 48, 128, 128, 64, 1, 4),
}


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tag: int) -> int:
    z = np.array([(seed * int(_GAMMA) + tag) & _MASK64], dtype=np.uint64)
    with np.errstate(over="ignore"):
        return int(_mix64(z)[0])


def uniform53(key: int, start: int, n: int) -> np.ndarray:
    """Uniform doubles in [0, 1): values start .. start+n-1 of stream ``key``."""
    i = np.arange(start, start + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + (i + np.uint64(1)) * _GAMMA
        u = _mix64(z) >> np.uint64(11)
    return u.astype(np.float64) * (1.0 / 9007199254740992.0)


def normal(key: int, start: int, n: int, chunk: int = 1 << 22) -> np.ndarray:
    """Standard normals start .. start+n-1 of stream ``key`` (Box-Muller)."""
    out = np.empty(n, dtype=np.float64)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        u = uniform53(key, 2 * (start + c0), 2 * (c1 - c0))
        u1 = 1.0 - u[0::2]  # (0, 1]
        u2 = u[1::2]
        out[c0:c1] = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)
    return out


def round_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns (uint16), round to nearest even, one rounding."""
    v = np.asarray(v, dtype=np.float64)
    _, ex = np.frexp(v)
    quantum = np.ldexp(1.0, np.maximum(ex, -125) - 8)
    r = np.rint(v / quantum) * quantum  # exact in fp64; representable in fp32
    bits = r.astype(np.float32).view(np.uint32)
    return (bits >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """fp64 -> FP8 E4M3 ("fn": bias 7, no infinities) codes, RNE, saturating at 448."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v)
    a = np.minimum(np.abs(v), FP8_E4M3_MAX)
    _, ex = np.frexp(a)
    e = ex.astype(np.int64) - 1  # floor(log2 a) for a > 0
    sub = e < -6
    # normal: code = (e + 7) * 8 + RNE(a * 2^(3 - e)) - 8 ; a mantissa carry moves into the exponent field
    e_n = np.where(sub, 0, e)
    normal_code = (e_n + 7) * 8 + np.rint(np.ldexp(a, 3 - e_n)).astype(np.int64) - 8
    sub_code = np.rint(np.ldexp(a, 9)).astype(np.int64)  # multiples of 2^-9; 8 -> first normal
    code = np.where(a == 0.0, 0, np.where(sub, sub_code, normal_code))
    code = np.minimum(code, 0x7E)  # saturate (448)
    return (code | (sign.astype(np.int64) << 7)).astype(np.uint8)


def quantize_fp8_blocks(w: np.ndarray, block: int = SCALE_BLOCK):
    """Block-scaled FP8 E4M3: one fp32 scale per ``block`` x ``block`` tile.

    Returns (codes uint8 [R, C], scales float32 [ceil(R/block), ceil(C/block)]),
    with dequantised value = decode(code) * scale.
    """
    w = np.asarray(w, dtype=np.float64)
    R, C = w.shape
    nbr, nbc = -(-R // block), -(-C // block)
    scales = np.empty((nbr, nbc), dtype=np.float32)
    codes = np.empty((R, C), dtype=np.uint8)
    for i in range(nbr):
        r0, r1 = i * block, min(R, (i + 1) * block)
        for j in range(nbc):
            c0, c1 = j * block, min(C, (j + 1) * block)
            blk = w[r0:r1, c0:c1]
            amax = float(np.max(np.abs(blk))) if blk.size else 0.0
            s = np.float32(amax / FP8_E4M3_MAX) if amax > 0.0 else np.float32(1.0)
            if s == 0.0:  # amax below the fp32 range of amax/448
                s = np.float32(np.finfo(np.float32).tiny)
            scales[i, j] = s
            codes[r0:r1, c0:c1] = e4m3_encode(blk / np.float64(s))
    return codes, scales


@dataclasses.dataclass
class KdaInputs:
    """Host copies of one workload: weights, initial state and per-step x."""

    shape: KdaShape
    x: np.ndarray  # uint16 bf16 bits [steps, B, H]
    wq: np.ndarray  # uint8 [nh*dk, H]
    sq: np.ndarray  # float32 [nh*dk/128, H/128]
    wk: np.ndarray
    sk: np.ndarray
    wv: np.ndarray  # uint8 [nh*dv, H]
    sv: np.ndarray
    wo: np.ndarray  # uint8 [H, nh*dv]
    so: np.ndarray
    wa_down: np.ndarray  # uint16 bf16 [r, H]
    wa_up: np.ndarray  # uint16 bf16 [nh*dk, r]
    wb: np.ndarray  # uint16 bf16 [nh, H]
    state0: np.ndarray  # float32 [B, nh, dk, dv]


def gen_x(shape: KdaShape, step: int, batch: Optional[int] = None, row0: int = 0) -> np.ndarray:
    """bf16 bits of x for one step: rows row0 .. row0+batch-1 of that step's [B, H] draw."""
    B = shape.batch if batch is None else batch
    H = shape.hidden
    key = stream_key(shape.seed, TAG_X)
    start = step * shape.batch * H + row0 * H
    return round_to_bf16_bits(normal(key, start, B * H)).reshape(B, H)


def _fp8_weight(shape: KdaShape, tag: int, rows: int, cols: int, fan_in: int):
    w = normal(stream_key(shape.seed, tag), 0, rows * cols).reshape(rows, cols) / np.sqrt(fan_in)
    return quantize_fp8_blocks(w)


def _bf16_weight(shape: KdaShape, tag: int, rows: int, cols: int, fan_in: int) -> np.ndarray:
    w = normal(stream_key(shape.seed, tag), 0, rows * cols).reshape(rows, cols) / np.sqrt(fan_in)
    return round_to_bf16_bits(w)


def gen_state(shape: KdaShape, batch: Optional[int] = None, row0: int = 0) -> np.ndarray:
    B = shape.batch if batch is None else batch
    per_seq = shape.num_heads * shape.head_dk * shape.head_dv
    v = normal(stream_key(shape.seed, TAG_STATE), row0 * per_seq, B * per_seq) * 0.02
    return v.astype(np.float32).reshape(B, shape.num_heads, shape.head_dk, shape.head_dv)


def generate(shape: KdaShape, steps: Optional[int] = None) -> KdaInputs:
    """All inputs of ``shape`` (x for ``steps`` steps, default shape.steps)."""
    T = shape.steps if steps is None else steps
    H, r, nh = shape.hidden, shape.alpha_rank, shape.num_heads
    Dk, Dv = shape.dk_total, shape.dv_total
    x = np.stack([gen_x(shape, t) for t in range(T)])
    wq, sq = _fp8_weight(shape, TAG_WQ, Dk, H, H)
    wk, sk = _fp8_weight(shape, TAG_WK, Dk, H, H)
    wv, sv = _fp8_weight(shape, TAG_WV, Dv, H, H)
    wo, so = _fp8_weight(shape, TAG_WO, H, Dv, Dv)
    wa_down = _bf16_weight(shape, TAG_WA_DOWN, r, H, H)
    wa_up = _bf16_weight(shape, TAG_WA_UP, Dk, r, r)
    wb = _bf16_weight(shape, TAG_WB, nh, H, H)
    return KdaInputs(shape, x, wq, sq, wk, sk, wv, sv, wo, so, wa_down, wa_up, wb, gen_state(shape))
