"""fp64 CPU oracle of the KDA decode step (ctypes front end of kda_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product path (the CUDA
library and its binding) never imports this package.

The arithmetic lives in ``kda_oracle.c`` (plain C, fp64); this module only
builds it with gcc, marshals numpy arrays and exposes:

* ``e4m3_decode(code)``             -- closed-form FP8 E4M3 value
* ``alpha(z)``, ``sigmoid(a)``      -- the gates
* ``OracleModel(inputs)``           -- dequantised fp64 weights
* ``OracleModel.step(x, state)``    -- one decode step, literal or rank-1 form
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile kda_oracle.c into libkda_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
                               "-shared", "-std=c99", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("hidden", ctypes.c_int), ("num_heads", ctypes.c_int),
                ("head_dk", ctypes.c_int), ("head_dv", ctypes.c_int), ("alpha_rank", ctypes.c_int)]


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        _lib.kda_oracle_e4m3_decode.restype = ctypes.c_double
        _lib.kda_oracle_e4m3_decode.argtypes = [ctypes.c_uint]
        _lib.kda_oracle_bf16_to_f64.restype = ctypes.c_double
        _lib.kda_oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        for f in ("kda_oracle_sigmoid", "kda_oracle_softplus", "kda_oracle_alpha"):
            getattr(_lib, f).restype = ctypes.c_double
            getattr(_lib, f).argtypes = [ctypes.c_double]
        _lib.kda_oracle_dequant_fp8.restype = None
        _lib.kda_oracle_dequant_fp8.argtypes = [P, P, ctypes.c_int, ctypes.c_int, P]
        _lib.kda_oracle_model_new.restype = P
        _lib.kda_oracle_model_new.argtypes = [ctypes.POINTER(_Dims)] + [P] * 11
        _lib.kda_oracle_model_free.restype = None
        _lib.kda_oracle_model_free.argtypes = [P]
        _lib.kda_oracle_step.restype = ctypes.c_int
        _lib.kda_oracle_step.argtypes = [P, P, P, P, ctypes.c_int, P]
        _lib.kda_oracle_num_threads.restype = ctypes.c_int
        _lib.kda_oracle_set_num_threads.argtypes = [ctypes.c_int]
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def e4m3_decode(code: int) -> float:
    return lib().kda_oracle_e4m3_decode(int(code))


def bf16_to_f64(bits: int) -> float:
    return lib().kda_oracle_bf16_to_f64(int(bits))


def sigmoid(a: float) -> float:
    return lib().kda_oracle_sigmoid(float(a))


def softplus(z: float) -> float:
    return lib().kda_oracle_softplus(float(z))


def alpha(z: float) -> float:
    return lib().kda_oracle_alpha(float(z))


def dequant_fp8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    out = np.empty(codes.shape, dtype=np.float64)
    lib().kda_oracle_dequant_fp8(_ptr(codes), _ptr(scales), codes.shape[0], codes.shape[1], _ptr(out))
    return out


def num_threads() -> int:
    return lib().kda_oracle_num_threads()


def set_num_threads(n: int) -> None:
    lib().kda_oracle_set_num_threads(int(n))


class OracleModel:
    """Dequantised fp64 weights of one workload; ``step`` runs the decode step."""

    def __init__(self, inp, batch: Optional[int] = None):
        s = inp.shape
        self.shape = s
        self.batch = s.batch if batch is None else batch
        self._keep = [np.ascontiguousarray(a) for a in (inp.wq, inp.sq, inp.wk, inp.sk, inp.wv, inp.sv, inp.wo,
                                                         inp.so, inp.wa_down, inp.wa_up, inp.wb)]
        self._dims = _Dims(self.batch, s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank)
        h = lib().kda_oracle_model_new(ctypes.byref(self._dims), *[_ptr(a) for a in self._keep])
        if not h:
            raise MemoryError("oracle: cannot allocate the fp64 weights")
        self._h = h

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().kda_oracle_model_free(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @property
    def dbg_width(self) -> int:
        s = self.shape
        return 4 * s.dk_total + 2 * s.dv_total + s.num_heads + s.alpha_rank

    def step(self, x_bits: np.ndarray, state: np.ndarray, literal: bool = False, debug: bool = False):
        """One step.  ``state`` (fp64 [B, nh, dk, dv]) is updated in place.

        Returns out [B, H] fp64, and with ``debug`` also a dict of the
        per-sequence intermediates (q, khat, v, beta, alpha, o, t, k).
        """
        s = self.shape
        x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(self.batch, s.hidden)
        assert state.dtype == np.float64 and state.flags["C_CONTIGUOUS"]
        assert state.shape == (self.batch, s.num_heads, s.head_dk, s.head_dv)
        out = np.empty((self.batch, s.hidden), dtype=np.float64)
        dbg = np.empty((self.batch, self.dbg_width), dtype=np.float64) if debug else None
        rc = lib().kda_oracle_step(self._h, _ptr(x_bits), _ptr(state), _ptr(out), int(bool(literal)),
                                   _ptr(dbg) if dbg is not None else None)
        if rc != 0:
            raise MemoryError("oracle: step failed to allocate")
        if not debug:
            return out
        Dk, Dv, nh, r = s.dk_total, s.dv_total, s.num_heads, s.alpha_rank
        names = [("q", Dk), ("khat", Dk), ("v", Dv), ("beta", nh), ("alpha", Dk), ("o", Dv), ("t", r), ("k", Dk)]
        parts, c = {}, 0
        for n, w in names:
            parts[n] = dbg[:, c:c + w].copy()
            c += w
        return out, parts
