"""ctypes binding of libkda_decode.so (include/kda_decode.h).

Argument marshalling only: every step of the decode path runs in the CUDA
library.  The functions keep the C names; a non-zero status raises KdaError.
``KdaDecoder`` is a small convenience wrapper that takes torch tensors and
binds torch's current CUDA stream.  If the library is missing the first call
raises: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libkda_decode.so")

KDA_OK = 0
KDA_ERR_INVALID_ARG = 1
KDA_ERR_UNSUPPORTED_SHAPE = 2
KDA_ERR_CUDA = 3
KDA_ERR_DEVICE_TIMEOUT = 4
KDA_ERR_NO_DEVICE = 5
KDA_ERR_OUT_OF_MEMORY = 6
KDA_OUT_F32 = 0
KDA_OUT_BF16 = 1
KDA_ENGINE_AUTO = 0
KDA_ENGINE_SIMPLE = 1
KDA_ENGINE_FUSED = 2

# every symbol include/kda_decode.h declares
EXPORTS = (
    "kda_decode_init", "kda_decode_set_stream", "kda_decode_step", "kda_decode_step_host", "kda_decode_sync",
    "kda_decode_destroy", "kda_decode_engine", "kda_decode_launches_per_step", "kda_decode_scratch_bytes",
    "kda_status_string", "kda_decode_last_error", "kda_decode_abi_version", "kda_decode_debug_copy",
    "kda_decode_step_noalloc", "kda_decode_step_tokens", "kda_state_checkpoint", "kda_state_restore",
    "kda_decode_set_launch_overlap", "kda_decode_tokens_engine", "kda_prefill", "kda_tp_configure",
    "kda_tp_set_peer", "kda_decode_step_host_async",
)
KDA_TP_HANDLE_BYTES = 64
KDA_NOALLOC_MAX_SCRATCH_BYTES = 1 << 20
KDA_DEBUG_Q, KDA_DEBUG_K, KDA_DEBUG_V, KDA_DEBUG_BETA_PRE, KDA_DEBUG_T = range(5)


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        name = _lib_or_none().kda_status_string(status).decode() if _lib_or_none() else str(status)
        super().__init__(f"{where}: {name}" + (f" ({detail})" if detail else ""))


class kda_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("num_heads", ctypes.c_int), ("head_dk", ctypes.c_int),
                ("head_dv", ctypes.c_int), ("alpha_rank", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("out_dtype", ctypes.c_int), ("engine", ctypes.c_int), ("reserved", ctypes.c_int * 8)]


WEIGHT_FIELDS = ("wq", "wk", "wv", "wo", "sq", "sk", "sv", "so", "wa_down", "wa_up", "wb")


class kda_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


_lib = None


def _lib_or_none():
    return _lib


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing "
                           "(python -m linear_attention_layer_kda_b200.build)")
    lib = ctypes.CDLL(path)
    P, I = ctypes.c_void_p, ctypes.c_int
    sig = {
        "kda_decode_init": (I, [ctypes.POINTER(kda_config), ctypes.POINTER(P)]),
        "kda_decode_set_stream": (I, [P, P]),
        "kda_decode_step": (I, [P, P, ctypes.POINTER(kda_weights), P, P, I]),
        "kda_decode_step_host": (I, [P, P, ctypes.POINTER(kda_weights), P, P, I]),
        "kda_decode_sync": (I, [P]),
        "kda_decode_destroy": (I, [P]),
        "kda_decode_engine": (I, [P, I]),
        "kda_decode_launches_per_step": (I, [P, I]),
        "kda_decode_scratch_bytes": (I, [ctypes.POINTER(kda_config), ctypes.POINTER(ctypes.c_size_t)]),
        "kda_status_string": (ctypes.c_char_p, [I]),
        "kda_decode_last_error": (ctypes.c_char_p, [P]),
        "kda_decode_abi_version": (I, []),
        "kda_decode_debug_copy": (I, [P, I, P, ctypes.c_size_t]),
        "kda_decode_step_noalloc": (I, [ctypes.POINTER(kda_config), P, ctypes.POINTER(kda_weights), P, P, I, P]),
        "kda_decode_step_tokens": (I, [P, P, ctypes.POINTER(kda_weights), P, P, I, I]),
        "kda_state_checkpoint": (I, [P, P, I, I, P]),
        "kda_state_restore": (I, [P, P, P, I, I]),
        "kda_decode_set_launch_overlap": (I, [P, I]),
        "kda_decode_tokens_engine": (I, [P, I, I]),
        "kda_prefill": (I, [P, P, ctypes.POINTER(kda_weights), P, P, I, I, I]),
        "kda_tp_configure": (I, [P, I, I, P]),
        "kda_tp_set_peer": (I, [P, I, P]),
        "kda_decode_step_host_async": (I, [P, P, ctypes.POINTER(kda_weights), P, P, I]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def _check(rc: int, where: str, h=None) -> None:
    if rc != KDA_OK:
        detail = load().kda_decode_last_error(h).decode() if h else ""
        raise KdaError(rc, where, detail)


# ------------------------------------------------------------------ C-named wrappers

def kda_decode_init(cfg: kda_config) -> int:
    h = ctypes.c_void_p()
    _check(load().kda_decode_init(ctypes.byref(cfg), ctypes.byref(h)), "kda_decode_init")
    return h.value


def kda_decode_set_stream(h: int, stream: int) -> None:
    _check(load().kda_decode_set_stream(h, stream), "kda_decode_set_stream", h)


def kda_decode_step(h: int, x: int, w: kda_weights, state: int, out: int, batch: int) -> None:
    _check(load().kda_decode_step(h, x, ctypes.byref(w), state, out, batch), "kda_decode_step", h)


def kda_decode_step_tokens(h: int, x: int, w: kda_weights, state: int, out: int, batch: int, tokens: int) -> None:
    _check(load().kda_decode_step_tokens(h, x, ctypes.byref(w), state, out, batch, tokens), "kda_decode_step_tokens", h)


def kda_prefill(h: int, x: int, w: kda_weights, state: int, out: int, batch: int, tokens: int, chunk: int) -> None:
    _check(load().kda_prefill(h, x, ctypes.byref(w), state, out, batch, tokens, chunk), "kda_prefill", h)


def kda_state_checkpoint(h: int, state: int, seq0: int, nseq: int, host_dst: int) -> None:
    _check(load().kda_state_checkpoint(h, state, seq0, nseq, host_dst), "kda_state_checkpoint", h)


def kda_state_restore(h: int, host_src: int, state: int, seq0: int, nseq: int) -> None:
    _check(load().kda_state_restore(h, host_src, state, seq0, nseq), "kda_state_restore", h)


def kda_decode_step_host(h: int, x_host: int, w: kda_weights, state: int, out_host: int, batch: int) -> None:
    _check(load().kda_decode_step_host(h, x_host, ctypes.byref(w), state, out_host, batch), "kda_decode_step_host", h)


def kda_decode_step_host_async(h: int, x_host: int, w: kda_weights, state: int, out_host: int, batch: int) -> None:
    _check(load().kda_decode_step_host_async(h, x_host, ctypes.byref(w), state, out_host, batch),
           "kda_decode_step_host_async", h)


def kda_decode_set_launch_overlap(h: int, on: bool) -> None:
    _check(load().kda_decode_set_launch_overlap(h, 1 if on else 0), "kda_decode_set_launch_overlap", h)


def kda_tp_configure(h: int, rank: int, world: int) -> bytes:
    buf = ctypes.create_string_buffer(KDA_TP_HANDLE_BYTES)
    _check(load().kda_tp_configure(h, rank, world, buf), "kda_tp_configure", h)
    return buf.raw


def kda_tp_set_peer(h: int, peer: int, handle: bytes) -> None:
    if len(handle) != KDA_TP_HANDLE_BYTES:
        raise ValueError(f"an exchange handle has {KDA_TP_HANDLE_BYTES} bytes, got {len(handle)}")
    buf = ctypes.create_string_buffer(handle, KDA_TP_HANDLE_BYTES)
    _check(load().kda_tp_set_peer(h, peer, buf), "kda_tp_set_peer", h)


def kda_decode_sync(h: int) -> None:
    _check(load().kda_decode_sync(h), "kda_decode_sync", h)


def kda_decode_destroy(h: int) -> None:
    _check(load().kda_decode_destroy(h), "kda_decode_destroy")


def kda_decode_engine(h: int, batch: int) -> int:
    return load().kda_decode_engine(h, batch)


def kda_decode_tokens_engine(h: int, batch: int, tokens: int) -> int:
    return load().kda_decode_tokens_engine(h, batch, tokens)


def kda_decode_launches_per_step(h: int, batch: int) -> int:
    return load().kda_decode_launches_per_step(h, batch)


def kda_decode_scratch_bytes(cfg: kda_config) -> int:
    n = ctypes.c_size_t()
    _check(load().kda_decode_scratch_bytes(ctypes.byref(cfg), ctypes.byref(n)), "kda_decode_scratch_bytes")
    return n.value


def kda_decode_debug_copy(h: int, which: int, dst: int, nbytes: int) -> None:
    _check(load().kda_decode_debug_copy(h, which, dst, nbytes), "kda_decode_debug_copy", h)


def kda_decode_step_noalloc(cfg: kda_config, x: int, w: kda_weights, state: int, out: int, batch: int,
                            stream: int) -> None:
    _check(load().kda_decode_step_noalloc(ctypes.byref(cfg), x, ctypes.byref(w), state, out, batch, stream),
           "kda_decode_step_noalloc")


def kda_status_string(status: int) -> str:
    return load().kda_status_string(status).decode()


def kda_decode_abi_version() -> int:
    return load().kda_decode_abi_version()


# ------------------------------------------------------------------ torch convenience

def make_config(hidden, num_heads, head_dk, head_dv, alpha_rank, max_batch, out_dtype=KDA_OUT_F32,
                engine=KDA_ENGINE_AUTO) -> kda_config:
    c = kda_config()
    c.hidden, c.num_heads, c.head_dk, c.head_dv = hidden, num_heads, head_dk, head_dv
    c.alpha_rank, c.max_batch, c.out_dtype, c.engine = alpha_rank, max_batch, out_dtype, engine
    return c


def weights_from_tensors(t: Dict[str, "object"]) -> kda_weights:
    """kda_weights from a dict of CUDA tensors keyed by WEIGHT_FIELDS.

    The returned struct keeps references to the tensors, so the device memory
    its pointers name stays allocated as long as the struct is alive.
    """
    w = kda_weights()
    for n in WEIGHT_FIELDS:
        a = t[n]
        if not a.is_cuda or not a.is_contiguous():
            raise ValueError(f"weight {n} must be a contiguous CUDA tensor")
        setattr(w, n, a.data_ptr())
    w._tensors = dict(t)
    return w


class KdaDecoder:
    """Owns one library handle; steps take torch tensors (device pointers are passed through)."""

    def __init__(self, hidden, num_heads, head_dk, head_dv, alpha_rank, max_batch, out_dtype=KDA_OUT_F32,
                 engine=KDA_ENGINE_AUTO):
        import torch

        self.cfg = make_config(hidden, num_heads, head_dk, head_dv, alpha_rank, max_batch, out_dtype, engine)
        self.h = kda_decode_init(self.cfg)
        self._stream = None
        self._torch = torch

    def _bind_stream(self):
        s = self._torch.cuda.current_stream().cuda_stream
        if s != self._stream:
            kda_decode_set_stream(self.h, s)
            self._stream = s

    def step(self, x, weights: kda_weights, state, out, batch: Optional[int] = None) -> None:
        for n, a in (("x", x), ("state", state), ("out", out)):
            if not a.is_cuda or not a.is_contiguous():
                raise ValueError(f"{n} must be a contiguous CUDA tensor")
        b = x.shape[0] if batch is None else batch
        self._bind_stream()
        kda_decode_step(self.h, x.data_ptr(), weights, state.data_ptr(), out.data_ptr(), b)

    def step_host(self, x_host, weights: kda_weights, state, out_host, batch: Optional[int] = None) -> None:
        b = x_host.shape[0] if batch is None else batch
        self._bind_stream()
        kda_decode_step_host(self.h, x_host.data_ptr(), weights, state.data_ptr(), out_host.data_ptr(), b)

    def step_host_async(self, x_host, weights: kda_weights, state, out_host, batch: Optional[int] = None) -> None:
        """Host-buffer step without waiting (copies on the handle's copy stream); out_host is
        valid after sync()."""
        b = x_host.shape[0] if batch is None else batch
        self._bind_stream()
        kda_decode_step_host_async(self.h, x_host.data_ptr(), weights, state.data_ptr(), out_host.data_ptr(), b)

    def step_tokens(self, x, weights: kda_weights, state, out, batch: int, tokens: int) -> None:
        """`tokens` tokens of each of `batch` sequences; x and out are [batch * tokens, H]."""
        for n, a in (("x", x), ("state", state), ("out", out)):
            if not a.is_cuda or not a.is_contiguous():
                raise ValueError(f"{n} must be a contiguous CUDA tensor")
        rows = batch * tokens
        if x.shape[0] < rows or out.shape[0] < rows or state.shape[0] < batch:
            raise ValueError(f"x and out need {rows} rows and state {batch} sequences")
        self._bind_stream()
        kda_decode_step_tokens(self.h, x.data_ptr(), weights, state.data_ptr(), out.data_ptr(), batch, tokens)

    def prefill(self, x, weights: kda_weights, state, out, batch: int, tokens: int, chunk: int = 0) -> None:
        """`tokens` tokens of each of `batch` sequences through the chunked recurrence; x and out
        are [batch * tokens, H]."""
        for n, a in (("x", x), ("state", state), ("out", out)):
            if not a.is_cuda or not a.is_contiguous():
                raise ValueError(f"{n} must be a contiguous CUDA tensor")
        rows = batch * tokens
        if x.shape[0] < rows or out.shape[0] < rows or state.shape[0] < batch:
            raise ValueError(f"x and out need {rows} rows and state {batch} sequences")
        self._bind_stream()
        kda_prefill(self.h, x.data_ptr(), weights, state.data_ptr(), out.data_ptr(), batch, tokens, chunk)

    def _state_range(self, state, host, seq0: int, nseq: Optional[int]) -> int:
        n = state.shape[0] - seq0 if nseq is None else nseq
        c = self.cfg
        need = n * c.num_heads * c.head_dk * c.head_dv * 4
        if not state.is_cuda or not state.is_contiguous() or seq0 < 0 or n < 1 or seq0 + n > state.shape[0]:
            raise ValueError("state must be a contiguous CUDA tensor holding sequences [seq0, seq0 + nseq)")
        if host.is_cuda or not host.is_contiguous() or host.numel() * host.element_size() < need:
            raise ValueError(f"host must be a contiguous host tensor of at least {need} bytes")
        return n

    def checkpoint(self, state, host, seq0: int = 0, nseq: Optional[int] = None) -> None:
        """Enqueues a copy of sequences [seq0, seq0 + nseq) of `state` into the host tensor `host`."""
        n = self._state_range(state, host, seq0, nseq)
        self._bind_stream()
        kda_state_checkpoint(self.h, state.data_ptr(), seq0, n, host.data_ptr())

    def restore(self, host, state, seq0: int = 0, nseq: Optional[int] = None) -> None:
        """Enqueues a copy of the host tensor `host` into sequences [seq0, seq0 + nseq) of `state`."""
        n = self._state_range(state, host, seq0, nseq)
        self._bind_stream()
        kda_state_restore(self.h, host.data_ptr(), state.data_ptr(), seq0, n)

    def sync(self) -> None:
        kda_decode_sync(self.h)

    def set_launch_overlap(self, on: bool) -> None:
        """Overlap of consecutive fused steps (programmatic dependent launch); on by default."""
        kda_decode_set_launch_overlap(self.h, on)

    def debug_tensor(self, which: int, batch: int):
        """fp32 copy of one intermediate of the last step (KDA_DEBUG_*), shape [batch, n]."""
        c = self.cfg
        n = {KDA_DEBUG_Q: c.num_heads * c.head_dk, KDA_DEBUG_K: c.num_heads * c.head_dk,
             KDA_DEBUG_V: c.num_heads * c.head_dv, KDA_DEBUG_BETA_PRE: c.num_heads,
             KDA_DEBUG_T: c.alpha_rank}[which]
        t = self._torch.empty(batch, n, device="cuda", dtype=self._torch.float32)
        self._bind_stream()
        kda_decode_debug_copy(self.h, which, t.data_ptr(), t.numel() * 4)
        return t

    def tp_configure(self, rank: int, world: int) -> bytes:
        """Exchange region of rank `rank` of `world`; returns its IPC handle for the peers."""
        return kda_tp_configure(self.h, rank, world)

    def tp_set_peer(self, peer: int, handle: bytes) -> None:
        kda_tp_set_peer(self.h, peer, handle)

    def engine(self, batch: int) -> int:
        return kda_decode_engine(self.h, batch)

    def tokens_engine(self, batch: int, tokens: int) -> int:
        return kda_decode_tokens_engine(self.h, batch, tokens)

    def launches_per_step(self, batch: int) -> int:
        return kda_decode_launches_per_step(self.h, batch)

    def close(self) -> None:
        if self.h:
            kda_decode_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
