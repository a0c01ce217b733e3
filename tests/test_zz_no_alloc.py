"""kda_decode_step_noalloc: the five-kernel decode step on the library's fixed device array.

The file name sorts last, so in a full run these tests come after every other test has
used the library in the same process; the fresh-process test runs them again in a new
interpreter, where the first call does the per-device set-up.  Both paths are compared
bit for bit with kda_decode_step on a KDA_ENGINE_SIMPLE handle (the same kernels on the
handle's own scratch) over two calls in a row, so the second call starts from the state
the first one wrote.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

from linear_attention_layer_kda_b200 import binding, inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# dk != dv, hidden of three 128-blocks, ragged batch, bf16 out
RAGGED = I.KdaShape("ragged_b5_h384_2x128x64", batch=5, hidden=384, num_heads=2, head_dk=128, head_dv=64,
                    alpha_rank=32, steps=2, seed=33)


def _bits(t):
    import torch
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def noalloc_matches_step(shape, out_dtype):
    """Two calls in a row through both entry points; the no-alloc call goes first each time."""
    import torch

    from linear_attention_layer_kda_b200 import tensors
    inp = I.generate(shape.replace(steps=2))
    B, H = shape.batch, shape.hidden
    w = tensors.weights_struct(tensors.to_device_weights(inp))
    cfg = binding.make_config(H, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B, out_dtype,
                              binding.KDA_ENGINE_SIMPLE)
    odt = torch.bfloat16 if out_dtype == binding.KDA_OUT_BF16 else torch.float32
    st_noalloc = tensors.state_tensor(inp.state0)
    st_step = st_noalloc.clone()
    out_noalloc = torch.full((B, H), float("nan"), device="cuda", dtype=odt)
    out_step = torch.full((B, H), float("nan"), device="cuda", dtype=odt)
    stream = torch.cuda.current_stream().cuda_stream
    dec = None
    try:
        for t in range(2):
            x = tensors.bf16_tensor(inp.x[t])
            binding.kda_decode_step_noalloc(cfg, x.data_ptr(), w, st_noalloc.data_ptr(), out_noalloc.data_ptr(), B,
                                            stream)
            if dec is None:  # the handle is made after the first no-alloc call
                dec = binding.KdaDecoder(H, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B,
                                         out_dtype, binding.KDA_ENGINE_SIMPLE)
            dec.step(x, w, st_step, out_step)
            dec.sync()
            torch.cuda.synchronize()
            assert bool(torch.isfinite(out_noalloc.float()).all()), f"call {t}: out not written"
            assert torch.equal(_bits(out_noalloc), _bits(out_step)), f"call {t}: out differs"
            assert torch.equal(_bits(st_noalloc), _bits(st_step)), f"call {t}: state differs"
            assert not torch.equal(st_noalloc, tensors.state_tensor(inp.state0)), "state not updated"
    finally:
        if dec is not None:
            dec.close()


@pytest.mark.gpu
def test_noalloc_matches_step_in_process():
    noalloc_matches_step(I.CONFIGS[1], binding.KDA_OUT_F32)
    noalloc_matches_step(RAGGED, binding.KDA_OUT_BF16)


@pytest.mark.gpu
def test_noalloc_alone_in_fresh_process():
    env = dict(os.environ)
    env["PYTHONPATH"] = os.pathsep.join([ROOT, os.path.join(ROOT, "tests")] +
                                        ([env["PYTHONPATH"]] if env.get("PYTHONPATH") else []))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", "-m", "gpu",
                        os.path.join(ROOT, "tests", "test_zz_no_alloc.py"), "-k", "in_process"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "1 passed" in r.stdout, r.stdout[-2000:]


def test_over_the_limit_is_rejected_before_any_device_work():
    """Needs no GPU: the size check comes before the first CUDA call (the pointers are never used)."""
    from linear_attention_layer_kda_b200.binding import kda_weights
    s = I.CONFIGS[4]  # batch 64, hidden 6144, 48 heads of 128 x 128
    cfg = binding.make_config(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank, s.batch)
    need = s.batch * (3 * s.num_heads * s.head_dk + 2 * s.num_heads * s.head_dv + s.num_heads + s.alpha_rank) * 4
    assert need > binding.KDA_NOALLOC_MAX_SCRATCH_BYTES
    w = kda_weights()
    for i, n in enumerate(binding.WEIGHT_FIELDS):
        setattr(w, n, 1 << 40 | (i + 1) << 20)  # aligned, non-null, never dereferenced
    x, st, out = 1 << 41, 1 << 42, 1 << 43
    lib = binding.load()
    import ctypes
    rc = lib.kda_decode_step_noalloc(ctypes.byref(cfg), x, ctypes.byref(w), st, out, s.batch, None)
    assert rc == binding.KDA_ERR_UNSUPPORTED_SHAPE
    # and the plain argument errors come first, as for kda_decode_step
    assert lib.kda_decode_step_noalloc(ctypes.byref(cfg), x, ctypes.byref(w), st, out, 0, None) == \
        binding.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_step_noalloc(ctypes.byref(cfg), None, ctypes.byref(w), st, out, 1, None) == \
        binding.KDA_ERR_INVALID_ARG


def test_documented_limit_matches_the_header():
    txt = open(os.path.join(ROOT, "include", "kda_decode.h")).read()
    assert "#define KDA_NOALLOC_MAX_SCRATCH_BYTES (1u << 20)" in txt
    assert binding.KDA_NOALLOC_MAX_SCRATCH_BYTES == 1 << 20
    # batch 12 of the 32 x 128 x 128 layer (hidden 4096, r 64) fits, as the header says
    s = I.CONFIGS[3]
    need = sum(-(-n // 256) * 256 for n in [s.batch * s.num_heads * s.head_dk * 4] * 3 +
               [s.batch * s.num_heads * s.head_dv * 4] * 2 + [s.batch * s.num_heads * 4, s.batch * s.alpha_rank * 4])
    assert need <= binding.KDA_NOALLOC_MAX_SCRATCH_BYTES
    assert np.isfinite(need)
