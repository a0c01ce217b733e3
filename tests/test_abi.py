"""The C-ABI library builds, loads and exports every symbol include/kda_decode.h declares.

Host-only calls (no kernel launches) are exercised here; everything that
computes runs in the gpu-marked tests.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda_decode.h")


@pytest.fixture(scope="module")
def lib():
    from linear_attention_layer_kda_b200 import binding, build
    build.build()
    return binding.load()


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^KDA_API\s+[\w\s\*]*?\b(kda_\w+)\s*\(", txt, flags=re.M)))


def test_header_declares_the_documented_entry_points():
    syms = declared_symbols()
    for s in ("kda_decode_init", "kda_decode_step", "kda_decode_destroy", "kda_decode_set_stream",
              "kda_decode_sync", "kda_status_string"):
        assert s in syms


def test_every_declared_symbol_is_exported(lib):
    from linear_attention_layer_kda_b200 import binding
    syms = declared_symbols()
    assert set(syms) == set(binding.EXPORTS)
    for s in syms:
        assert hasattr(lib, s), s


def test_library_links_no_torch(lib):
    from linear_attention_layer_kda_b200 import binding
    deps = os.popen(f"ldd {binding.LIB_PATH}").read()
    assert "torch" not in deps and "libc10" not in deps


def test_status_strings_and_version(lib):
    from linear_attention_layer_kda_b200 import binding as b
    assert b.kda_decode_abi_version() == 1
    names = {b.KDA_OK: "KDA_OK", b.KDA_ERR_INVALID_ARG: "KDA_ERR_INVALID_ARG",
             b.KDA_ERR_UNSUPPORTED_SHAPE: "KDA_ERR_UNSUPPORTED_SHAPE", b.KDA_ERR_CUDA: "KDA_ERR_CUDA",
             b.KDA_ERR_DEVICE_TIMEOUT: "KDA_ERR_DEVICE_TIMEOUT", b.KDA_ERR_NO_DEVICE: "KDA_ERR_NO_DEVICE",
             b.KDA_ERR_OUT_OF_MEMORY: "KDA_ERR_OUT_OF_MEMORY"}
    for k, v in names.items():
        assert b.kda_status_string(k) == v
    assert b.kda_status_string(99) == "KDA_ERR_UNKNOWN"


def test_config_validation_is_host_side(lib):
    from linear_attention_layer_kda_b200 import binding as b
    good = b.make_config(4096, 32, 128, 128, 64, 8)
    assert b.kda_decode_scratch_bytes(good) > 0
    bad = [
        (dict(hidden=100), b.KDA_ERR_UNSUPPORTED_SHAPE),
        (dict(head_dk=96), b.KDA_ERR_UNSUPPORTED_SHAPE),
        (dict(num_heads=1, head_dk=64), b.KDA_ERR_UNSUPPORTED_SHAPE),  # nh*dk = 64
        (dict(alpha_rank=0), b.KDA_ERR_UNSUPPORTED_SHAPE),
        (dict(alpha_rank=24), b.KDA_ERR_UNSUPPORTED_SHAPE),
        (dict(max_batch=0), b.KDA_ERR_INVALID_ARG),
        (dict(max_batch=257), b.KDA_ERR_INVALID_ARG),
        (dict(out_dtype=7), b.KDA_ERR_INVALID_ARG),
        (dict(engine=9), b.KDA_ERR_INVALID_ARG),
    ]
    for over, want in bad:
        kw = dict(hidden=4096, num_heads=32, head_dk=128, head_dv=128, alpha_rank=64, max_batch=8)
        kw.update(over)
        c = b.make_config(**kw)
        with pytest.raises(b.KdaError) as ei:
            b.kda_decode_scratch_bytes(c)
        assert ei.value.status == want, over
    c = b.make_config(4096, 32, 128, 128, 64, 8)
    c.reserved[3] = 1
    with pytest.raises(b.KdaError):
        b.kda_decode_scratch_bytes(c)


def test_null_arguments_are_rejected(lib):
    from linear_attention_layer_kda_b200 import binding as b
    assert lib.kda_decode_init(None, None) == b.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_step(None, None, None, None, None, 1) == b.KDA_ERR_INVALID_ARG
    assert lib.kda_decode_destroy(None) == b.KDA_OK
    assert lib.kda_decode_sync(None) == b.KDA_ERR_INVALID_ARG


def test_init_without_gpu_fails_loudly(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    from linear_attention_layer_kda_b200 import binding as b
    with pytest.raises(b.KdaError) as ei:
        b.kda_decode_init(b.make_config(256, 2, 64, 64, 64, 1))
    assert ei.value.status in (b.KDA_ERR_NO_DEVICE, b.KDA_ERR_CUDA)


def test_missing_library_raises(tmp_path):
    from linear_attention_layer_kda_b200 import binding as b
    saved = b._lib
    try:
        b._lib = None
        with pytest.raises(RuntimeError, match="not built"):
            b.load(str(tmp_path / "nope.so"))
    finally:
        b._lib = saved


def test_binding_rejects_bad_state_copies_without_a_device():
    """The Python checks run before any library call (the decoder here has no handle)."""
    import torch
    from linear_attention_layer_kda_b200 import binding as b
    dec = object.__new__(b.KdaDecoder)
    dec.cfg = b.make_config(256, 2, 64, 64, 64, 4)
    dec.h = None
    per_seq = 2 * 64 * 64
    host = torch.empty(4, per_seq)
    with pytest.raises(ValueError, match="contiguous CUDA tensor"):
        dec.checkpoint(torch.empty(4, 2, 64, 64), host)  # state not on a device
    with pytest.raises(ValueError):
        dec._state_range(torch.empty(4, 2, 64, 64), torch.empty(1), 0, 1)


def test_header_compiles_as_c99_and_host_calls_behave(lib, tmp_path):
    """A plain C program against include/kda_decode.h and the built library."""
    import subprocess
    from linear_attention_layer_kda_b200 import binding
    exe = str(tmp_path / "abi_check")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-o", exe, os.path.join(ROOT, "tests", "abi_check.c"),
                           "-I" + os.path.join(ROOT, "include"), binding.LIB_PATH,
                           "-Wl,-rpath," + os.path.dirname(binding.LIB_PATH)])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "abi_check ok" in r.stdout


def test_noalloc_checks_shape_only(lib):
    """kda_decode_step_noalloc ignores max_batch and engine: a config with max_batch 0 and an
    unknown engine passes validation (and then, without a GPU, stops at the device check),
    while a bad shape or out dtype is still rejected before any CUDA call."""
    import ctypes
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present: the call would run")
    from linear_attention_layer_kda_b200 import binding as b
    w = b.kda_weights()
    for n in b.WEIGHT_FIELDS:
        setattr(w, n, 0x1000)
    ptr = ctypes.c_void_p
    x, st, out = ptr(0x100000), ptr(0x200000000), ptr(0x300000000)

    def call(**over):
        kw = dict(hidden=256, num_heads=2, head_dk=64, head_dv=64, alpha_rank=64, max_batch=0, engine=99)
        kw.update(over)
        c = b.make_config(**kw)
        return lib.kda_decode_step_noalloc(ctypes.byref(c), x, ctypes.byref(w), st, out, 1, None)

    assert call() in (b.KDA_ERR_NO_DEVICE, b.KDA_ERR_CUDA)
    assert call(hidden=100) == b.KDA_ERR_UNSUPPORTED_SHAPE
    assert call(out_dtype=5) == b.KDA_ERR_INVALID_ARG
