"""The fused engine's tile schedule (host code, csrc/schedule.cu), checked without a GPU.

Built here with g++ together with a small shim (tests/schedule_shim.cpp).  For several
shapes and CTA counts: every weight tile is streamed exactly once; CTAs differ by at most
one tile; every CTA streams its q/k/v tiles before its W_o tiles; runs of one row block are
contiguous and each owns a distinct partial-sum slot inside its row block's range, as the
consumers that add the partials expect.
"""
import collections
import ctypes
import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_attention_layer_kda_b200", "csrc")
SEG_START, SEG_END = 1, 2


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("sched") / "libsched.so")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-shared", "-fPIC", "-x", "c++",
                           os.path.join(CSRC, "schedule.cu"), os.path.join(ROOT, "tests", "schedule_shim.cpp"),
                           "-I" + os.path.join(ROOT, "include"), "-I" + CSRC, "-I/usr/local/cuda/include", "-o", out])
    return ctypes.CDLL(out)


def schedule(lib, H, nh, dk, dv, r, P):
    cap = 4 * (nh * max(dk, dv) // 128 + 1) * (H // 128 + 1) * 2
    arr = {n: np.zeros(cap, t) for n, t in (("mat", np.uint8), ("flags", np.uint8), ("rb", np.uint16),
                                            ("kb", np.uint16), ("seg", np.uint32), ("seg0", np.uint32),
                                            ("nseg", np.uint16))}
    off = np.zeros(P + 1, np.uint32)
    rbinfo = np.zeros(2 * (4 * cap), np.uint32)
    nt, ns = ctypes.c_size_t(), ctypes.c_size_t()
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = lib.kda_test_schedule(8, H, nh, dk, dv, r, P, ctypes.c_size_t(cap), p(arr["mat"]), p(arr["flags"]),
                               p(arr["rb"]), p(arr["kb"]), p(arr["seg"]), p(arr["seg0"]), p(arr["nseg"]), p(off),
                               p(rbinfo), ctypes.c_size_t(rbinfo.size), ctypes.byref(nt), ctypes.byref(ns))
    assert rc == 0
    n = nt.value
    return {k: v[:n] for k, v in arr.items()}, off, rbinfo, ns.value


SHAPES = [(4096, 32, 128, 128, 64), (6144, 48, 128, 128, 64), (256, 2, 64, 64, 64), (384, 2, 128, 64, 32),
          (1024, 16, 64, 128, 16)]


@pytest.mark.parametrize("P", [148, 132, 7])
@pytest.mark.parametrize("H,nh,dk,dv,r", SHAPES)
@pytest.mark.parametrize("lag", [None, "2"])
def test_schedule_invariants(lib, monkeypatch, H, nh, dk, dv, r, P, lag):
    if lag is None:
        monkeypatch.delenv("KDA_WO_LAG", raising=False)
    else:
        monkeypatch.setenv("KDA_WO_LAG", lag)
    t, off, rbinfo, nseg_total = schedule(lib, H, nh, dk, dv, r, P)
    nKBx, nRBq, nRBv, nRBo, nKBo = H // 128, nh * dk // 128, nh * dv // 128, H // 128, nh * dv // 128
    # every tile exactly once
    got = collections.Counter(zip(t["mat"].tolist(), t["rb"].tolist(), t["kb"].tolist()))
    want = collections.Counter()
    for m, nrb, nkb in ((0, nRBq, nKBx), (1, nRBq, nKBx), (2, nRBv, nKBx), (3, nRBo, nKBo)):
        for rb in range(nrb):
            for kb in range(nkb):
                want[(m, rb, kb)] += 1
    assert got == want
    # balance
    counts = np.diff(off.astype(np.int64))
    assert counts.sum() == len(t["mat"]) and counts.max() - counts.min() <= 1
    # segments and their slots
    key = np.where(t["mat"] == 3, 2 * nRBq + nRBv + t["rb"],
                   np.where(t["mat"] == 2, 2 * nRBq + t["rb"], t["mat"].astype(np.int64) * nRBq + t["rb"]))
    runs = collections.Counter()
    slots = set()
    for c in range(P):
        lo, hi = int(off[c]), int(off[c + 1])
        if lag is None and hi > lo:  # q/k/v tiles first, then W_o
            m = t["mat"][lo:hi]
            assert np.all(np.diff((m == 3).astype(np.int8)) >= 0)
        i = lo
        while i < hi:
            j = i
            while j + 1 < hi and key[j + 1] == key[i]:
                j += 1
            k = int(key[i])
            assert t["flags"][i] & SEG_START and t["flags"][j] & SEG_END
            assert np.all(t["seg"][i:j + 1] == t["seg"][i])
            s0, ns = int(rbinfo[2 * k]), int(rbinfo[2 * k + 1])
            assert np.all(t["seg0"][i:j + 1] == s0) and np.all(t["nseg"][i:j + 1] == ns)
            assert s0 <= int(t["seg"][i]) < s0 + ns
            assert int(t["seg"][i]) not in slots
            slots.add(int(t["seg"][i]))
            runs[k] += 1
            i = j + 1
    assert len(slots) == nseg_total
    for k, n in runs.items():
        assert int(rbinfo[2 * k + 1]) == n
