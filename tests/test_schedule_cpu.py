"""The fused engine's tile schedule (host code, csrc/schedule.cu), checked without a GPU.

Built here with g++ together with a small shim (tests/schedule_shim.cpp).  For several
shapes, padded batches and CTA counts: every weight tile (a row group of N weight rows x one
128-wide K block) is streamed exactly once; CTAs differ by at most one tile; every CTA
streams its q/k/v tiles before its W_o tiles; the tiles are dealt in waves, earliest heads
first; runs of one row group are contiguous and each owns a distinct partial-sum slot inside
its row group's range, as the consumers that add the partials expect.  The shim also
exposes the host's decoding of the kernels' status words (csrc/status.cu).
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
                           os.path.join(CSRC, "schedule.cu"), os.path.join(CSRC, "status.cu"),
                           os.path.join(ROOT, "tests", "schedule_shim.cpp"),
                           "-I" + os.path.join(ROOT, "include"), "-I" + CSRC, "-I/usr/local/cuda/include", "-o", out])
    return ctypes.CDLL(out)


def sched_geo(lib, BP, H, nh, dk, dv, r):
    nx, no, run = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    lib.kda_test_sched_geo(BP, H, nh, dk, dv, r, ctypes.byref(nx), ctypes.byref(no), ctypes.byref(run))
    return nx.value, no.value, run.value


def schedule(lib, BP, H, nh, dk, dv, r, P):
    nx, no, run = sched_geo(lib, BP, H, nh, dk, dv, r)
    cap = 4 * (nh * max(dk, dv) // 64 + H // 64 + 4) * (H // 128 + nh * dv // 128 + 2)
    arr = {n: np.zeros(cap, t) for n, t in (("mat", np.uint8), ("flags", np.uint8), ("rg", np.uint16),
                                            ("kb", np.uint16), ("seg", np.uint32), ("seg0", np.uint32),
                                            ("nseg", np.uint16))}
    off = np.zeros(P + 1, np.uint32)
    rbinfo = np.zeros(2 * cap, np.uint32)
    nt, ns = ctypes.c_size_t(), ctypes.c_size_t()
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = lib.kda_test_schedule(BP, H, nh, dk, dv, r, P, ctypes.c_size_t(cap), p(arr["mat"]), p(arr["flags"]),
                               p(arr["rg"]), p(arr["kb"]), p(arr["seg"]), p(arr["seg0"]), p(arr["nseg"]), p(off),
                               p(rbinfo), ctypes.c_size_t(rbinfo.size), ctypes.byref(nt), ctypes.byref(ns))
    assert rc == 0
    n = nt.value
    return {k: v[:n] for k, v in arr.items()}, off, rbinfo, ns.value, (nx, no, run)


SHAPES = [(4096, 32, 128, 128, 64), (6144, 48, 128, 128, 64), (256, 2, 64, 64, 64), (384, 2, 128, 64, 32),
          (1024, 16, 64, 128, 16)]


@pytest.mark.parametrize("BP,want", [(8, (256, 256, 2)), (16, (256, 256, 4)), (32, (256, 128, 8)),
                                     (64, (128, 64, 32))])
def test_sched_geo(lib, BP, want):
    assert sched_geo(lib, BP, 4096, 32, 128, 128, 64) == want


@pytest.mark.parametrize("BP,H,run", [(64, 6144, 24), (32, 6144, 8), (8, 6144, 2), (64, 384, 3), (8, 384, 2),
                                      (16, 128, 1), (64, 5120, 20), (32, 1280, 5)])
def test_runs_cut_the_k_blocks_evenly(lib, BP, H, run):
    """A row group's K blocks are cut into the fewest equal runs no longer than the padded
    batch's longest run (2, 4, 8, BP / 2)."""
    assert sched_geo(lib, BP, H, H // 128, 128, 128, 64)[2] == run


@pytest.mark.parametrize("P", [148, 132, 7])
@pytest.mark.parametrize("H,nh,dk,dv,r", SHAPES)
@pytest.mark.parametrize("BP", [8, 32, 64])
def test_schedule_invariants(lib, monkeypatch, H, nh, dk, dv, r, P, BP):
    monkeypatch.delenv("KDA_RUN", raising=False)
    t, off, rbinfo, nseg_total, (nx, no, run) = schedule(lib, BP, H, nh, dk, dv, r, P)
    Dk, Dv = nh * dk, nh * dv
    nKBx, nKBo = H // 128, Dv // 128
    nRGq, nRGv, nRGo = -(-Dk // nx), -(-Dv // nx), -(-H // no)
    # every tile exactly once
    got = collections.Counter(zip(t["mat"].tolist(), t["rg"].tolist(), t["kb"].tolist()))
    want = collections.Counter()
    for m, nrg, nkb in ((0, nRGq, nKBx), (1, nRGq, nKBx), (2, nRGv, nKBx), (3, nRGo, nKBo)):
        for rg in range(nrg):
            for kb in range(nkb):
                want[(m, rg, kb)] += 1
    assert got == want
    # balance
    counts = np.diff(off.astype(np.int64))
    assert counts.sum() == len(t["mat"]) and counts.max() - counts.min() <= 1
    # waves: the i-th tile of every CTA in wave i // run never holds later heads than wave i // run + 1
    first_head = np.where(t["mat"] == 3, 10 ** 6 + t["kb"].astype(np.int64) // run,
                          np.where(t["mat"] == 2, t["rg"].astype(np.int64) * nx // dv,
                                   t["rg"].astype(np.int64) * nx // dk))
    full_waves = min(int(c) for c in counts) // run
    for w in range(full_waves - 1):
        cur = [first_head[int(off[c]) + w * run + i] for c in range(P) for i in range(run)]
        nxt = [first_head[int(off[c]) + (w + 1) * run + i] for c in range(P) for i in range(run)]
        assert max(cur) <= min(nxt)
    # segments and their slots
    key = np.where(t["mat"] == 3, 2 * nRGq + nRGv + t["rg"],
                   np.where(t["mat"] == 2, 2 * nRGq + t["rg"], t["mat"].astype(np.int64) * nRGq + t["rg"]))
    runs = collections.Counter()
    slots = set()
    for c in range(P):
        lo, hi = int(off[c]), int(off[c + 1])
        if hi > lo:  # q/k/v tiles first, then W_o
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


def take_status(lib, words, fatal=0):
    w = (ctypes.c_int * 3)(*words)
    f = ctypes.c_int(fatal)
    msg = ctypes.create_string_buffer(256)
    st = lib.kda_test_take_status(w, ctypes.byref(f), msg, ctypes.c_size_t(256))
    return st, list(w), f.value, msg.value.decode()


def test_status_words_decoding(lib):
    OK, TIMEOUT = 0, 4
    assert take_status(lib, [0, 0, 0]) == (OK, [0, 0, 0], 0, "")
    st, w, fatal, msg = take_status(lib, [TIMEOUT, 7, 0])
    assert st == TIMEOUT and w == [0, 0, 0] and fatal == 0 and "wait site 7" in msg
    # a drain that gave up makes the handle unusable, even without a recorded status code
    st, w, fatal, msg = take_status(lib, [0, 0, 1])
    assert st == TIMEOUT and fatal == 1 and w == [0, 0, 0] and "unusable" in msg
    st, w, fatal, msg = take_status(lib, [TIMEOUT, 3, 1])
    assert st == TIMEOUT and fatal == 1 and "wait site 3" in msg
    # the fatal mark is never cleared by later clean words
    st, w, fatal, msg = take_status(lib, [0, 0, 0], fatal=1)
    assert st == OK and fatal == 1
