"""Failure detection on the GPU without a GPU fault.

The fused kernel bounds every wait with a global-timer limit (KDA_WAIT_LIMIT_MS).  With
KDA_DEBUG_SKIP_GATE_RELEASE set when a handle is created, the kernel never publishes its
gate rows, so the state units' wait on them runs out: the kernel records
KDA_ERR_DEVICE_TIMEOUT in the handle's status word, raises its abort flag, lets every CTA
finish its copies in flight and returns.  The context stays usable: the same handle runs
(and times out) again after its counters are reset, and a fresh handle then computes the
step correctly.  The test runs in a child process so the environment switches stay local.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

CHILD = r"""
import os, sys
import numpy as np
import torch
import oracle
from linear_attention_layer_kda_b200 import binding, inputs as I, tensors
from gpu_util import OUT_TOL, STATE_TOL, maxrel

shape = I.CONFIGS[0]
inp = I.generate(shape.replace(steps=2))
B = shape.batch

def make():
    return binding.KdaDecoder(shape.hidden, shape.num_heads, shape.head_dk, shape.head_dv, shape.alpha_rank, B,
                              engine=binding.KDA_ENGINE_FUSED)

w = tensors.weights_struct(tensors.to_device_weights(inp))
out = torch.zeros(B, shape.hidden, device="cuda")

os.environ["KDA_WAIT_LIMIT_MS"] = "50"
os.environ["KDA_DEBUG_SKIP_GATE_RELEASE"] = "1"
bad = make()
assert bad.engine(B) == binding.KDA_ENGINE_FUSED
for attempt in range(2):
    st = tensors.state_tensor(inp.state0)
    bad.step(tensors.bf16_tensor(inp.x[0]), w, st, out)
    try:
        bad.sync()
        print("NO_TIMEOUT", attempt)
    except binding.KdaError as e:
        print("TIMEOUT", attempt, e.status, str(e).replace(chr(10), " "))
bad.close()

del os.environ["KDA_DEBUG_SKIP_GATE_RELEASE"]
os.environ["KDA_WAIT_LIMIT_MS"] = "2000"
good = make()
st = tensors.state_tensor(inp.state0)
model = oracle.OracleModel(inp, batch=B)
S = inp.state0.astype(np.float64).copy()
for t in range(2):
    good.step(tensors.bf16_tensor(inp.x[t]), w, st, out)
    ref = model.step(inp.x[t], S)
good.sync()
eo = maxrel(out.double().cpu().numpy(), ref)
es = maxrel(st.double().cpu().numpy(), S)
print("RECOVERED", eo, es, eo <= OUT_TOL and es <= STATE_TOL)
good.close()
model.close()
"""


def test_bounded_wait_times_out_and_the_context_recovers():
    env = dict(os.environ)
    env["PYTHONPATH"] = os.pathsep.join([ROOT, os.path.join(ROOT, "tests")] +
                                        ([env["PYTHONPATH"]] if env.get("PYTHONPATH") else []))
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    log = r.stdout + r.stderr
    assert r.returncode == 0, log[-4000:]
    lines = r.stdout.splitlines()
    timeouts = [ln for ln in lines if ln.startswith("TIMEOUT")]
    assert len(timeouts) == 2, log[-4000:]
    for ln in timeouts:
        assert f" {4} " in ln and "KDA_ERR_DEVICE_TIMEOUT" in ln and "wait site" in ln, ln
    rec = [ln for ln in lines if ln.startswith("RECOVERED")]
    assert rec and rec[0].endswith("True"), log[-4000:]
