"""Writes the regression fixtures of this folder.  Calls only the input
generator and ``oracle/`` (never the CUDA library).

  tiny_inputs.sha256   SHA-256 of every input byte of the tiny workload
                       (batch 1, hidden 256, 2 heads of 64, 16 steps, seed 0)
  tiny_oracle_out.txt  oracle out[step][i] on a sample of (step, i) and the
                       sum of the final fp64 state

Run from the repository root:  python tests/golden/make_golden.py
"""
import hashlib
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from linear_attention_layer_kda_b200 import inputs as I  # noqa: E402


def main():
    shape = I.CONFIGS[0]
    inp = I.generate(shape)
    h = hashlib.sha256()
    for a in (inp.x, inp.wq, inp.sq, inp.wk, inp.sk, inp.wv, inp.sv, inp.wo, inp.so, inp.wa_down, inp.wa_up,
              inp.wb, inp.state0):
        h.update(np.ascontiguousarray(a).tobytes())
    with open(os.path.join(HERE, "tiny_inputs.sha256"), "w") as f:
        f.write("# SHA-256 of the tiny workload's input bytes (x, wq, sq, wk, sk, wv, sv, wo, so, wa_down,\n")
        f.write("# wa_up, wb, state0 in that order); written by make_golden.py\n")
        f.write(h.hexdigest() + "\n")
    m = oracle.OracleModel(inp)
    S = inp.state0.astype(np.float64).copy()
    rows = []
    for t in range(shape.steps):
        out = m.step(inp.x[t], S)
        for i in (0, 1, 77, 128, 255):
            rows.append((t, i, out[0, i]))
    with open(os.path.join(HERE, "tiny_oracle_out.txt"), "w") as f:
        f.write("# fp64 oracle (rank-1 form) on the tiny workload: step index out[0][index]\n")
        f.write("# written by make_golden.py from oracle/ only; last line: sum of the final state\n")
        for t, i, v in rows:
            f.write(f"{t} {i} {float(v)!r}\n")
        f.write(f"state_sum - {float(S.sum())!r}\n")


if __name__ == "__main__":
    main()
