"""GPU-side test helpers: run the CUDA path through the C ABI and the oracle side by side."""
import numpy as np

import oracle
from linear_attention_layer_kda_b200 import binding, inputs as I, tensors

OUT_TOL = 2e-3    # max-norm relative error of out
STATE_TOL = 1e-3  # max-norm relative error of the updated state


def maxrel(got, ref):
    den = float(np.abs(ref).max())
    return float(np.abs(np.asarray(got, np.float64) - ref).max() / (den if den > 0 else 1.0))


def block_report(got, ref, shape):
    """Per-head error map of a [B, nh, dk, dv] state (printed when a check fails)."""
    g = np.asarray(got, np.float64)
    e = np.abs(g - ref).max(axis=(2, 3)) / max(float(np.abs(ref).max()), 1e-300)
    rows = [" ".join(f"{v:.1e}" for v in e[b]) for b in range(e.shape[0])]
    return "per-(seq, head) max error / max|ref|:\n" + "\n".join(rows)


def run_parity(inp, steps, engine=binding.KDA_ENGINE_AUTO, out_dtype=binding.KDA_OUT_F32, batch=None,
               max_batch=None, check_every=1, return_state=False):
    """Runs `steps` steps on both sides; returns a list of (out_err, state_err) per checked step
    and the engine used (and, with return_state, the CUDA path's final state as fp64)."""
    import torch
    s = inp.shape
    B = s.batch if batch is None else batch
    dec = binding.KdaDecoder(s.hidden, s.num_heads, s.head_dk, s.head_dv, s.alpha_rank,
                             max_batch or B, out_dtype, engine)
    wt = tensors.to_device_weights(inp)
    w = tensors.weights_struct(wt)
    state = tensors.state_tensor(inp.state0[:B])
    odt = torch.bfloat16 if out_dtype == binding.KDA_OUT_BF16 else torch.float32
    out = torch.empty(B, s.hidden, device="cuda", dtype=odt)
    model = oracle.OracleModel(inp, batch=B)
    S = inp.state0[:B].astype(np.float64).copy()
    errs = []
    try:
        for t in range(steps):
            x = tensors.bf16_tensor(inp.x[t][:B])
            dec.step(x, w, state, out)
            ref = model.step(inp.x[t][:B], S)
            if (t + 1) % check_every == 0 or t == steps - 1:
                dec.sync()
                got_out = out.float().double().cpu().numpy()
                got_state = state.double().cpu().numpy()
                eo, es = maxrel(got_out, ref), maxrel(got_state, S)
                if not (eo <= OUT_TOL and es <= STATE_TOL):
                    print(block_report(got_state, S, s))
                errs.append((t, eo, es))
        dec.sync()
        final = state.double().cpu().numpy() if return_state else None
    finally:
        engine_used = dec.engine(B)
        dec.close()
        model.close()
    if return_state:
        return errs, engine_used, final
    return errs, engine_used
