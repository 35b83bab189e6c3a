"""Helpers shared by the GPU parity tests (no method arithmetic here)."""
import dataclasses

import numpy as np
import torch

import synth

# float outputs: max |gpu - oracle| / max |oracle| per head (bf16 in, fp32 accumulate)
REL_TOL = 2e-2


def workload(name, **over):
    w = synth.WORKLOADS[name]
    return dataclasses.replace(w, **over) if over else w


def rel_err_per_head(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    errs = []
    for h in range(ref.shape[0]):
        den = np.abs(ref[h]).max()
        errs.append(np.abs(got[h] - ref[h]).max() / (den if den > 0 else 1.0))
    return max(errs)


def bf16_round_f64(x):
    """Nearest bf16 value (ties to even) of fp64 values, returned as fp64.

    Keeps 8 significant bits of each value's binary significand with numpy's
    round-half-to-even (for values in bf16's normal range)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                 # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


def host(t):
    return synth.to_f64(t)


def sync_ok():
    import linear_hybrid_attention_b200 as zb
    torch.cuda.synchronize()
    zb.zb_last_device_status()
