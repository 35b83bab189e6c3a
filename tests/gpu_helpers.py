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


# the per-element figure reported beside it: |gpu - oracle| / max(|oracle|, floor),
# floor = ELEM_FLOOR * max |oracle| of the head
ELEM_FLOOR = 1e-3

# (test, label, per-head error, per-element error) of every check_close in this session
REPORT = []


def elem_err_per_head(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    errs = []
    for h in range(ref.shape[0]):
        a = np.abs(ref[h])
        den = np.maximum(a, ELEM_FLOOR * a.max()) if a.max() > 0 else np.ones_like(a)
        errs.append((np.abs(got[h] - ref[h]) / den).max())
    return max(errs)


def check_close(got, ref, tol=REL_TOL, label=""):
    """Assert the per-head error bar; record it with the per-element figure."""
    import os
    head = rel_err_per_head(got, ref)
    elem = elem_err_per_head(got, ref)
    REPORT.append({"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "label": label,
                   "per_head": float(head), "per_element": float(elem), "tol": tol})
    assert head <= tol, (label, head, elem)
    return head, elem


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
