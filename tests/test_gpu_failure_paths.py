"""Device-side failure paths, exercised without faulting the GPU.

Each failure is made on the host, and the kernels turn it into a status word
that zb_last_device_status() reports:
  * ZB_ERR_INDEX: index lists that are out of range, descending or repeated.
    The producers clamp every index before loading, so a bad list never leads
    to an out-of-bounds read; the output stays finite and the context usable.
  * ZB_ERR_SINGULAR: a calibration set whose rows are all equal, so the centred
    Gram matrix is zero (the ridge is then zero too) and the Cholesky factor
    does not exist; that head's A and b are NaN, the other heads are fitted.
  * ZB_ERR_TIMEOUT: a child process whose bounded waits are given a 100 ns
    limit (ZB_WAIT_TIMEOUT_NS).  The producer of every work item then gives up
    on its first idle period, the CTA drains its copies and MMAs (drain waits
    keep a 2 s floor) and returns; the host reads the status, the context stays
    usable and the status word is clear afterwards.
"""
import json
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402
from tests.gpu_helpers import REL_TOL, host, check_close, sync_ok, workload  # noqa: E402

pytestmark = pytest.mark.gpu

ZB_OK, ZB_ERR_TIMEOUT, ZB_ERR_INDEX, ZB_ERR_SINGULAR = 0, 7, 9, 10


def _status():
    """The device status word (synchronises; clears it)."""
    from linear_hybrid_attention_b200 import _lib
    return int(_lib.load().zb_last_device_status(torch.cuda.current_stream().cuda_stream))


def test_bad_index_lists_set_index_status_and_keep_output_finite():
    import linear_hybrid_attention_b200 as zb
    w = workload("tiny")               # 2 heads, T = 4 tiles of 64, k = 2
    Q, K, V = synth.make_qkv(w, device="cuda")
    lm = zb.zb_landmark_build(Q, K, V, w.tile)
    sync_ok()
    good = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, w.k)
    bad_rows = {"out of range": [1, 9], "negative": [-3, 2], "descending": [3, 1], "repeated": [2, 2]}
    for what, row in bad_rows.items():
        idx = good.clone()
        idx[1, 2] = torch.tensor(row, dtype=torch.int32, device="cuda")
        O = torch.zeros_like(Q)
        for wave in (True, False):
            zb.zb_tile_sparse_attn(Q, K, V, lm.Kbar_bf16, lm.Vbar_bf16, idx, w.k, w.tile, out=O,
                                   wave_sync=wave)
            assert _status() == ZB_ERR_INDEX, what
            assert _status() == ZB_OK, what          # read once, then clear
            assert bool(torch.isfinite(O.float()).all()), what
    # the context is still usable: a good call matches the oracle
    O = zb.zb_tile_sparse_attn(Q, K, V, lm.Kbar_bf16, lm.Vbar_bf16, good, w.k, w.tile)
    sync_ok()
    Q64, K64, V64 = host(Q), host(K), host(V)
    ref = oracle.sparse_attention(Q64, K64, V64, w.tile, good.cpu().numpy(), 1 / math.sqrt(64))
    check_close(host(O), ref)


def test_gather_tiles_out_of_range_sets_index_status():
    import linear_hybrid_attention_b200 as zb
    w = workload("tiny")
    Q, _, _ = synth.make_qkv(w, device="cuda")
    tiles = torch.tensor([0, 4], dtype=torch.int32, device="cuda")   # T = 4: tile 4 does not exist
    out = zb.zb_gather_tiles(Q, w.tile, tiles)
    assert _status() == ZB_ERR_INDEX
    assert bool((out[:, w.tile:].float() == 0).all())
    assert torch.equal(out[:, :w.tile], Q[:, :w.tile])


def test_singular_fit_sets_status_and_writes_nan_for_that_head_only():
    import linear_hybrid_attention_b200 as zb
    g = torch.Generator(device="cuda").manual_seed(31)
    H, R = 2, 256
    X = torch.randn(H, R, 64, generator=g, device="cuda")
    X[1] = X[1, :1].expand(R, 64)      # head 1: every calibration row the same
    Y = torch.randn(H, R, 64, generator=g, device="cuda")
    A, b = zb.zb_affine_fit(X, Y)
    assert _status() == ZB_ERR_SINGULAR
    assert bool(torch.isnan(A[1]).all()) and bool(torch.isnan(b[1]).all())
    A_ref, b_ref = oracle.affine_fit(X[:1].double().cpu().numpy(), Y[:1].double().cpu().numpy())
    np.testing.assert_allclose(A[0].cpu().numpy(), A_ref[0], rtol=0, atol=1e-4 * np.abs(A_ref).max())
    np.testing.assert_allclose(b[0].cpu().numpy(), b_ref[0], rtol=0, atol=1e-4 * np.abs(b_ref).max() + 1e-6)


def _timeout_child():
    """Run in a child process with ZB_WAIT_TIMEOUT_NS=100: one tile-sparse call
    (no landmarks, index lists from the oracle, so no other kernel of the
    library runs under the short limit) with 40 steps per work item, so the
    producers' rings fill and they idle; wave synchronisation on.  Prints the
    statuses as JSON."""
    import linear_hybrid_attention_b200 as zb
    torch.cuda.set_device(0)
    w = workload("views32", heads=2, n_tokens=20000)   # T = 157 tiles of 128
    Q, K, V = synth.make_qkv(w, device="cuda")
    Q64, K64 = host(Q), host(K)
    idx = oracle.select_tiles(oracle.tile_scores(oracle.landmark_means(Q64, w.tile),
                                                 oracle.landmark_means(K64, w.tile)), 40)
    idx = torch.from_numpy(idx.astype(np.int32)).cuda()
    torch.cuda.synchronize()
    before = _status()
    O = torch.zeros_like(Q)
    zb.zb_tile_sparse_attn(Q, K, V, None, None, idx, 40, w.tile, use_landmarks=False, out=O, wave_sync=True)
    first = _status()
    second = _status()
    finite = bool(torch.isfinite(O.float()).all())
    x = torch.arange(1000, device="cuda", dtype=torch.float32)   # the context still works
    usable = float(x.sum().item()) == 499500.0
    print(json.dumps({"before": before, "first": first, "second": second, "finite": finite, "usable": usable}))


def test_wait_timeout_returns_status_and_leaves_context_usable():
    env = dict(os.environ, ZB_WAIT_TIMEOUT_NS="100")
    r = subprocess.run([sys.executable, os.path.abspath(__file__)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["before"] == ZB_OK and res["first"] == ZB_ERR_TIMEOUT, res
    assert res["second"] == ZB_OK, res
    assert res["finite"] and res["usable"], res


if __name__ == "__main__":
    _timeout_child()
