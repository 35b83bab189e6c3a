"""GPU parity: linear-attention state and output, affine fit, and the fitted stage."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import REL_TOL, host, rel_err_per_head, sync_ok, workload

pytestmark = pytest.mark.gpu


def _zb():
    import linear_hybrid_attention_b200 as zb
    return zb


def _phi_bf16(x64):
    # phi rounded to bf16, as the state kernel feeds the tensor core
    f = oracle.elu_plus_one(x64)
    return torch.from_numpy(f).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("heads,n", [(2, 256), (3, 5000), (16, 43968)])
def test_linear_state_matches_oracle(heads, n):
    zb = _zb()
    w = workload("linear256", heads=heads, n_tokens=n)
    Q, K, V = synth.make_qkv(w, device="cuda")
    S, z = zb.zb_linear_state(K, V)
    sync_ok()
    S_ref, z_ref = oracle.linear_state(host(K), host(V))
    assert rel_err_per_head(S.cpu().numpy(), S_ref) <= 1e-2
    np.testing.assert_allclose(z.cpu().numpy(), z_ref, rtol=5e-3)


@pytest.mark.parametrize("heads,n,affine", [(2, 256, False), (3, 5000, True), (16, 43968, True)])
def test_linear_attention_matches_oracle(heads, n, affine):
    zb = _zb()
    w = workload("linear256", heads=heads, n_tokens=n)
    Q, K, V = synth.make_qkv(w, device="cuda")
    A = b = None
    if affine:
        g = torch.Generator(device="cuda").manual_seed(3)
        A = (torch.eye(64, device="cuda") + 0.1 * torch.randn(heads, 64, 64, generator=g, device="cuda")).contiguous()
        b = (0.01 * torch.randn(heads, 64, generator=g, device="cuda")).contiguous()
    S, z = zb.zb_linear_state(K, V)
    O = zb.zb_linear_apply(Q, S, z, A, b)
    sync_ok()
    ref = oracle.linear_attention(host(Q), host(K), host(V),
                                  None if A is None else A.double().cpu().numpy(),
                                  None if b is None else b.double().cpu().numpy())
    assert rel_err_per_head(host(O), ref) <= REL_TOL


def test_affine_fit_matches_oracle_on_same_inputs():
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(11)
    H, R = 4, 1000
    X = (torch.randn(H, R, 64, generator=g, device="cuda") * 0.1 + 0.02).to(torch.bfloat16)
    A0 = torch.randn(H, 64, 64, generator=g, device="cuda") * 0.2
    Y = (torch.bmm(X.float(), A0) + 0.05 * torch.randn(H, R, 64, generator=g, device="cuda")).to(torch.bfloat16)
    A, b = zb.zb_affine_fit(X, Y)
    sync_ok()
    A_ref, b_ref = oracle.affine_fit(host(X), host(Y))
    np.testing.assert_allclose(A.cpu().numpy(), A_ref, rtol=0, atol=1e-4 * np.abs(A_ref).max())
    np.testing.assert_allclose(b.cpu().numpy(), b_ref, rtol=0, atol=1e-4 * np.abs(b_ref).max() + 1e-6)


def test_affine_fit_recovers_planted_map():
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(12)
    H, R = 2, 512
    X = torch.randn(H, R, 64, generator=g, device="cuda").to(torch.bfloat16)
    # A0 with small-integer entries and b0 so that Y = X A0 + b0 is exact in bf16?  Not in
    # general; compare against the oracle fit of the rounded Y instead, and check the fit
    # is close to the planted map.
    A0 = torch.randint(-2, 3, (H, 64, 64), generator=g, device="cuda").float() / 4
    b0 = torch.randint(-4, 5, (H, 64), generator=g, device="cuda").float() / 8
    Y = (torch.bmm(X.float(), A0) + b0[:, None, :]).to(torch.bfloat16)
    A, b = zb.zb_affine_fit(X, Y)
    sync_ok()
    A_ref, b_ref = oracle.affine_fit(host(X), host(Y))
    np.testing.assert_allclose(A.cpu().numpy(), A_ref, atol=1e-4)
    np.testing.assert_allclose(A.cpu().numpy(), A0.cpu().numpy(), atol=2e-2)
    np.testing.assert_allclose(b.cpu().numpy(), b0.cpu().numpy(), atol=2e-2)


def test_fitted_linear_stage_tiny_end_to_end():
    """HybridLayer on the tiny case: sparse output, fitted linear output vs the oracle
    computing every step in fp64 from the same inputs."""
    zb = _zb()
    w = workload("tiny")
    Q, K, V = synth.make_qkv(w, device="cuda")
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, calib)
    o_s, o_l = layer.step(Q, K, V)
    sync_ok()
    Q64, K64, V64 = host(Q), host(K), host(V)
    s = 1 / 8
    idx = oracle.select_tiles(oracle.tile_scores(oracle.landmark_means(Q64, w.tile),
                                                 oracle.landmark_means(K64, w.tile)), w.k)
    assert rel_err_per_head(host(o_s), oracle.sparse_attention(Q64, K64, V64, w.tile, idx, s)) <= REL_TOL
    rows = oracle.calibration_rows(w.n_tokens, w.tile, calib)
    X = oracle.linear_attention(Q64[:, rows], K64, V64)
    Y = oracle.dense_attention(Q64[:, rows], K64, V64, s)
    A, b = oracle.affine_fit(X, Y)
    ref = oracle.linear_attention(Q64, K64, V64, A, b)
    assert rel_err_per_head(host(o_l), ref) <= REL_TOL


def test_fitted_linear_stage_calibration_rows():
    """linear256 recipe at a reduced length: the fitted stage on all rows vs the oracle."""
    zb = _zb()
    w = workload("linear256", heads=2, n_tokens=20000)
    Q, K, V = synth.make_qkv(w, device="cuda")
    calib = synth.calibration_tiles(w.n_tiles, 32)
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, 1, calib)
    layer.calibrate(Q, K, V)
    o_l = layer.linear(Q, K, V)
    sync_ok()
    Q64, K64, V64 = host(Q), host(K), host(V)
    rows = oracle.calibration_rows(w.n_tokens, w.tile, calib)
    X = oracle.linear_attention(Q64[:, rows], K64, V64)
    Y = oracle.dense_attention(Q64[:, rows], K64, V64, 1 / 8)
    A, b = oracle.affine_fit(X, Y)
    ref = oracle.linear_attention(Q64, K64, V64, A, b)
    err = rel_err_per_head(host(o_l), ref)
    assert err <= REL_TOL, err
