"""GPU parity: the linear-centered variant (each head's keys shifted by their mean
over all tokens before the feature map), through the C ABI against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import REL_TOL, host, check_close, rel_err_per_head, sync_ok, workload

pytestmark = pytest.mark.gpu


def _zb():
    import linear_hybrid_attention_b200 as zb
    return zb


def _offset_keys(K, seed, scale=0.5):
    """K plus one random vector per head, rounded to bf16: keys whose mean is far from zero
    (the synthetic keys alone have a mean near zero, where centring changes little)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    off = scale * torch.randn(K.shape[0], 1, K.shape[2], generator=g, device="cuda")
    return (K.float() + off).to(torch.bfloat16).contiguous()


def _affine(heads, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    A = (torch.eye(64, device="cuda") + 0.1 * torch.randn(heads, 64, 64, generator=g, device="cuda")).contiguous()
    b = (0.01 * torch.randn(heads, 64, generator=g, device="cuda")).contiguous()
    return A, b


@pytest.mark.parametrize("heads,n,offset", [(2, 256, False), (1, 1, True), (5, 130, True),
                                            (3, 5000, True), (16, 43968, True)])
def test_key_mean_matches_oracle(heads, n, offset):
    zb = _zb()
    w = workload("linear256", heads=heads, n_tokens=n)
    _, K, _ = synth.make_qkv(w, device="cuda")
    if offset:
        K = _offset_keys(K, 21)
    mu = zb.zb_key_mean(K)
    sync_ok()
    K64 = host(K)
    ref = oracle.key_mean(K64)
    # fp32 partial sums of at most a few hundred rows each, fp64 across them
    assert np.abs(mu.cpu().numpy() - ref).max() <= 1e-6 * np.abs(K64).max()


@pytest.mark.parametrize("heads,n", [(2, 256), (3, 5000), (16, 43968)])
def test_linear_state_centered_matches_oracle(heads, n):
    zb = _zb()
    w = workload("linear256", heads=heads, n_tokens=n)
    _, K, V = synth.make_qkv(w, device="cuda")
    K = _offset_keys(K, 22)
    mu = zb.zb_key_mean(K)
    S, z = zb.zb_linear_state_centered(K, V, mu)
    sync_ok()
    K64, V64 = host(K), host(V)
    S_ref, z_ref = oracle.linear_state_centered(K64, V64)
    check_close(S.cpu().numpy(), S_ref, tol=1e-2)
    np.testing.assert_allclose(z.cpu().numpy(), z_ref, rtol=5e-3)
    # the shift is not a no-op on these keys
    S_u, _ = oracle.linear_state(K64, V64)
    assert rel_err_per_head(S_u, S_ref) > 0.1


@pytest.mark.parametrize("heads,n,affine", [(2, 300, False), (3, 5000, True), (16, 43968, True)])
def test_linear_attention_centered_matches_oracle(heads, n, affine):
    zb = _zb()
    w = workload("linear256", heads=heads, n_tokens=n)
    Q, K, V = synth.make_qkv(w, device="cuda")
    K = _offset_keys(K, 23)
    A, b = _affine(heads, 6) if affine else (None, None)
    mu = zb.zb_key_mean(K)
    S, z = zb.zb_linear_state_centered(K, V, mu)
    O = zb.zb_linear_apply(Q, S, z, A, b)
    sync_ok()
    ref = oracle.linear_attention_centered(host(Q), host(K), host(V),
                                           None if A is None else A.double().cpu().numpy(),
                                           None if b is None else b.double().cpu().numpy())
    check_close(host(O), ref)


@pytest.mark.parametrize("name,heads,n", [("tiny", None, None), ("linear256", 2, 20000)])
def test_fitted_centered_stage_end_to_end(name, heads, n):
    """HybridLayer(centered=True): key mean, centred state, fit against dense attention on
    the calibration tiles, fitted output on every row, against the oracle doing each step in
    fp64 from the same inputs."""
    zb = _zb()
    w = workload(name) if heads is None else workload(name, heads=heads, n_tokens=n)
    Q, K, V = synth.make_qkv(w, device="cuda")
    K = _offset_keys(K, 25)
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k or 1, calib, centered=True)
    layer.calibrate(Q, K, V)
    o_l = layer.linear(Q, K, V)
    sync_ok()
    Q64, K64, V64 = host(Q), host(K), host(V)
    rows = oracle.calibration_rows(w.n_tokens, w.tile, calib)
    X = oracle.linear_attention_centered(Q64[:, rows], K64, V64)
    Y = oracle.dense_attention(Q64[:, rows], K64, V64, 1 / 8)
    A, b = oracle.affine_fit(X, Y)
    ref = oracle.linear_attention_centered(Q64, K64, V64, A, b)
    check_close(host(o_l), ref)
