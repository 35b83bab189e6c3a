"""GPU parity: linear-attention state and output, affine fit, and the fitted stage."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import REL_TOL, host, check_close, sync_ok, workload

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
    check_close(S.cpu().numpy(), S_ref, tol=1e-2)
    np.testing.assert_allclose(z.cpu().numpy(), z_ref, rtol=5e-3)


@pytest.mark.parametrize("heads,n,affine", [(2, 256, False), (3, 5000, True), (2, 1000, True), (16, 43968, True)])
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
    check_close(host(O), ref)


@pytest.mark.parametrize("heads,n,affine", [(2, 300, False), (3, 5000, True)])
def test_linear_attn_one_call_matches_oracle(heads, n, affine):
    """zb_linear_attn (state + output in one C call) against the fp64 oracle, and
    bit-identical to the two separate calls it is made of."""
    zb = _zb()
    w = workload("linear256", heads=heads, n_tokens=n)
    Q, K, V = synth.make_qkv(w, device="cuda")
    A = b = None
    if affine:
        g = torch.Generator(device="cuda").manual_seed(5)
        A = (torch.eye(64, device="cuda") + 0.1 * torch.randn(heads, 64, 64, generator=g, device="cuda")).contiguous()
        b = (0.01 * torch.randn(heads, 64, generator=g, device="cuda")).contiguous()
    O = zb.zb_linear_attn(Q, K, V, A, b)
    S, z = zb.zb_linear_state(K, V)
    O2 = zb.zb_linear_apply(Q, S, z, A, b)
    sync_ok()
    assert torch.equal(O, O2)
    ref = oracle.linear_attention(host(Q), host(K), host(V),
                                  None if A is None else A.double().cpu().numpy(),
                                  None if b is None else b.double().cpu().numpy())
    check_close(host(O), ref)


def test_affine_fit_matches_oracle_on_same_inputs():
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(11)
    H, R = 4, 1000
    X = torch.randn(H, R, 64, generator=g, device="cuda") * 0.1 + 0.02
    A0 = torch.randn(H, 64, 64, generator=g, device="cuda") * 0.2
    Y = torch.bmm(X, A0) + 0.05 * torch.randn(H, R, 64, generator=g, device="cuda")
    A, b = zb.zb_affine_fit(X, Y)
    sync_ok()
    A_ref, b_ref = oracle.affine_fit(X.double().cpu().numpy(), Y.double().cpu().numpy())
    np.testing.assert_allclose(A.cpu().numpy(), A_ref, rtol=0, atol=1e-4 * np.abs(A_ref).max())
    np.testing.assert_allclose(b.cpu().numpy(), b_ref, rtol=0, atol=1e-4 * np.abs(b_ref).max() + 1e-6)


def test_affine_fit_recovers_planted_map():
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(12)
    H, R = 2, 512
    X = torch.randn(H, R, 64, generator=g, device="cuda")
    A0 = torch.randint(-2, 3, (H, 64, 64), generator=g, device="cuda").float() / 4
    b0 = torch.randint(-4, 5, (H, 64), generator=g, device="cuda").float() / 8
    Y = torch.bmm(X, A0) + b0[:, None, :]
    A, b = zb.zb_affine_fit(X, Y)
    sync_ok()
    np.testing.assert_allclose(A.cpu().numpy(), A0.cpu().numpy(), atol=1e-4)
    np.testing.assert_allclose(b.cpu().numpy(), b0.cpu().numpy(), atol=1e-4)


def test_affine_fit_degenerate_calibration_is_finite():
    # calibration outputs varying in only 3 of 64 directions (plain least squares
    # would be singular): the ridge keeps the fit finite and it still reproduces Y
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(13)
    H, R = 2, 700
    basis = torch.randn(3, 64, generator=g, device="cuda")
    X = torch.randn(H, R, 3, generator=g, device="cuda") @ basis + 0.5
    A0 = torch.randn(H, 64, 64, generator=g, device="cuda") * 0.1
    Y = torch.bmm(X, A0) + 0.2
    A, b = zb.zb_affine_fit(X, Y)
    sync_ok()
    assert torch.isfinite(A).all() and torch.isfinite(b).all()
    fit = torch.bmm(X, A) + b[:, None, :]
    assert (fit - Y).abs().max().item() <= 1e-3 * Y.abs().max().item()


def test_affine_fit_recovers_planted_map_to_the_ridge_bias():
    # Y = X A0 + b0 in fp64, rounded once to fp32.  The fp64 solve returns A0, b0
    # up to the ridge's relative bias (1e-8 * max diag G / s_min^2, about 2e-8
    # here) and the fp32 roundings of Y and of the result (about 1e-7).
    zb = _zb()
    rng = np.random.default_rng(41)
    H, R = 2, 2048
    X = rng.standard_normal((H, R, 64)).astype(np.float32)
    A0 = rng.standard_normal((H, 64, 64)) * 0.2
    b0 = rng.standard_normal((H, 64))
    Y = (X.astype(np.float64) @ A0 + b0[:, None, :]).astype(np.float32)
    A, b = zb.zb_affine_fit(torch.from_numpy(X).cuda(), torch.from_numpy(Y).cuda())
    sync_ok()
    np.testing.assert_allclose(A.cpu().numpy(), A0, rtol=0, atol=1e-5)
    np.testing.assert_allclose(b.cpu().numpy(), b0, rtol=0, atol=1e-5)


def test_affine_fit_rank_deficient_gives_the_minimum_norm_solution():
    # Centred calibration rows of rank 40 < 64 (explicit SVD, singular values
    # 1..10): every least-squares minimiser fits Y, and the ridge picks the one
    # of minimum norm, A_mn = P A* with P the projector on the rows' span and
    # b = b* + xm (I - P) A* (closed form).  X and Y are rounded to fp32 once,
    # which adds directions far below the ridge's cut (1e-4 of the largest).
    zb = _zb()
    rng = np.random.default_rng(42)
    H, R, d, r = 2, 1024, 64, 40
    Xs, Ys, As, bs = [], [], [], []
    for _ in range(H):
        U, _ = np.linalg.qr(rng.standard_normal((R, r)))
        U -= U.mean(axis=0)
        U, _ = np.linalg.qr(U)
        Vr, _ = np.linalg.qr(rng.standard_normal((d, r)))
        xm = rng.standard_normal(d)
        X = xm + (U * np.linspace(1.0, 10.0, r)) @ Vr.T
        A0 = rng.standard_normal((d, d))
        b0 = rng.standard_normal(d)
        P = Vr @ Vr.T
        Xs.append(X)
        Ys.append(X @ A0 + b0)
        As.append(P @ A0)
        bs.append(b0 + xm @ (np.eye(d) - P) @ A0)
    X32 = np.stack(Xs).astype(np.float32)
    Y32 = np.stack(Ys).astype(np.float32)
    A, b = zb.zb_affine_fit(torch.from_numpy(X32).cuda(), torch.from_numpy(Y32).cuda())
    sync_ok()
    A_mn, b_mn = np.stack(As), np.stack(bs)
    np.testing.assert_allclose(A.cpu().numpy(), A_mn, rtol=0, atol=1e-4 * np.abs(A_mn).max())
    np.testing.assert_allclose(b.cpu().numpy(), b_mn, rtol=0, atol=1e-4 * np.abs(b_mn).max())
    fit = oracle.affine_apply(X32.astype(np.float64), A.double().cpu().numpy(), b.double().cpu().numpy())
    assert np.abs(fit - np.stack(Ys)).max() <= 1e-5 * np.abs(np.stack(Ys)).max()


def test_linear_apply_fp32_matches_oracle():
    zb = _zb()
    w = workload("linear256", heads=3, n_tokens=5000)
    Q, K, V = synth.make_qkv(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(4)
    A = (torch.eye(64, device="cuda") + 0.1 * torch.randn(3, 64, 64, generator=g, device="cuda")).contiguous()
    b = (0.01 * torch.randn(3, 64, generator=g, device="cuda")).contiguous()
    S, z = zb.zb_linear_state(K, V)
    for AA, bb in ((None, None), (A, b)):
        O = zb.zb_linear_apply(Q, S, z, AA, bb, out_fp32=True)
        sync_ok()
        ref = oracle.linear_attention(host(Q), host(K), host(V),
                                      None if AA is None else AA.double().cpu().numpy(),
                                      None if bb is None else bb.double().cpu().numpy())
        check_close(O.double().cpu().numpy(), ref)


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
    check_close(host(o_s), oracle.sparse_attention(Q64, K64, V64, w.tile, idx, s))
    rows = oracle.calibration_rows(w.n_tokens, w.tile, calib)
    X = oracle.linear_attention(Q64[:, rows], K64, V64)
    Y = oracle.dense_attention(Q64[:, rows], K64, V64, s)
    A, b = oracle.affine_fit(X, Y)
    ref = oracle.linear_attention(Q64, K64, V64, A, b)
    check_close(host(o_l), ref)


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
    check_close(host(o_l), ref)


def _oracle_fitted_linear(Q64, K64, V64, tile, calib, heads, sample_tiles):
    """Oracle fitted linear stage on selected heads: fit on the calibration rows
    (dense rows evaluated in chunks), output on sampled query tiles."""
    rows = oracle.calibration_rows(Q64.shape[1], tile, calib)
    out = {}
    for h in heads:
        q, k, v = Q64[h:h + 1], K64[h:h + 1], V64[h:h + 1]
        X = oracle.linear_attention(q[:, rows], k, v)
        Y = np.concatenate([oracle.dense_attention(q[:, rows[c:c + 256]], k, v, 1 / 8)
                            for c in range(0, len(rows), 256)], axis=1)
        A, b = oracle.affine_fit(X, Y)
        srows = oracle.calibration_rows(Q64.shape[1], tile, sample_tiles)
        out[h] = (srows, oracle.linear_attention(q[:, srows], k, v, A, b)[0])
    return out


def test_fitted_linear_stage_full_256_views_sampled():
    """The 256-view linear workload at full size (16 heads x 351,744 tokens, fit on
    4,096 calibration rows): the whole stage on the GPU, the oracle on 3 heads
    (fit in full, outputs on sampled query tiles including the last)."""
    zb = _zb()
    w = workload("linear256")
    Q, K, V = synth.make_qkv(w, device="cuda")
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, 1, calib)
    layer.calibrate(Q, K, V)
    o_l = layer.linear(Q, K, V)
    sync_ok()
    heads = [0, 7, 15]
    sample = [0, 1000, w.n_tiles - 1]
    Q64, K64, V64 = (host(t[heads]) for t in (Q, K, V))
    ref = _oracle_fitted_linear(Q64, K64, V64, w.tile, calib, range(len(heads)), sample)
    for slot, h in enumerate(heads):
        srows, want = ref[slot]
        got = host(o_l[h:h + 1, srows])[0]
        check_close(got[None], want[None], label=f"head {h}")


def test_saved_fit_reproduces_the_linear_stage_on_new_inputs(tmp_path):
    """A fit saved by one layer and loaded by another gives the same linear output on a new
    input, bit for bit, with no calibration in the second layer."""
    zb = _zb()
    w = workload("linear256", heads=2, n_tokens=5000)
    Q, K, V = synth.make_qkv(w, device="cuda")
    calib = synth.calibration_tiles(w.n_tiles, 4)
    first = zb.HybridLayer(w.heads, w.n_tokens, w.tile, 1, calib)
    first.calibrate(Q, K, V)
    path = tmp_path / "fit.npz"
    first.save_fit(path)
    Q2, K2, V2 = synth.make_qkv(w, layer=1, device="cuda")   # another input of the same shape
    want = first.linear(Q2, K2, V2, refresh_state=True).clone()
    second = zb.HybridLayer(w.heads, w.n_tokens, w.tile, 1, calib)
    second.load_fit(path)
    got = second.linear(Q2, K2, V2, refresh_state=True)
    sync_ok()
    assert torch.equal(got, want)
