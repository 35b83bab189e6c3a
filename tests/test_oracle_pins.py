"""Pins for the fp64 oracle: closed forms, invariants, library routines, brute force.

Each test ties one oracle function to something other than itself, chosen so
that a plausible slip (a dropped term, a wrong sign or index, a transposed
operand, a wrong log base) fails at least one test.  CPU only.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth

RNG = np.random.default_rng(12345)


def _bf16_grid(shape, std=1.0, rng=RNG):
    """Random values that are exactly representable in bf16 (as fp64)."""
    x = torch.from_numpy(rng.standard_normal(shape) * std).to(torch.bfloat16)
    return x.to(torch.float64).numpy()


# ----------------------------------------------------------------- tiles ----

def test_tile_lengths_closed_form():
    assert oracle.tile_lengths(256, 64).tolist() == [64, 64, 64, 64]
    n = oracle.tile_lengths(32 * 1374, 128)
    assert n.shape == (344,) and n[-1] == 43968 - 343 * 128 == 64
    assert (n[:-1] == 128).all() and n.sum() == 43968
    assert oracle.tile_lengths(1, 128).tolist() == [1]
    assert oracle.tile_lengths(1024 * 1374, 128).shape == (10992,)


def test_landmark_means_equal_correctly_rounded_sums():
    X = _bf16_grid((2, 300, 8), std=0.125)
    got = oracle.landmark_means(X, 64)
    n = oracle.tile_lengths(300, 64)
    for h in range(2):
        for j in range(len(n)):
            rows = X[h, j * 64: j * 64 + n[j]]
            for c in range(8):
                want = math.fsum(rows[:, c].tolist()) / float(n[j])
                assert got[h, j, c] == want  # bit-exact


def test_landmark_means_of_constant_tile():
    X = np.zeros((1, 200, 4))
    X[0, :128] = 0.375
    X[0, 128:] = -1.5
    got = oracle.landmark_means(X, 128)
    assert (got[0, 0] == 0.375).all() and (got[0, 1] == -1.5).all()


# --------------------------------------------------------------- scoring ----

def test_tile_scores_pick_coordinates():
    # Qbar rows are basis vectors, so score[i, j] = Kbar[j, i]; a transposed
    # product or swapped operands gives a different matrix.
    d = 5
    Qbar = np.eye(d)[None]
    Kbar = RNG.standard_normal((1, 7, d))
    s = oracle.tile_scores(Qbar, Kbar)
    assert s.shape == (1, d, 7)
    np.testing.assert_array_equal(s[0], Kbar[0].T)


def test_tile_scores_cauchy_schwarz():
    A = RNG.standard_normal((1, 9, 6))
    s = oracle.tile_scores(A, A)
    norms = (A[0] ** 2).sum(-1)
    np.testing.assert_allclose(np.diag(s[0]), norms, rtol=1e-14)
    assert (np.abs(s[0]) <= np.sqrt(norms[:, None] * norms[None, :]) * (1 + 1e-14)).all()


def test_select_top_k_equals_best_subset_by_brute_force():
    for trial in range(20):
        T, k = 7, 3
        s = RNG.standard_normal(T)
        best = max(itertools.combinations(range(T), k), key=lambda c: sum(s[list(c)]))
        got = oracle.select_tiles(s[None], k)[0]
        assert got.tolist() == sorted(best)


def test_select_tie_break_lower_index_and_ascending():
    row = np.array([[1.0, 3.0, 3.0, 2.0, 3.0]])
    assert oracle.select_tiles(row, 2)[0].tolist() == [1, 2]
    assert oracle.select_tiles(row, 3)[0].tolist() == [1, 2, 4]
    assert oracle.select_tiles(row, 4)[0].tolist() == [1, 2, 3, 4]
    assert oracle.select_tiles(row, 0)[0].tolist() == []
    assert oracle.select_tiles(row, 5)[0].tolist() == [0, 1, 2, 3, 4]
    neg = np.array([[-0.0, 0.0, -1e-300, 1e-300]])
    assert oracle.select_tiles(neg, 1)[0].tolist() == [3]
    assert oracle.select_tiles(neg, 3)[0].tolist() == [0, 1, 3]


def test_select_keeps_planted_tiles_tiny():
    w = synth.WORKLOADS["tiny"]
    Q, K, V = synth.make_qkv(w)
    Qbar = oracle.landmark_means(synth.to_f64(Q), w.tile)
    Kbar = oracle.landmark_means(synth.to_f64(K), w.tile)
    idx = oracle.select_tiles(oracle.tile_scores(Qbar, Kbar), w.k)
    hh, ii, jj = synth.planted_pairs(w, synth.default_seed(w))
    for h, i, j in zip(hh, ii, jj):
        assert j in idx[h, i]


# ------------------------------------------------------ softmax attention ----

def _qkv(H, N, d, std=0.5, rng=RNG):
    return (rng.standard_normal((H, N, d)) * std, rng.standard_normal((H, N, d)) * std,
            rng.standard_normal((H, N, d)))


def test_dense_attention_matches_library_sdpa():
    Q, K, V = _qkv(2, 37, 8)
    s = 1 / math.sqrt(8)
    got = oracle.dense_attention(Q, K, V, s)
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0]
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-12, atol=1e-13)


def test_keep_all_tiles_equals_dense():
    H, N, d, t = 2, 150, 8, 32   # ragged last tile (22 rows)
    Q, K, V = _qkv(H, N, d)
    T = oracle.tile_lengths(N, t).shape[0]
    idx = np.broadcast_to(np.arange(T), (H, T, T))
    got = oracle.sparse_attention(Q, K, V, t, idx, 0.125, use_landmarks=True)
    np.testing.assert_allclose(got, oracle.dense_attention(Q, K, V, 0.125), rtol=1e-12, atol=1e-14)


def test_tile_length_one_makes_landmarks_exact():
    H, N, d = 1, 40, 4
    Q, K, V = _qkv(H, N, d)
    for k in (0, 1, 7, 40):
        idx = np.stack([np.sort(RNG.choice(N, size=k, replace=False)) for _ in range(N)])[None]
        got = oracle.sparse_attention(Q, K, V, 1, idx, 0.3, use_landmarks=True)
        np.testing.assert_allclose(got, oracle.dense_attention(Q, K, V, 0.3), rtol=1e-12, atol=1e-14)


def test_tile_constant_keys_make_landmarks_exact_for_any_selection():
    # Every row of a key tile is the same vector, so a landmark (mean key, mean
    # value, bias ln n_j) reproduces the tile's n_j exact keys.  Values are not
    # tile-constant.  The last tile is ragged.
    H, N, d, t = 2, 200, 8, 32
    T = oracle.tile_lengths(N, t).shape[0]
    Q, _, V = _qkv(H, N, d)
    Kt = RNG.standard_normal((H, T, d))
    K = np.repeat(Kt, t, axis=1)[:, :N]
    dense = oracle.dense_attention(Q, K, V, 0.25)
    for k in (0, 1, 3, T):
        idx = np.stack([np.stack([np.sort(RNG.choice(T, size=k, replace=False)) for _ in range(T)])
                        for _ in range(H)])
        got = oracle.sparse_attention(Q, K, V, t, idx, 0.25, use_landmarks=True)
        np.testing.assert_allclose(got, dense, rtol=1e-12, atol=1e-14)


def test_landmarks_only_equal_expanded_mean_keys():
    # k = 0: the output equals dense attention over a key set where each tile's
    # mean key (with its mean value) is repeated n_j times.
    H, N, d, t = 1, 90, 6, 16
    Q, K, V = _qkv(H, N, d)
    n = oracle.tile_lengths(N, t)
    Kb, Vb = oracle.landmark_means(K, t), oracle.landmark_means(V, t)
    Kx = np.repeat(Kb, n, axis=1)
    Vx = np.repeat(Vb, n, axis=1)
    idx = np.zeros((H, len(n), 0), dtype=np.int64)
    got = oracle.sparse_attention(Q, K, V, t, idx, 0.4, use_landmarks=True)
    np.testing.assert_allclose(got, oracle.dense_attention(Q, Kx, Vx, 0.4), rtol=1e-12, atol=1e-14)


def test_no_landmarks_single_tile_is_local_softmax():
    H, N, d, t = 1, 96, 8, 32
    Q, K, V = _qkv(H, N, d)
    T = 3
    idx = np.array([[[2], [0], [1]]])
    got = oracle.sparse_attention(Q, K, V, t, idx, 0.5, use_landmarks=False)
    for i, j in enumerate([2, 0, 1]):
        want = oracle.dense_attention(Q[:, i * t:(i + 1) * t], K[:, j * t:(j + 1) * t],
                                      V[:, j * t:(j + 1) * t], 0.5)
        np.testing.assert_allclose(got[:, i * t:(i + 1) * t], want, rtol=1e-12, atol=1e-14)


def test_sparse_output_is_convex_combination():
    H, N, d, t = 2, 130, 8, 32
    Q, K, V = _qkv(H, N, d, std=2.0)
    T = 5
    idx = np.stack([np.stack([np.sort(RNG.choice(T, size=2, replace=False)) for _ in range(T)])
                    for _ in range(H)])
    O = oracle.sparse_attention(Q, K, V, t, idx, 0.125)
    lo, hi = V.min(axis=1, keepdims=True), V.max(axis=1, keepdims=True)
    assert (O >= lo - 1e-12).all() and (O <= hi + 1e-12).all()


def test_query_tile_subset_matches_full():
    H, N, d, t = 1, 100, 4, 32
    Q, K, V = _qkv(H, N, d)
    T = 4
    idx = np.stack([np.sort(RNG.choice(T, size=2, replace=False)) for _ in range(T)])[None]
    full = oracle.sparse_attention(Q, K, V, t, idx, 0.2)
    sub = oracle.sparse_attention(Q, K, V, t, idx, 0.2, query_tiles=[3, 1])
    np.testing.assert_array_equal(sub[:, :4], full[:, 96:100])
    assert (sub[:, 4:32] == 0).all()
    np.testing.assert_array_equal(sub[:, 32:64], full[:, 32:64])


# --------------------------------------------------------- linear stage ----

def test_elu_plus_one_closed_form():
    x = np.array([-2.0, -0.5, 0.0, 0.5, 3.0])
    want = [math.exp(-2.0), math.exp(-0.5), 1.0, 1.5, 4.0]
    assert oracle.elu_plus_one(x).tolist() == want
    assert (oracle.elu_plus_one(np.linspace(-30, 30, 101)) > 0).all()


def test_linear_associative_equals_quadratic():
    Q, K, V = _qkv(2, 50, 8, std=1.0)
    np.testing.assert_allclose(oracle.linear_attention(Q, K, V),
                               oracle.linear_attention_quadratic(Q, K, V), rtol=1e-12, atol=1e-13)


def test_linear_zero_keys_give_mean_value():
    Q, _, V = _qkv(1, 30, 4)
    O = oracle.linear_attention(Q, np.zeros_like(Q), V)
    np.testing.assert_allclose(O, np.broadcast_to(V.mean(axis=1, keepdims=True), O.shape), rtol=1e-13)


def test_linear_state_single_token():
    Q, K, V = _qkv(1, 1, 4)
    S, z = oracle.linear_state(K, V)
    phik = oracle.elu_plus_one(K[0, 0])
    np.testing.assert_allclose(S[0], np.outer(phik, V[0, 0]), rtol=1e-15)
    np.testing.assert_allclose(z[0], phik, rtol=1e-15)
    np.testing.assert_allclose(oracle.linear_attention(Q, K, V)[0, 0], V[0, 0], rtol=1e-14)


# ------------------------------------------------------ linear-centered ----

def test_key_mean_equals_exact_rational_mean():
    # bf16 inputs: every partial sum is exact in fp64, so the mean is the
    # correctly rounded exact rational mean
    from fractions import Fraction
    H, N, d = 2, 37, 5
    K = _bf16_grid((H, N, d))
    mu = oracle.key_mean(K)
    assert mu.shape == (H, d)
    for h in range(H):
        for c in range(d):
            exact = sum(Fraction(float(v)) for v in K[h, :, c]) / N
            assert mu[h, c] == float(exact)


def test_centered_linear_is_invariant_to_a_key_shift():
    Q, K, V = _qkv(2, 40, 6, std=1.0)
    shift = RNG.standard_normal((2, 1, 6))
    A = RNG.standard_normal((2, 6, 6))
    b = RNG.standard_normal((2, 6))
    O = oracle.linear_attention_centered(Q, K, V, A, b)
    np.testing.assert_allclose(oracle.linear_attention_centered(Q, K + shift, V, A, b), O,
                               rtol=1e-11, atol=1e-12)
    # not vacuous: the uncentred operator does move with the keys
    moved = oracle.linear_attention(Q, K + shift, V) - oracle.linear_attention(Q, K, V)
    assert np.abs(moved).max() > 1e-3


def test_centered_linear_equals_quadratic_form_of_zero_mean_keys():
    # the associative centred operator against the (separately pinned) quadratic
    # form, fed keys whose column means are exactly zero by construction
    Q, _, V = _qkv(2, 25, 8, std=1.0)
    K = _bf16_grid((2, 25, 8))  # bf16 values: the column sums below are exact
    Kz = np.concatenate([K, -K], axis=1)
    Vz = np.concatenate([V, V[:, ::-1]], axis=1)
    np.testing.assert_array_equal(oracle.key_mean(Kz), 0.0)
    np.testing.assert_allclose(oracle.linear_attention_centered(Q, Kz, Vz),
                               oracle.linear_attention_quadratic(Q, Kz, Vz), rtol=1e-12, atol=1e-13)
    # shifted keys: centring must bring back the same output
    shift = RNG.standard_normal((2, 1, 8))
    np.testing.assert_allclose(oracle.linear_attention_centered(Q, Kz + shift, Vz),
                               oracle.linear_attention_quadratic(Q, Kz, Vz), rtol=1e-11, atol=1e-12)


def test_dense_attention_is_invariant_to_a_key_shift():
    # why centring keeps the fit target: softmax ignores a constant per query
    Q, K, V = _qkv(2, 30, 6)
    shift = RNG.standard_normal((2, 1, 6))
    np.testing.assert_allclose(oracle.dense_attention(Q, K + shift, V, 0.3),
                               oracle.dense_attention(Q, K, V, 0.3), rtol=1e-12, atol=1e-13)


# ---------------------------------------------- block-mass diagnostic ----

def test_block_mass_rows_hold_one_unit_per_query():
    # every query row's probabilities sum to 1, so a block row holds its length
    Q, K, _ = _qkv(2, 300, 8, std=1.0)
    M = oracle.block_mass(Q, K, 0.4, 64)
    assert M.shape == (2, 5, 5)
    np.testing.assert_allclose(M.sum(axis=-1), np.broadcast_to(oracle.tile_lengths(300, 64), (2, 5)), rtol=1e-13)
    assert (M >= 0).all()


def test_block_mass_of_uniform_attention():
    # all-zero keys: p = 1/N everywhere, M[a, b] = n_a n_b / N
    Q, _, _ = _qkv(1, 150, 4)
    n = oracle.tile_lengths(150, 64)
    M = oracle.block_mass(Q, np.zeros_like(Q), 0.5, 64)
    np.testing.assert_allclose(M[0], np.outer(n, n) / 150.0, rtol=1e-13)


def test_block_mass_is_attention_with_block_indicator_values():
    # dense attention (pinned against the library's SDPA) with V = the one-hot
    # key-block indicator gives each row's mass per key block; summing the rows
    # of a query block gives M
    H, N, d, B = 2, 130, 8, 64
    Q, K, _ = _qkv(H, N, d, std=1.0)
    T = -(-N // B)
    E = np.zeros((N, T))
    E[np.arange(N), np.arange(N) // B] = 1.0
    R = oracle.dense_attention(Q, K, np.broadcast_to(E, (H, N, T)).copy(), 0.7)
    want = np.stack([np.stack([R[h, a * B:(a + 1) * B].sum(axis=0) for a in range(T)]) for h in range(H)])
    np.testing.assert_allclose(oracle.block_mass(Q, K, 0.7, B), want, rtol=1e-12, atol=1e-14)
    # block size 1: the probability matrix itself
    np.testing.assert_allclose(oracle.block_mass(Q[:, :9], K[:, :9], 0.7, 1),
                               oracle.dense_attention(Q[:, :9], K[:, :9], np.broadcast_to(np.eye(9), (H, 9, 9)).copy(), 0.7),
                               rtol=1e-12, atol=1e-14)


def test_top_mass_fraction_is_the_best_subset():
    M = RNG.random((2, 3, 7))
    for m in range(0, 8):
        got = oracle.top_mass_fraction(M, m)
        for h in range(2):
            for a in range(3):
                best = max((sum(M[h, a, list(c)]) for c in itertools.combinations(range(7), m)), default=0.0)
                assert abs(got[h, a] - best / M[h, a].sum()) <= 1e-14


def test_selected_mass_fraction_of_the_top_tiles_and_of_all():
    M = RNG.random((2, 4, 6))
    idx = np.sort(np.argsort(-M, axis=-1)[..., :2], axis=-1)
    np.testing.assert_allclose(oracle.selected_mass_fraction(M, idx), oracle.top_mass_fraction(M, 2), rtol=1e-14)
    every = np.broadcast_to(np.arange(6), (2, 4, 6))
    np.testing.assert_allclose(oracle.selected_mass_fraction(M, every), 1.0, rtol=1e-14)
    # one hand-worked row
    M1 = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    assert oracle.selected_mass_fraction(M1, np.array([[[0, 2]]]))[0, 0] == 0.4


# ----------------------------------------------------------- affine fit ----

def test_affine_fit_recovers_planted_map():
    H, R, d = 3, 400, 8
    X = RNG.standard_normal((H, R, d))
    A0 = RNG.standard_normal((H, d, d))
    b0 = RNG.standard_normal((H, d))
    Y = oracle.affine_apply(X, A0, b0)
    A, b = oracle.affine_fit(X, Y)
    # the vanishing ridge (1e-8 relative) biases A by O(1e-8)
    np.testing.assert_allclose(A, A0, rtol=0, atol=1e-6)
    np.testing.assert_allclose(b, b0, rtol=0, atol=1e-6)
    A, b = oracle.affine_fit(X, Y, ridge_rel=0.0)
    np.testing.assert_allclose(A, A0, rtol=0, atol=1e-10)
    np.testing.assert_allclose(b, b0, rtol=0, atol=1e-10)


def test_affine_fit_identity():
    X = RNG.standard_normal((2, 100, 6))
    A, b = oracle.affine_fit(X, X, ridge_rel=0.0)
    np.testing.assert_allclose(A, np.broadcast_to(np.eye(6), A.shape), atol=1e-12)
    np.testing.assert_allclose(b, 0, atol=1e-12)


def test_affine_fit_normal_equations_with_ridge():
    # stationarity of ||[X 1] W - Y||^2 + lam ||A||^2:  [X 1]^T E = [lam A; 0]
    X = RNG.standard_normal((2, 300, 5))
    Y = RNG.standard_normal((2, 300, 5))
    for rr in (0.0, 1e-8, 1e-2):
        A, b = oracle.affine_fit(X, Y, ridge_rel=rr)
        E = Y - oracle.affine_apply(X, A, b)
        for h in range(2):
            Xc = X[h] - X[h].mean(0)
            lam = rr * (Xc * Xc).sum(0).max()
            D = np.concatenate([X[h], np.ones((300, 1))], axis=1)
            want = np.concatenate([lam * A[h], np.zeros((1, 5))], axis=0)
            np.testing.assert_allclose(D.T @ E[h], want, atol=1e-9)


def test_affine_fit_rank_deficient_calibration_is_finite():
    # outputs varying in only 2 of 6 directions: plain least squares is singular,
    # the vanishing ridge gives the minimum-norm-like finite solution that still
    # reproduces Y on the calibration rows
    H, R, d = 1, 200, 6
    basis = RNG.standard_normal((2, d))
    X = (RNG.standard_normal((H, R, 2)) @ basis) + 0.3
    A0 = RNG.standard_normal((H, d, d))
    Y = oracle.affine_apply(X, A0, np.ones((H, d)))
    A, b = oracle.affine_fit(X, Y)
    assert np.isfinite(A).all() and np.abs(A).max() < 1e3
    np.testing.assert_allclose(oracle.affine_apply(X, A, b), Y, atol=1e-6)


def _rank_deficient_case(seed, R=300, d=16, r=10):
    """X with centred rank r < d built from an explicit SVD Xc = U_r diag(s) V_r^T
    (singular values 1..10), and Y = X A* + b* exactly, for a planted A* that has
    components in the null space of Xc too."""
    rng = np.random.default_rng(seed)
    U, _ = np.linalg.qr(rng.standard_normal((R, r)))
    U -= U.mean(axis=0)                      # columns orthogonal to the all-ones vector
    U, _ = np.linalg.qr(U)
    Vr, _ = np.linalg.qr(rng.standard_normal((d, r)))
    s = np.linspace(1.0, 10.0, r)
    xm = rng.standard_normal(d)
    X = xm + (U * s) @ Vr.T
    A0 = rng.standard_normal((d, d))
    b0 = rng.standard_normal(d)
    Y = X @ A0 + b0
    return X, Y, xm, Vr, A0, b0


def test_affine_fit_rank_deficient_is_the_minimum_norm_solution():
    # With centred rank r < d the least-squares minimisers form an affine family;
    # the minimum-norm one has A_mn = P A* (P = V_r V_r^T, the projector on the
    # row space of Xc) and b = b* + xm (I - P) A*, in closed form.  The ridge
    # (lam -> 0) converges to it: its bias is lam / s_i^2 <= 1e-8 * (10 / 1)^2.
    for seed in (1, 2):
        X, Y, xm, Vr, A0, b0 = _rank_deficient_case(seed)
        P = Vr @ Vr.T
        A_mn = P @ A0
        b_mn = b0 + xm @ (np.eye(len(xm)) - P) @ A0
        A, b = oracle.affine_fit(X[None], Y[None])
        np.testing.assert_allclose(A[0], A_mn, rtol=0, atol=1e-5 * np.abs(A_mn).max())
        np.testing.assert_allclose(b[0], b_mn, rtol=0, atol=1e-5 * np.abs(b_mn).max())
        # fitted rows: the ridge's relative bias is at most 1e-8 * (s_max / s_min)^2 = 1e-6
        np.testing.assert_allclose(oracle.affine_apply(X[None], A, b)[0], Y, rtol=0, atol=2e-6 * np.abs(Y).max())


def test_linear_output_lies_on_a_hyperplane_and_the_fit_ignores_its_normal():
    # O_r = u_r S with u_r = phi(q_r) / (phi(q_r) . z), and u_r . z = 1, so every
    # linear-attention output row satisfies O_r . (S^-1 z) = 1: the centred
    # calibration matrix X is rank-deficient by one for this operator, and the
    # fitted A (the minimum-norm minimiser) has no component along v = S^-1 z.
    rng = np.random.default_rng(5)
    H, N, d = 2, 600, 16
    Q = rng.standard_normal((H, N, d)) / 4
    K = rng.standard_normal((H, N, d)) / 4
    V = rng.standard_normal((H, N, d))
    S, z = oracle.linear_state(K, V)
    X = oracle.linear_attention(Q[:, :200], K, V)
    Y = oracle.dense_attention(Q[:, :200], K, V, 0.25)
    A, _ = oracle.affine_fit(X, Y)
    for h in range(H):
        v = np.linalg.solve(S[h], z[h])
        np.testing.assert_allclose(X[h] @ v, 1.0, rtol=0, atol=1e-9)
        vn = v / np.linalg.norm(v)
        assert np.abs(vn @ A[h]).max() <= 1e-6 * np.abs(A[h]).max()


def test_calibration_rows():
    rows = oracle.calibration_rows(200, 64, [3, 0])
    assert rows.tolist() == list(range(192, 200)) + list(range(0, 64))
    assert synth.calibration_tiles(2748, 32)[:3].tolist() == [0, 85, 171]
    assert synth.calibration_tiles(4, None).tolist() == [0, 1, 2, 3]


# ------------------------------------------------------- spatial tiles ----

def test_spatial_order_hand_worked_small_grid():
    # 5 x 5 patches after 1 special token, windows of 2 x 3 patches, worked by
    # hand from the definition: window rows {0,1}, {2,3}, {4}; window columns
    # {0,1,2}, {3,4}; patch (y, x) is token 1 + 5 y + x
    want = [0, 1, 2, 3, 6, 7, 8, 4, 5, 9, 10, 11, 12, 13, 16, 17, 18, 14, 15, 19, 20,
            21, 22, 23, 24, 25]
    got = oracle.spatial_order(2, grid=5, specials=1, win_rows=2, win_cols=3)
    assert got[:26].tolist() == want
    assert got[26:].tolist() == [26 + t for t in want]


def test_spatial_order_is_a_permutation_with_compact_windows():
    views, grid, sp = 3, 37, 5
    order = oracle.spatial_order(views)
    N = views * (sp + grid * grid)
    assert sorted(order.tolist()) == list(range(N))
    X = RNG.standard_normal((2, N, 3))
    np.testing.assert_array_equal(X[:, order][:, oracle.inverse_order(order)], X)
    per_view = sp + grid * grid
    for v in range(views):
        seg = order[v * per_view:(v + 1) * per_view] - v * per_view
        assert seg[:sp].tolist() == list(range(sp))          # specials first, inside their view
        y, x = np.divmod(seg[sp:] - sp, grid)
        # each of the 4 full-height window rows holds 8 x 16 + 8 x 16 + 8 x 5 = 296
        # patches; its first two windows are full (128 patches each, a contiguous run
        # covering an 8 x 16 rectangle), the third is the ragged right edge
        for wy in range(4):
            for wx, width in ((0, 128), (128, 128), (256, 40)):
                a = 296 * wy + wx
                yy, xx = y[a:a + width], x[a:a + width]
                assert yy.min() == 8 * wy and yy.max() == 8 * wy + 7
                assert xx.max() - xx.min() == (15 if width == 128 else 4)
        assert len(seg) == per_view


def test_spatial_sparse_attention_keep_all_is_dense_and_identity_order_is_plain():
    H, views, grid, sp, t = 2, 2, 7, 1, 16
    N = views * (sp + grid * grid)
    Q, K, V = _qkv(H, N, 8)
    order = oracle.spatial_order(views, grid=grid, specials=sp, win_rows=4, win_cols=4)
    T = len(oracle.tile_lengths(N, t))
    O, idx = oracle.spatial_sparse_attention(Q, K, V, t, order, 0.3, k=T)
    np.testing.assert_allclose(O, oracle.dense_attention(Q, K, V, 0.3), rtol=1e-12, atol=1e-14)
    ident = np.arange(N)
    O1, idx1 = oracle.spatial_sparse_attention(Q, K, V, t, ident, 0.3, k=2)
    want_idx = oracle.select_tiles(oracle.tile_scores(oracle.landmark_means(Q, t), oracle.landmark_means(K, t)), 2)
    np.testing.assert_array_equal(idx1, want_idx)
    np.testing.assert_array_equal(O1, oracle.sparse_attention(Q, K, V, t, want_idx, 0.3))
    # with a real reordering and k < T the result differs from the plain tiling
    O2, _ = oracle.spatial_sparse_attention(Q, K, V, t, order, 0.3, k=2)
    assert np.abs(O2 - O1).max() > 1e-6
