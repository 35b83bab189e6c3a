"""GPU parity: landmarks (bit-exact fp64 means) and tile selection (bit-exact sets)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import bf16_round_f64, host, sync_ok, workload

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", {}),                                       # t = 64, T = 4, k = 2
    ("views32", {"heads": 3, "n_tokens": 5000}),        # ragged last tile (8 rows), odd heads
    ("views32", {}),                                    # full 32-view stage: T = 344, k = 69
]


def _ids(c):
    return c[0] + ("-" + "-".join(f"{k}{v}" for k, v in c[1].items()) if c[1] else "")


@pytest.fixture(scope="module", params=CASES, ids=[_ids(c) for c in CASES])
def case(request):
    import linear_hybrid_attention_b200 as zb
    name, over = request.param
    w = workload(name, **over)
    Q, K, V = synth.make_qkv(w, device="cuda")
    lm = zb.zb_landmark_build(Q, K, V, w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, w.k)
    sync_ok()
    Qb = oracle.landmark_means(host(Q), w.tile)
    Kb = oracle.landmark_means(host(K), w.tile)
    Vb = oracle.landmark_means(host(V), w.tile)
    return w, (Q, K, V), lm, idx, (Qb, Kb, Vb)


def test_landmark_means_bit_exact(case):
    w, _, lm, _, (Qb, Kb, Vb) = case
    assert np.array_equal(lm.Qbar.cpu().numpy(), Qb)
    assert np.array_equal(lm.Kbar.cpu().numpy(), Kb)


def test_landmark_bf16_correctly_rounded(case):
    w, _, lm, _, (Qb, Kb, Vb) = case
    assert np.array_equal(host(lm.Kbar_bf16), bf16_round_f64(Kb))
    assert np.array_equal(host(lm.Vbar_bf16), bf16_round_f64(Vb))


def test_selection_bit_exact(case):
    w, _, _, idx, (Qb, Kb, _) = case
    ref = oracle.select_tiles(oracle.tile_scores(Qb, Kb), w.k)
    got = idx.cpu().numpy().astype(np.int64)
    if not np.array_equal(got, ref):
        bad = np.argwhere((got != ref).any(-1))
        scores = oracle.tile_scores(Qb, Kb)
        h, i = bad[0]
        s = np.sort(scores[h, i])[::-1]
        raise AssertionError(f"{len(bad)} rows differ; first (h={h}, i={i}); k-th/k+1-th score gap "
                             f"{s[w.k - 1] - s[w.k]:.3e}")


def test_selection_keeps_planted_tiles_tiny():
    import linear_hybrid_attention_b200 as zb
    w = workload("tiny")
    Q, K, V = synth.make_qkv(w, device="cuda")
    lm = zb.zb_landmark_build(Q, K, V, w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, w.k).cpu().numpy()
    hh, ii, jj = synth.planted_pairs(w, synth.default_seed(w))
    for h, i, j in zip(hh, ii, jj):
        assert j in idx[h, i]


@pytest.mark.parametrize("k", [1, 17, 39, 40])
def test_selection_edge_budgets(k):
    import linear_hybrid_attention_b200 as zb
    w = workload("views32", heads=2, n_tokens=5000)
    Q, K, V = synth.make_qkv(w, device="cuda", seed=77)
    lm = zb.zb_landmark_build(Q, K, V, w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, k)
    sync_ok()
    ref = oracle.select_tiles(oracle.tile_scores(oracle.landmark_means(host(Q), w.tile),
                                                 oracle.landmark_means(host(K), w.tile)), k)
    assert np.array_equal(idx.cpu().numpy(), ref)


def test_selection_ties_go_to_lower_index():
    # zero queries: every score is 0 (or -0), so the k lowest indices are kept
    import linear_hybrid_attention_b200 as zb
    H, N, t, k = 2, 1000, 64, 5
    Qbar = torch.zeros(H, 16, 64, dtype=torch.float64, device="cuda")
    Kbar = torch.randn(H, 16, 64, dtype=torch.float64, device="cuda")
    Qbar[1, :, 0] = -0.0
    idx = zb.zb_tile_score_topk(Qbar, Kbar, N, t, k)
    sync_ok()
    assert (idx.cpu() == torch.arange(k, dtype=torch.int32)).all()


def test_gather_tiles():
    import linear_hybrid_attention_b200 as zb
    w = workload("views32", heads=2, n_tokens=1000)   # T = 8, last tile 104 rows
    Q, _, _ = synth.make_qkv(w, device="cuda")
    tiles = torch.tensor([7, 0, 3], dtype=torch.int32, device="cuda")
    out = zb.zb_gather_tiles(Q, w.tile, tiles)
    sync_ok()
    q = Q.cpu()
    o = out.cpu()
    assert torch.equal(o[:, :104], q[:, 896:1000])
    assert (o[:, 104:128] == 0).all()
    assert torch.equal(o[:, 128:256], q[:, 0:128])
    assert torch.equal(o[:, 256:384], q[:, 384:512])


# ---- the boundary of the selection: near ties, wide bands, exact ties, extreme rows
def _select_gpu(Qb, Kb, tile, k):
    import linear_hybrid_attention_b200 as zb
    H, T, _ = Qb.shape
    idx = zb.zb_tile_score_topk(torch.from_numpy(Qb).cuda(), torch.from_numpy(Kb).cuda(), T * tile, tile, k)
    sync_ok()
    return idx.cpu().numpy().astype(np.int64)


def _cluster_case(T, n_cluster, spread, seed):
    # every query row has a positive first component; the cluster's key rows are one
    # large vector plus perturbations of relative size `spread`, so their scores lead
    # every row and only the perturbations order them
    g = np.random.default_rng(seed)
    H = 2
    Qb = g.standard_normal((H, T, 64))
    Qb[..., 0] = 1.0 + 0.1 * np.abs(Qb[..., 0])
    Kb = g.standard_normal((H, T, 64))
    cl = g.choice(T, n_cluster, replace=False)
    base = np.zeros(64)
    base[0] = 30.0
    Kb[:, cl] = base + 30.0 * spread * g.standard_normal((H, n_cluster, 64))
    return Qb, Kb


def test_selection_near_ties_are_decided_in_fp64():
    # 60 near-equal key tiles (gaps ~1e-10 relative, far inside the int8 bound, far
    # outside fp64 rounding) with k = 40: the whole decision falls in the band
    Qb, Kb = _cluster_case(T=300, n_cluster=60, spread=1e-8, seed=5)
    got = _select_gpu(Qb, Kb, 64, 40)
    assert np.array_equal(got, oracle.select_tiles(oracle.tile_scores(Qb, Kb), 40))


def test_selection_wide_band_radix_path():
    # 700 near-equal key tiles (more than the 512 a band ranks directly), k = 600
    Qb, Kb = _cluster_case(T=1000, n_cluster=700, spread=1e-8, seed=6)
    got = _select_gpu(Qb, Kb, 64, 600)
    assert np.array_equal(got, oracle.select_tiles(oracle.tile_scores(Qb, Kb), 600))


def test_selection_exact_ties_beyond_the_band_cap():
    # all scores 0 in 2,000 key tiles: ties go to the lowest indices
    g = np.random.default_rng(7)
    Qb = np.zeros((1, 2000, 64))
    Kb = g.standard_normal((1, 2000, 64))
    got = _select_gpu(Qb, Kb, 64, 5)
    assert (got == np.arange(5)).all()


def test_selection_rows_with_a_large_dynamic_range():
    # one component 1e6 times the others in every query and key row, plus rows of
    # very different magnitudes: the fixed-point copies lose the small components,
    # the band widens, the selection stays that of the fp64 scores
    g = np.random.default_rng(8)
    H, T, k = 2, 400, 37
    Qb = g.standard_normal((H, T, 64))
    Kb = g.standard_normal((H, T, 64))
    Qb[..., 3] *= 1e6
    Kb[..., 3] *= 1e6
    Kb *= np.exp2(g.integers(-60, 20, size=(H, T, 1)))
    Qb[:, ::7] *= 1e-200
    got = _select_gpu(Qb, Kb, 64, k)
    assert np.array_equal(got, oracle.select_tiles(oracle.tile_scores(Qb, Kb), k))


def test_selection_non_finite_rows_give_valid_sets():
    # a NaN in one query row and an inf in one key row of head 1: the call succeeds
    # and every row is a strictly ascending set of k indices in range; head 0 (finite)
    # matches the oracle
    g = np.random.default_rng(9)
    H, T, k = 2, 200, 11
    Qb = g.standard_normal((H, T, 64))
    Kb = g.standard_normal((H, T, 64))
    Qb[0, 17, 5] = np.nan
    Kb[1, 40, 2] = np.inf
    got = _select_gpu(Qb, Kb, 64, k)
    assert ((got >= 0) & (got < T)).all()
    assert (np.diff(got, axis=-1) > 0).all()
    ref = oracle.select_tiles(oracle.tile_scores(Qb[:1], Kb[:1]), k)
    rows = np.arange(T) != 17
    assert np.array_equal(got[0, rows], ref[0, rows])


@pytest.mark.parametrize("seed", [101, 202, 303, 404, 505, 606, 707, 808])
def test_selection_every_row_of_the_32_view_stage_many_seeds(seed):
    # 16 heads x 344 query tiles per seed, every row against the oracle
    import linear_hybrid_attention_b200 as zb
    w = workload("views32")
    Q, K, V = synth.make_qkv(w, device="cuda", seed=seed)
    lm = zb.zb_landmark_build(Q, K, V, w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, w.k)
    sync_ok()
    ref = oracle.select_tiles(oracle.tile_scores(oracle.landmark_means(host(Q), w.tile),
                                                 oracle.landmark_means(host(K), w.tile)), w.k)
    assert np.array_equal(idx.cpu().numpy().astype(np.int64), ref)
