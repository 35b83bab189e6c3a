"""GPU parity at the workloads' full sizes, in the launch configuration the
bench times (HybridLayer on all 16 heads), checked on sampled outputs that the
fp64 oracle computes one by one: for sampled heads and query tiles, the
selected key-tile set must be bit-exact and the attention output within the
relative-error bar; every output row must be a convex combination of values.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import REL_TOL, check_close, host, sync_ok, workload

pytestmark = pytest.mark.gpu


def _check_sparse_sampled(w, layer_seed, heads, tiles):
    import linear_hybrid_attention_b200 as zb
    Q, K, V = synth.make_qkv(w, device="cuda", seed=layer_seed)
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, calib)
    O = layer.sparse(Q, K, V)
    sync_ok()
    # convex-combination bound on every row of the full output
    vmax = V.float().amax(dim=1, keepdim=True)
    vmin = V.float().amin(dim=1, keepdim=True)
    assert bool(((O.float() <= vmax + 1e-2) & (O.float() >= vmin - 1e-2)).all())
    s = 1 / math.sqrt(w.head_dim)
    n = oracle.tile_lengths(w.n_tokens, w.tile)
    for h in heads:
        q64, k64, v64 = host(Q[h:h + 1]), host(K[h:h + 1]), host(V[h:h + 1])
        Qb = oracle.landmark_means(q64, w.tile)
        Kb = oracle.landmark_means(k64, w.tile)
        ref_idx = oracle.select_tiles(oracle.tile_scores(Qb[:, tiles], Kb), w.k)[0]
        got_idx = layer.idx[h, tiles].cpu().numpy()
        assert np.array_equal(got_idx, ref_idx), (h, tiles)
        idx_full = np.zeros((1, w.n_tiles, w.k), dtype=np.int64)
        idx_full[0, tiles] = ref_idx
        ref = oracle.sparse_attention(q64, k64, v64, w.tile, idx_full, s, query_tiles=tiles)[0]
        for slot, i in enumerate(tiles):
            rows = slice(i * w.tile, i * w.tile + n[i])
            got = host(O[h, rows])
            want = ref[slot * w.tile: slot * w.tile + n[i]]
            check_close(got[None], want[None], label=f"head {h} tile {i}")


def _sample_tiles(T, n, seed):
    """The first and the (ragged) last query tile plus n - 2 seeded others, ascending."""
    g = np.random.default_rng(seed)
    mid = g.choice(np.arange(1, T - 1), n - 2, replace=False)
    return sorted({0, T - 1, *mid.tolist()})


def test_sparse_stage_1024_views_full_size_sampled():
    """1,024 views: 16 heads x 1,406,976 tokens, T = 10,992, k = 660; 16 query tiles
    of each of 3 heads."""
    w = workload("views1024")
    _check_sparse_sampled(w, synth.default_seed(w), heads=[0, 9, 15], tiles=_sample_tiles(w.n_tiles, 16, 11))


def test_sparse_stage_512_views_layer0_full_size_sampled():
    """One tile-sparse layer of the 512-view stack: 16 x 703,488 tokens, k = 1,100;
    12 query tiles of each of 2 heads."""
    w = workload("stack512")
    _check_sparse_sampled(w, synth.default_seed(w, layer=0), heads=[3, 12], tiles=_sample_tiles(w.n_tiles, 12, 12))


def test_linear_stage_1024_views_full_size_sampled():
    """Fitted linear stage at 1,024 views: calibration (dense attention on 4,096
    rows, fp32 linear output, fit) and the output on all rows on the GPU; the
    oracle fits one head in full and checks sampled query tiles."""
    import linear_hybrid_attention_b200 as zb
    w = workload("views1024")
    Q, K, V = synth.make_qkv(w, device="cuda")
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, calib)
    layer.calibrate(Q, K, V)
    o_l = layer.linear(Q, K, V)
    sync_ok()
    h = 5
    q64, k64, v64 = host(Q[h:h + 1]), host(K[h:h + 1]), host(V[h:h + 1])
    rows = oracle.calibration_rows(w.n_tokens, w.tile, calib)
    X = oracle.linear_attention(q64[:, rows], k64, v64)
    Y = np.concatenate([oracle.dense_attention(q64[:, rows[c:c + 128]], k64, v64, 1 / 8)
                        for c in range(0, len(rows), 128)], axis=1)
    A, b = oracle.affine_fit(X, Y)
    tiles = [0, 7777, w.n_tiles - 1]
    srows = oracle.calibration_rows(w.n_tokens, w.tile, tiles)
    want = oracle.linear_attention(q64[:, srows], k64, v64, A, b)[0]
    got = host(o_l[h, srows])
    check_close(got[None], want[None], label=f"head {h}")


def test_linear_stage_512_views_layer1_full_size_sampled():
    """A linear layer of the 512-view stack (layer 1, its own seed): 16 x 703,488 tokens,
    calibration and output on the GPU, one head fitted in full by the oracle."""
    import linear_hybrid_attention_b200 as zb
    w = workload("stack512")
    assert 1 in w.linear_layers
    Q, K, V = synth.make_qkv(w, device="cuda", seed=synth.default_seed(w, layer=1))
    calib = synth.calibration_tiles(w.n_tiles, w.calib_tiles)
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, calib)
    layer.calibrate(Q, K, V)
    o_l = layer.linear(Q, K, V)
    sync_ok()
    h = 10
    q64, k64, v64 = host(Q[h:h + 1]), host(K[h:h + 1]), host(V[h:h + 1])
    rows = oracle.calibration_rows(w.n_tokens, w.tile, calib)
    X = oracle.linear_attention(q64[:, rows], k64, v64)
    Y = np.concatenate([oracle.dense_attention(q64[:, rows[c:c + 128]], k64, v64, 1 / 8)
                        for c in range(0, len(rows), 128)], axis=1)
    A, b = oracle.affine_fit(X, Y)
    tiles = [0, 2748, w.n_tiles - 1]
    srows = oracle.calibration_rows(w.n_tokens, w.tile, tiles)
    want = oracle.linear_attention(q64[:, srows], k64, v64, A, b)[0]
    got = host(o_l[h, srows])
    check_close(got[None], want[None], label=f"head {h}")


def test_selection_1024_views_every_row_of_one_head():
    """Every one of the 10,992 query tiles of head 5 at 1,024 views, in the bench's
    launch configuration: the selected sets equal the oracle's."""
    import linear_hybrid_attention_b200 as zb
    w = workload("views1024")
    Q, K, V = synth.make_qkv(w, device="cuda")
    h = 5
    lm = zb.zb_landmark_build(Q[h:h + 1].contiguous(), K[h:h + 1].contiguous(), V[h:h + 1].contiguous(), w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, w.k)
    sync_ok()
    got = idx.cpu().numpy()[0]
    del lm, idx
    Qb = oracle.landmark_means(host(Q[h:h + 1]), w.tile)
    Kb = oracle.landmark_means(host(K[h:h + 1]), w.tile)
    del Q, K, V
    ref = oracle.select_tiles(oracle.tile_scores(Qb, Kb), w.k)[0]
    bad = np.flatnonzero((got != ref).any(-1))
    assert bad.size == 0, (bad.size, bad[:5])


def test_selection_1024_views_keep20_every_row_of_one_head():
    """The pages' keep-20% budget (k = 2,199 of 10,992) on head 11 at 1,024 views: every
    query tile's selected set equals the oracle's."""
    import linear_hybrid_attention_b200 as zb
    w = workload("views1024")
    k20 = -(-w.n_tiles // 5)
    Q, K, V = synth.make_qkv(w, device="cuda")
    h = 11
    lm = zb.zb_landmark_build(Q[h:h + 1].contiguous(), K[h:h + 1].contiguous(), V[h:h + 1].contiguous(), w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, k20)
    sync_ok()
    got = idx.cpu().numpy()[0]
    del lm, idx
    Qb = oracle.landmark_means(host(Q[h:h + 1]), w.tile)
    Kb = oracle.landmark_means(host(K[h:h + 1]), w.tile)
    del Q, K, V
    ref = oracle.select_tiles(oracle.tile_scores(Qb, Kb), k20)[0]
    bad = np.flatnonzero((got != ref).any(-1))
    assert bad.size == 0, (bad.size, bad[:5])
