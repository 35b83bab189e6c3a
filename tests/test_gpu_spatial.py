"""GPU parity of spatial tiles: the tile-sparse stage run on tokens reordered
into 2-D windows ("3D reconstruction drops dense attention layer by layer ...",
synopsis: exact softmax over selected spatial tiles), through HybridLayer with
the spatial option (zb_gather_rows in, the same three calls, zb_gather_rows
out), against oracle.spatial_sparse_attention."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import REL_TOL, host, check_close, sync_ok, workload

pytestmark = pytest.mark.gpu

GEOM = (synth.GRID, synth.SPECIALS, 8, 16)


def test_gather_rows_equals_indexing_and_flags_bad_rows():
    import linear_hybrid_attention_b200 as zb
    g = torch.Generator(device="cuda").manual_seed(3)
    X = torch.randn(3, 5000, 64, generator=g, device="cuda").to(torch.bfloat16)
    rows = torch.randint(0, 5000, (7777,), generator=g, device="cuda", dtype=torch.int32)
    out = zb.zb_gather_rows(X, rows)
    sync_ok()
    assert torch.equal(out, X[:, rows.long()])
    bad = rows.clone()
    bad[17] = 5000
    bad[4000] = -1
    out = zb.zb_gather_rows(X, bad)
    with pytest.raises(zb.ZbError) as e:
        zb.zb_last_device_status()
    assert e.value.status == 9
    assert bool((out[:, 17] == 0).all()) and bool((out[:, 4000] == 0).all())
    keep = torch.ones(7777, dtype=torch.bool, device="cuda")
    keep[17] = keep[4000] = False
    assert torch.equal(out[:, keep], X[:, rows.long()][:, keep])


def test_spatial_sparse_stage_two_views_matches_oracle():
    import linear_hybrid_attention_b200 as zb
    w = workload("spatial32", heads=2, n_tokens=2 * synth.TOKENS_PER_VIEW)   # T = 22, k = 5
    Q, K, V = synth.make_qkv(w, device="cuda")
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, [0], spatial=(2,) + GEOM)
    O = layer.sparse(Q, K, V)
    sync_ok()
    order = oracle.spatial_order(2)
    Q64, K64, V64 = host(Q), host(K), host(V)
    ref, ref_idx = oracle.spatial_sparse_attention(Q64, K64, V64, w.tile, order, 1 / math.sqrt(64), w.k)
    assert np.array_equal(layer.idx.cpu().numpy(), ref_idx)
    check_close(host(O), ref)
    # the spatial order really changes the result against the plain tiling
    plain = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, [0]).sparse(Q, K, V)
    sync_ok()
    assert not torch.equal(plain, O)


def test_spatial_sparse_stage_32_views_full_size_sampled():
    """The 32-view spatial workload at full size (16 heads x 43,968 tokens, k = 69):
    sampled query tiles of the reordered sequence against the oracle, selection
    bit-exact, and the convex-combination bound on every row."""
    import linear_hybrid_attention_b200 as zb
    w = workload("spatial32")
    views = w.n_tokens // synth.TOKENS_PER_VIEW
    Q, K, V = synth.make_qkv(w, device="cuda")
    layer = zb.HybridLayer(w.heads, w.n_tokens, w.tile, w.k, [0], spatial=(views,) + GEOM)
    O = layer.sparse(Q, K, V)
    sync_ok()
    vmax = V.float().amax(dim=1, keepdim=True)
    vmin = V.float().amin(dim=1, keepdim=True)
    assert bool(((O.float() <= vmax + 1e-2) & (O.float() >= vmin - 1e-2)).all())
    order = oracle.spatial_order(views)
    inv = oracle.inverse_order(order)
    s = 1 / math.sqrt(64)
    tiles = [0, 171, w.n_tiles - 1]
    n = oracle.tile_lengths(w.n_tokens, w.tile)
    for h in (2, 13):
        q, k, v = (host(t[h:h + 1])[:, order] for t in (Q, K, V))
        idx = oracle.select_tiles(oracle.tile_scores(oracle.landmark_means(q, w.tile)[:, tiles],
                                                     oracle.landmark_means(k, w.tile)), w.k)[0]
        assert np.array_equal(layer.idx[h, tiles].cpu().numpy(), idx), h
        full = np.zeros((1, w.n_tiles, w.k), dtype=np.int64)
        full[0, tiles] = idx
        ref = oracle.sparse_attention(q, k, v, w.tile, full, s, query_tiles=tiles)[0]
        got = host(O[h])
        for m, i in enumerate(tiles):
            rows_new = np.arange(i * w.tile, i * w.tile + n[i])
            want = ref[m * w.tile: m * w.tile + n[i]]
            part = got[order[rows_new]]          # original positions of the tile's tokens
            check_close(part[None], want[None], label=f"head {h} tile {i}")
    del inv
