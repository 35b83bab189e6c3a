"""GPU parity: tile-sparse attention with landmarks, and dense attention."""
import math

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


def _sparse_gpu(w, Q, K, V, k=None, use_landmarks=True, want_lse=False):
    zb = _zb()
    k = w.k if k is None else k
    lm = zb.zb_landmark_build(Q, K, V, w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, k)
    out = zb.zb_tile_sparse_attn(Q, K, V, lm.Kbar_bf16, lm.Vbar_bf16, idx, k, w.tile,
                                 use_landmarks=use_landmarks, want_lse=want_lse)
    sync_ok()
    return out, idx


def _oracle_idx(w, Q64, K64, k):
    return oracle.select_tiles(oracle.tile_scores(oracle.landmark_means(Q64, w.tile),
                                                  oracle.landmark_means(K64, w.tile)), k)


FULL_CASES = [
    ("tiny", {}, None),
    ("views32", {"heads": 2, "n_tokens": 5000}, 8),       # T = 40, ragged 8-row last tile
    ("views32", {"heads": 3, "n_tokens": 2000, "tile": 64}, 5),  # t = 64 with landmarks
]


@pytest.mark.parametrize("name,over,k", FULL_CASES)
def test_sparse_attention_matches_oracle(name, over, k):
    w = workload(name, **over)
    k = w.k if k is None else k
    Q, K, V = synth.make_qkv(w, device="cuda")
    O, idx = _sparse_gpu(w, Q, K, V, k)
    Q64, K64, V64 = host(Q), host(K), host(V)
    ref_idx = _oracle_idx(w, Q64, K64, k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    ref = oracle.sparse_attention(Q64, K64, V64, w.tile, ref_idx, 1 / math.sqrt(64))
    check_close(host(O), ref)


def test_sparse_attention_rescales_o_when_the_row_max_grows():
    """Keys scaled up tile by tile (tile j by 1 + 0.75 j) and queries by 4: each
    row's running max grows by more than the lazy-rescale threshold (8 in log2
    units) partway through its item, at different steps for different rows of
    one warp, so the O rescale runs inside items and with rows that disagree."""
    w = workload("views32", heads=2, n_tokens=3000)          # T = 24, ragged 56-row last tile
    Q, K, V = synth.make_qkv(w, device="cuda")
    grow = 1.0 + 0.75 * (torch.arange(w.n_tokens, device="cuda") // w.tile).float()
    Q = (Q.float() * 4).to(torch.bfloat16)
    K = (K.float() * 4 * grow[None, :, None]).to(torch.bfloat16)
    k = 12
    O, idx = _sparse_gpu(w, Q, K, V, k)
    Q64, K64, V64 = host(Q), host(K), host(V)
    ref_idx = _oracle_idx(w, Q64, K64, k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    # the planted rescale really happens: row maxima of the first and last
    # selected tiles differ by more than 8 in log2 units for many rows
    s = 1 / math.sqrt(64)
    lg = np.log2(np.e) * s
    first = np.array([[(Q64[h, i * 128:(i + 1) * 128] @ K64[h, j0 * 128:(j0 + 1) * 128].T).max(1)
                       for i, j0 in enumerate(ref_idx[h, :, 0][:23])] for h in range(2)])
    last = np.array([[(Q64[h, i * 128:(i + 1) * 128] @ K64[h, j1 * 128:min(j1 * 128 + 128, w.n_tokens)].T).max(1)
                      for i, j1 in enumerate(ref_idx[h, :, -1][:23])] for h in range(2)])
    assert ((last - first) * lg > 8).mean() > 0.2
    ref = oracle.sparse_attention(Q64, K64, V64, w.tile, ref_idx, s)
    check_close(host(O), ref)


def test_sparse_lse_matches_oracle_logsumexp():
    w = workload("tiny")
    Q, K, V = synth.make_qkv(w, device="cuda")
    (O, lse), idx = _sparse_gpu(w, Q, K, V, want_lse=True)
    Q64, K64, V64 = host(Q), host(K), host(V)
    s = 1 / math.sqrt(64)
    ref_idx = _oracle_idx(w, Q64, K64, w.k)
    n = oracle.tile_lengths(w.n_tokens, w.tile)
    Kb = oracle.landmark_means(K64, w.tile)
    got = lse.cpu().numpy()
    for h in range(w.heads):
        for i in range(w.n_tiles):
            sel = ref_idx[h, i]
            cols = np.concatenate([np.arange(j * w.tile, j * w.tile + n[j]) for j in sel])
            lm = np.setdiff1d(np.arange(w.n_tiles), sel)
            q = Q64[h, i * w.tile:(i + 1) * w.tile]
            logits = np.concatenate([s * q @ K64[h, cols].T, s * q @ Kb[h, lm].T + np.log(n[lm])], axis=1)
            m = logits.max(1, keepdims=True)
            ref = (m + np.log(np.exp(logits - m).sum(1, keepdims=True)))[:, 0]
            np.testing.assert_allclose(got[h, i * w.tile:(i + 1) * w.tile], ref, atol=2e-2)


def test_keep_all_tiles_equals_dense():
    w = workload("views32", heads=2, n_tokens=3000)
    Q, K, V = synth.make_qkv(w, device="cuda")
    O, idx = _sparse_gpu(w, Q, K, V, k=w.n_tiles)
    ref = oracle.dense_attention(host(Q), host(K), host(V), 1 / math.sqrt(64))
    check_close(host(O), ref)


def test_tile_constant_keys_make_landmarks_exact():
    # every key row of a tile equal: the landmark path must reproduce dense attention
    w = workload("views32", heads=2, n_tokens=3000)
    Q, _, V = synth.make_qkv(w, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(5)
    Kt = (torch.randn(2, w.n_tiles, 64, generator=g, device="cuda") * 0.5).to(torch.bfloat16)
    K = Kt.repeat_interleave(w.tile, dim=1)[:, : w.n_tokens].contiguous()
    for k in (0, 3, 11):
        O, _ = _sparse_gpu(w, Q, K, V, k=k)
        ref = oracle.dense_attention(host(Q), host(K), host(V), 1 / math.sqrt(64))
        check_close(host(O), ref, label=str(k))


@pytest.mark.parametrize("k,use_lm", [(0, True), (4, False), (1, True)])
def test_sparse_variants(k, use_lm):
    w = workload("views32", heads=2, n_tokens=2500)
    Q, K, V = synth.make_qkv(w, device="cuda", seed=9)
    O, idx = _sparse_gpu(w, Q, K, V, k=k, use_landmarks=use_lm)
    Q64, K64, V64 = host(Q), host(K), host(V)
    ref_idx = _oracle_idx(w, Q64, K64, k)
    ref = oracle.sparse_attention(Q64, K64, V64, w.tile, ref_idx, 1 / math.sqrt(64), use_landmarks=use_lm)
    check_close(host(O), ref)


def test_sparse_full_views32_sampled():
    """Full 32-view stage (T = 344, k = 69): selection compared in full, outputs
    on sampled query tiles (first, middle, last = ragged) of every head."""
    w = workload("views32")
    Q, K, V = synth.make_qkv(w, device="cuda")
    O, idx = _sparse_gpu(w, Q, K, V)
    Q64, K64, V64 = host(Q), host(K), host(V)
    ref_idx = _oracle_idx(w, Q64, K64, w.k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    tiles = [0, w.n_tiles // 2, w.n_tiles - 1]
    ref = oracle.sparse_attention(Q64, K64, V64, w.tile, ref_idx, 1 / math.sqrt(64), query_tiles=tiles)
    got = np.concatenate([host(O)[:, j * w.tile: j * w.tile + w.tile] for j in tiles[:-1]]
                         + [np.pad(host(O)[:, (w.n_tiles - 1) * w.tile:], ((0, 0), (0, 64), (0, 0)))], axis=1)
    check_close(got, ref)
    # every output row is a convex combination of value rows
    Vh = V.float()
    assert (O.float() <= Vh.amax(1, keepdim=True) + 1e-2).all()
    assert (O.float() >= Vh.amin(1, keepdim=True) - 1e-2).all()


def test_wave_sync_is_bit_identical():
    """The 32-view stage (about 18 rounds per slot on every SM) with and without
    the wave synchronisation: only the schedule differs, not one bit of O."""
    zb = _zb()
    w = workload("views32")
    Q, K, V = synth.make_qkv(w, device="cuda")
    lm = zb.zb_landmark_build(Q, K, V, w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, w.n_tokens, w.tile, w.k)
    a, la = zb.zb_tile_sparse_attn(Q, K, V, lm.Kbar_bf16, lm.Vbar_bf16, idx, w.k, w.tile, want_lse=True,
                                   wave_sync=True)
    b, lb = zb.zb_tile_sparse_attn(Q, K, V, lm.Kbar_bf16, lm.Vbar_bf16, idx, w.k, w.tile, want_lse=True,
                                   wave_sync=False)
    sync_ok()
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("nq,nk", [(300, 1000), (128, 128), (1, 77), (4096, 6000)])
def test_dense_matches_oracle(nq, nk):
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(nq + nk)
    Q = torch.randn(2, nq, 64, generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn(2, nk, 64, generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn(2, nk, 64, generator=g, device="cuda").to(torch.bfloat16)
    O = zb.zb_dense_attn(Q, K, V)
    sync_ok()
    ref = oracle.dense_attention(host(Q), host(K), host(V), 1 / 8)
    check_close(host(O), ref)


@pytest.mark.parametrize("nq,nk,splits", [(300, 1000, 4), (4096, 6000, 3), (1, 77, 7), (257, 4096, 2), (128, 640, 5)])
def test_dense_split_matches_oracle(nq, nk, splits):
    """Keys split in equal parts and merged by log-sum-exp: the dense softmax over
    all keys, in fp32 and bf16 outputs, with the merged log-sum-exp."""
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(3 * nq + nk + splits)
    H = 3
    Q = torch.randn(H, nq, 64, generator=g, device="cuda").to(torch.bfloat16)
    K = torch.randn(H, nk, 64, generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn(H, nk, 64, generator=g, device="cuda").to(torch.bfloat16)
    O32, lse = zb.zb_dense_attn_split(Q, K, V, splits, want_lse=True, out_fp32=True)
    O16 = zb.zb_dense_attn_split(Q, K, V, splits)
    sync_ok()
    q, k, v = host(Q), host(K), host(V)
    ref = oracle.dense_attention(q, k, v, 1 / 8)
    check_close(O32.cpu().numpy(), ref, label=f"fp32 splits {splits}")
    check_close(host(O16), ref, label=f"bf16 splits {splits}")
    logits = np.einsum("hqd,hkd->hqk", q, k) / 8
    m = logits.max(-1)
    ref_lse = m + np.log(np.exp(logits - m[..., None]).sum(-1))
    assert np.abs(lse.cpu().numpy() - ref_lse).max() <= 1e-2 * max(1.0, np.abs(ref_lse).max())


def test_dense_split_of_one_is_the_dense_call():
    zb = _zb()
    w = workload("tiny")
    Q, K, V = synth.make_qkv(w, device="cuda")
    a = zb.zb_dense_attn(Q, K, V, out_fp32=True)
    b = zb.zb_dense_attn_split(Q, K, V, 1, out_fp32=True)
    sync_ok()
    assert torch.equal(a, b)
