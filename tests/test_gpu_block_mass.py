"""GPU parity: the block-mass diagnostic (dense softmax mass per 64 x 64 or
128 x 128 token block, and the share of it that a selection keeps)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.gpu_helpers import host, check_close, sync_ok, workload

pytestmark = pytest.mark.gpu

# M is recomputed from fp32 S and the fp32 row log-sum-exp, each p within a few
# ulp of fp32: far below the float bar of 2e-2, so a tight bound is used
MASS_TOL = 1e-3


def _zb():
    import linear_hybrid_attention_b200 as zb
    return zb


def _inputs(heads, n):
    zb = _zb()
    # the 32-view recipe plants 3 to 5 key tiles per query tile; sequences of a
    # few tiles use the tiny recipe (64-token tiles, one planted tile)
    w = workload("views32" if n >= 1000 else "tiny", heads=heads, n_tokens=n)
    Q, K, V = synth.make_qkv(w, device="cuda")
    _, lse = zb.zb_dense_attn(Q, K, V, 1 / 8, want_lse=True)
    return w, Q, K, lse


@pytest.mark.parametrize("heads,n,block", [(2, 256, 64), (1, 130, 64), (3, 1000, 64), (2, 1000, 128),
                                           (2, 5000, 64), (2, 5000, 128)])
def test_block_mass_matches_oracle(heads, n, block):
    zb = _zb()
    w, Q, K, lse = _inputs(heads, n)
    M = zb.zb_block_mass(Q, K, lse, block, 1 / 8)
    sync_ok()
    ref = oracle.block_mass(host(Q), host(K), 1 / 8, block)
    got = M.double().cpu().numpy()
    check_close(got, ref, tol=MASS_TOL)
    # one unit of mass per query row
    lengths = oracle.tile_lengths(n, block).astype(np.float64)
    np.testing.assert_allclose(got.sum(axis=-1), np.broadcast_to(lengths, got.shape[:2]), rtol=MASS_TOL)


@pytest.mark.parametrize("heads,n,block,frac", [(2, 1000, 64, 0.2), (3, 5000, 64, 0.2), (2, 5000, 128, 0.5)])
def test_top_fraction_matches_oracle(heads, n, block, frac):
    zb = _zb()
    w, Q, K, lse = _inputs(heads, n)
    M = zb.zb_block_mass(Q, K, lse, block, 1 / 8)
    Tb = M.shape[-1]
    m = math.ceil(frac * Tb)
    f = zb.zb_block_mass_top_fraction(M, m)
    sync_ok()
    ref = oracle.top_mass_fraction(oracle.block_mass(host(Q), host(K), 1 / 8, block), m)
    assert np.abs(f.double().cpu().numpy() - ref).max() <= 1e-4


def test_top_fraction_with_ties_zeros_and_edges():
    # small integers: many exact ties; the selection count must be exact
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(5)
    M = torch.randint(0, 4, (3, 70, 70), generator=g, device="cuda").float()
    M[:, :, 0] += 1.0
    M64 = M.double().cpu().numpy()
    for m in (0, 1, 13, 69, 70):
        f = zb.zb_block_mass_top_fraction(M, m)
        sync_ok()
        np.testing.assert_allclose(f.double().cpu().numpy(), oracle.top_mass_fraction(M64, m), rtol=0, atol=1e-6)


def test_top_fraction_long_rows():
    # 12,000 key blocks per row (a 1,024-view head has 21,984): rows held in shared memory
    zb = _zb()
    g = torch.Generator(device="cuda").manual_seed(6)
    T = 12000
    M = torch.rand(1, T, T, generator=g, device="cuda") ** 4
    m = math.ceil(0.2 * T)
    f = zb.zb_block_mass_top_fraction(M, m)
    sync_ok()
    rows = [0, 1, T // 2, T - 1]
    ref = oracle.top_mass_fraction(M[:, rows].double().cpu().numpy(), m)
    np.testing.assert_allclose(f[:, rows].double().cpu().numpy(), ref, rtol=0, atol=1e-6)


@pytest.mark.parametrize("heads,n", [(2, 1000), (3, 5000)])
def test_selected_fraction_matches_oracle(heads, n):
    """The mass that the method's mean-pooled selection keeps, at its own tile size."""
    zb = _zb()
    w, Q, K, lse = _inputs(heads, n)
    lm = zb.zb_landmark_build(Q, K, K, w.tile)
    idx = zb.zb_tile_score_topk(lm.Qbar, lm.Kbar, n, w.tile, w.k)
    M = zb.zb_block_mass(Q, K, lse, w.tile, 1 / 8)
    f = zb.zb_block_mass_selected_fraction(M, idx)
    sync_ok()
    ref = oracle.selected_mass_fraction(oracle.block_mass(host(Q), host(K), 1 / 8, w.tile),
                                        idx.long().cpu().numpy())
    assert np.abs(f.double().cpu().numpy() - ref).max() <= 1e-4
