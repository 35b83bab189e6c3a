"""The C ABI on the host: the library builds and loads, exports every function
that include/zb.h declares, and rejects bad arguments before touching the GPU.
CPU only: no call here reaches a CUDA API (validation runs first)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zb.h")


@pytest.fixture(scope="module")
def lib():
    from linear_hybrid_attention_b200 import build, _lib
    build.build()
    return _lib.load()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(zb_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_calls():
    names = _declared()
    for n in ["zb_landmark_build", "zb_tile_score_topk", "zb_tile_sparse_attn", "zb_dense_attn",
              "zb_linear_state", "zb_linear_apply", "zb_linear_attn", "zb_affine_fit", "zb_gather_tiles",
              "zb_last_device_status", "zb_status_string", "zb_abi_version", "zb_key_mean",
              "zb_linear_state_centered"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in _declared():
        assert hasattr(lib, n), n
    from linear_hybrid_attention_b200 import _lib
    assert set(_declared()) == set(_lib.PROTOTYPES)


def test_version_and_status_strings(lib):
    assert lib.zb_abi_version() == 101  # 1.1: zb_dense_attn_split, the int8 selection's workspace
    for code, name in [(0, "ZB_OK"), (2, "ZB_ERR_SHAPE"), (7, "ZB_ERR_TIMEOUT"), (9, "ZB_ERR_INDEX")]:
        assert lib.zb_status_string(code).decode().startswith(name)
    assert b"unknown" in lib.zb_status_string(1234)


def test_workspace_sizes(lib):
    n = lib.zb_linear_state_workspace_bytes(16, 1024 * 1374, 64)
    assert 0 < n < 64 * 2**20
    assert lib.zb_linear_state_workspace_bytes(16, 1000, 32) == 0
    assert lib.zb_affine_fit_workspace_bytes(16, 4096, 64) == 16 * (128 + 16 * 2 * 4096) * 8
    assert lib.zb_affine_fit_workspace_bytes(0, 4096, 64) == 0
    # the one-call linear stage holds S, z and the state partials, each 256-byte aligned
    lin = lib.zb_linear_attn_workspace_bytes(16, 1024 * 1374, 64)
    assert lin >= n + 16 * 64 * 65 * 4 and lin % 256 == 0
    assert lib.zb_linear_attn_workspace_bytes(16, 1000, 32) == 0
    # selection, per head: digit planes (192 B a row) and exponents of Qbar and Kbar,
    # the head summary and fp32 score rows padded to 128 columns, each 256-byte aligned
    assert lib.zb_tile_score_topk_workspace_bytes(_shape(H=16, N=1024 * 1374, t=128)) == 4 * _topk_head(10992)
    assert lib.zb_tile_score_topk_workspace_bytes(_shape(H=2, N=256, t=64)) == 2 * _topk_head(4)


def _topk_head(T):
    al = lambda x: -(-x // 256) * 256
    Tp = -(-T // 128) * 128
    return 2 * al(T * 192) + 2 * al(T * 4) + al(8) + al(T * Tp * 4)


def _shape(H=2, N=256, d=64, t=64):
    from linear_hybrid_attention_b200._lib import ZbShape
    return ZbShape(H, N, d, t)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def test_validation_errors_before_launch(lib):
    S = _shape()
    # unsupported head_dim / tile, bad sizes
    assert lib.zb_landmark_build(FAKE, FAKE, FAKE, _shape(d=32), FAKE, FAKE, FAKE, FAKE, None) == 4
    assert lib.zb_landmark_build(FAKE, FAKE, FAKE, _shape(t=96), FAKE, FAKE, FAKE, FAKE, None) == 4
    assert lib.zb_landmark_build(FAKE, FAKE, FAKE, _shape(N=0), FAKE, FAKE, FAKE, FAKE, None) == 2
    assert lib.zb_landmark_build(FAKE, None, FAKE, S, FAKE, FAKE, FAKE, FAKE, None) == 1
    assert lib.zb_landmark_build(FAKE, FAKE, FAKE, S, None, FAKE, FAKE, FAKE, None) == 1
    assert lib.zb_landmark_build(FAKE + 8, FAKE, FAKE, S, FAKE, FAKE, FAKE, FAKE, None) == 3
    # selection: k out of range, null output
    assert lib.zb_tile_score_topk(FAKE, FAKE, S, 5, FAKE, FAKE, 1 << 20, None) == 2
    assert lib.zb_tile_score_topk(FAKE, FAKE, S, -1, FAKE, FAKE, 1 << 20, None) == 2
    assert lib.zb_tile_score_topk(FAKE, FAKE, S, 2, None, FAKE, 1 << 20, None) == 1
    assert lib.zb_tile_score_topk(FAKE, FAKE, S, 2, FAKE, None, 1 << 20, None) == 5    # no workspace
    assert lib.zb_tile_score_topk(FAKE, FAKE, S, 2, FAKE, FAKE, _topk_head(4) - 16, None) == 5
    assert lib.zb_tile_score_topk(FAKE, FAKE, S, 0, None, None, 0, None) == 0  # nothing to do
    # sparse attention
    a = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert lib.zb_tile_sparse_attn(*a, 5, 1, 0.125, S, FAKE, None, None, 0, None) == 2          # k > T
    assert lib.zb_tile_sparse_attn(*a, 0, 0, 0.125, S, FAKE, None, None, 0, None) == 2          # no keys
    assert lib.zb_tile_sparse_attn(*a, 2, 1, -1.0, S, FAKE, None, None, 0, None) == 2           # scale
    assert lib.zb_tile_sparse_attn(FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 1, 0.125, S, FAKE, None, None, 0, None) == 1
    assert lib.zb_tile_sparse_attn(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 1, 0.125, S, FAKE, None, None, 0, None) == 1
    assert lib.zb_tile_sparse_attn(*a, 2, 1, 0.125, S, FAKE + 4, None, None, 0, None) == 3
    assert lib.zb_tile_sparse_attn(*a, 2, 1, 0.125, _shape(N=128 * 40000), FAKE, None, None, 0, None) == 4  # T > 32768
    wsa = lib.zb_tile_sparse_attn_workspace_bytes()
    assert wsa == 256
    assert lib.zb_tile_sparse_attn(*a, 2, 1, 0.125, S, FAKE, None, FAKE, wsa - 1, None) == 5   # short workspace
    assert lib.zb_tile_sparse_attn(*a, 2, 1, 0.125, S, FAKE, None, FAKE + 8, wsa, None) == 3   # misaligned
    # dense
    assert lib.zb_dense_attn(FAKE, 0, FAKE, FAKE, 10, 2, 64, 0.125, FAKE, 0, None, None) == 2
    assert lib.zb_dense_attn(FAKE, 10, FAKE, FAKE, 10, 2, 128, 0.125, FAKE, 1, None, None) == 4
    # linear
    need = lib.zb_linear_state_workspace_bytes(2, 256, 64)
    assert lib.zb_linear_state(FAKE, FAKE, 2, 256, 64, FAKE, FAKE, FAKE, need - 1, None) == 5
    assert lib.zb_linear_state(FAKE, FAKE, 2, 256, 64, FAKE, FAKE, None, need, None) == 5
    assert lib.zb_linear_state(FAKE, None, 2, 256, 64, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.zb_linear_apply(FAKE, 2, 256, 64, FAKE, None, None, None, FAKE, 0, None) == 1
    assert lib.zb_linear_apply(FAKE, 2, 256, 64, FAKE, FAKE, FAKE + 2, None, FAKE, 1, None) == 3
    # affine fit: too few rows, workspace
    lin = lib.zb_linear_attn_workspace_bytes(2, 256, 64)
    assert lib.zb_linear_attn(FAKE, FAKE, FAKE, 2, 0, 64, None, None, FAKE, FAKE, lin, None) == 2
    assert lib.zb_linear_attn(FAKE, FAKE, FAKE, 2, 256, 32, None, None, FAKE, FAKE, lin, None) == 4
    assert lib.zb_linear_attn(None, FAKE, FAKE, 2, 256, 64, None, None, FAKE, FAKE, lin, None) == 1
    assert lib.zb_linear_attn(FAKE, FAKE, FAKE, 2, 256, 64, FAKE + 4, None, FAKE, FAKE, lin, None) == 3
    assert lib.zb_linear_attn(FAKE, FAKE, FAKE, 2, 256, 64, None, None, FAKE, FAKE, lin - 1, None) == 5
    assert lib.zb_linear_attn(FAKE, FAKE, FAKE, 2, 256, 64, None, None, FAKE, None, lin, None) == 5
    assert lib.zb_affine_fit(FAKE, FAKE, 2, 64, 64, FAKE, FAKE, FAKE, 1 << 30, None) == 2
    wsn = lib.zb_affine_fit_workspace_bytes(2, 300, 64)
    assert lib.zb_affine_fit(FAKE, FAKE, 2, 300, 64, FAKE, FAKE, FAKE, wsn - 8, None) == 5
    # linear-centered: key mean and centred state
    kmw = lib.zb_key_mean_workspace_bytes(2, 256, 64)
    assert kmw > 0 and kmw % (64 * 8) == 0
    assert lib.zb_key_mean_workspace_bytes(2, 256, 32) == 0
    assert lib.zb_key_mean(FAKE, 2, 0, 64, FAKE, FAKE, kmw, None) == 2
    assert lib.zb_key_mean(FAKE, 2, 256, 32, FAKE, FAKE, kmw, None) == 4
    assert lib.zb_key_mean(FAKE, 70000, 256, 64, FAKE, FAKE, 1 << 40, None) == 4
    assert lib.zb_key_mean(None, 2, 256, 64, FAKE, FAKE, kmw, None) == 1
    assert lib.zb_key_mean(FAKE, 2, 256, 64, None, FAKE, kmw, None) == 1
    assert lib.zb_key_mean(FAKE, 2, 256, 64, FAKE + 4, FAKE, kmw, None) == 3
    assert lib.zb_key_mean(FAKE, 2, 256, 64, FAKE, FAKE, kmw - 8, None) == 5
    assert lib.zb_key_mean(FAKE, 2, 256, 64, FAKE, None, kmw, None) == 5
    assert lib.zb_linear_state_centered(FAKE, FAKE, None, 2, 256, 64, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.zb_linear_state_centered(FAKE, FAKE, FAKE + 4, 2, 256, 64, FAKE, FAKE, FAKE, need, None) == 3
    assert lib.zb_linear_state_centered(FAKE, FAKE, FAKE, 2, 256, 64, FAKE, FAKE, FAKE, need - 1, None) == 5
    assert lib.zb_linear_state_centered(FAKE, FAKE, FAKE, 2, 256, 16, FAKE, FAKE, FAKE, need, None) == 4
    assert lib.zb_linear_state_centered(FAKE, FAKE, FAKE, 0, 256, 64, FAKE, FAKE, FAKE, need, None) == 2
    # block-mass diagnostic
    assert lib.zb_block_mass(FAKE, FAKE, FAKE, _shape(t=96), 0.125, FAKE, None) == 4
    assert lib.zb_block_mass(FAKE, FAKE, None, S, 0.125, FAKE, None) == 1
    assert lib.zb_block_mass(FAKE, FAKE, FAKE, S, 0.0, FAKE, None) == 2
    assert lib.zb_block_mass(FAKE + 2, FAKE, FAKE, S, 0.125, FAKE, None) == 3
    assert lib.zb_block_mass(FAKE, FAKE, FAKE, _shape(N=64 * 50000), 0.125, FAKE, None) == 4  # Tb > 49152
    assert lib.zb_block_mass_top_fraction(FAKE, 2, 4, 5, FAKE, None) == 2                     # m > n_blocks
    assert lib.zb_block_mass_top_fraction(FAKE, 2, 4, -1, FAKE, None) == 2
    assert lib.zb_block_mass_top_fraction(None, 2, 4, 1, FAKE, None) == 1
    assert lib.zb_block_mass_top_fraction(FAKE, 2, 60000, 1, FAKE, None) == 4
    assert lib.zb_block_mass_selected_fraction(FAKE, 2, 4, FAKE, 0, FAKE, None) == 2
    assert lib.zb_block_mass_selected_fraction(FAKE, 2, 4, None, 2, FAKE, None) == 1
    assert lib.zb_block_mass_selected_fraction(FAKE + 4, 2, 4, FAKE, 2, FAKE, None) == 3
    # gather
    assert lib.zb_gather_tiles(FAKE, S, FAKE, 0, FAKE, None) == 2
    assert lib.zb_gather_tiles(FAKE, S, None, 2, FAKE, None) == 1


def test_binding_refuses_cpu_tensors():
    import torch
    import linear_hybrid_attention_b200 as zb
    x = torch.zeros(1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        zb.zb_landmark_build(x, x, x, 64)
    with pytest.raises(ValueError, match="CUDA"):
        zb.zb_linear_state(x, x)


def test_topk_launch_count_follows_the_launcher():
    # zb_tile_score_topk: nothing for k = 0, one fill kernel for k = T, else digit
    # planes, head summary, score GEMM and select per pass over the heads the workspace holds
    from linear_hybrid_attention_b200 import topk_launches
    N, t = 1024 * 1374, 128
    T, one = 10992, _topk_head(10992)
    assert topk_launches(16, N, t, 660, 4 * one) == 16
    assert topk_launches(16, N, t, 660, 16 * one) == 4
    assert topk_launches(16, N, t, 660, 5 * one - 1) == 16   # 4 heads per pass
    assert topk_launches(3, N, t, 660, 2 * one) == 8         # passes of 2 and 1 heads
    assert topk_launches(16, N, t, 0, 0) == 0
    assert topk_launches(16, N, t, T, 0) == 1


def test_dense_split_validation_and_workspace(lib):
    # workspace: query replicas (bf16), partial outputs (fp32) and their lse, 256-byte aligned
    al = lambda x: -(-x // 256) * 256
    rows = 4096 * 16 * 4
    assert lib.zb_dense_attn_split_workspace_bytes(4096, 16, 64, 4) == al(rows * 128) + al(rows * 256) + al(rows * 4)
    assert lib.zb_dense_attn_split_workspace_bytes(4096, 16, 64, 1) == 0
    assert lib.zb_dense_attn_split_workspace_bytes(4096, 16, 64, 17) == 0
    assert lib.zb_dense_attn_split_workspace_bytes(4096, 16, 32, 4) == 0
    call = lambda nq, nk, H, d, s, O, ws, wsb: lib.zb_dense_attn_split(FAKE, nq, FAKE, FAKE, nk, H, d, 0.125, s, O,
                                                                       1, None, ws, wsb, None)
    assert call(100, 1001, 2, 64, 4, FAKE, FAKE, 1 << 30) == 2     # keys not a multiple of the splits
    assert call(100, 1000, 2, 64, 0, FAKE, FAKE, 1 << 30) == 2     # no split
    assert call(100, 1000, 2, 64, 17, FAKE, FAKE, 1 << 30) == 2    # too many
    assert call(100, 1000, 2, 32, 4, FAKE, FAKE, 1 << 30) == 4     # head_dim
    assert call(100, 1000, 2, 64, 4, None, FAKE, 1 << 30) == 1     # no output
    assert call(100, 1000, 2, 64, 4, FAKE + 8, FAKE, 1 << 30) == 3 # misaligned output
    need = lib.zb_dense_attn_split_workspace_bytes(100, 2, 64, 4)
    assert call(100, 1000, 2, 64, 4, FAKE, FAKE, need - 1) == 5    # workspace too small
    assert call(100, 1000, 2, 64, 4, FAKE, None, need) == 5        # no workspace


def test_dense_splits_fill_the_pipelines():
    from linear_hybrid_attention_b200 import dense_splits
    # calibration at 1,024 views: 16 heads x 32 query tiles on 148 SMs x 2 pipelines;
    # 512 items need 2 sweeps, 4 splits 7 quarter sweeps (1.75)
    assert dense_splits(16, 4096, 1_406_976, 148) == 4
    # enough items already: no split
    assert dense_splits(16, 128 * 300, 1_406_976, 148) == 1
    # only counts dividing the key count
    assert dense_splits(16, 4096, 1_406_977, 148) == 1
    # one head, one query tile: as many splits as allowed that divide the keys
    assert dense_splits(1, 128, 8 * 1000, 148) == 8
