"""Zebra3D hybrid global-attention layer for NVIDIA B200 (sm_100a).

Thin Python binding of the C ABI in ``include/zb.h`` (``libzb.so``).  The
functions below carry the C names; they only marshal arguments: check tensors,
allocate outputs with PyTorch (device memory and the current stream are the
only things PyTorch provides), call the library, and raise ``ZbError`` on a
non-zero status.  Every step of the layer runs in the library's CUDA kernels;
there is no CPU fallback -- without the library or a CUDA device the calls
raise.

The layer ("Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D
Reconstruction", Abstract and Figure 1 (a) caption):
  * tile-sparse stage: landmarks -> tile selection -> tile-sparse softmax
    attention with mean-key/value landmarks for the omitted tiles;
  * linear stage: elu+1 linear attention -> closed-form affine map fitted to
    the dense output on calibration rows.
"""
from __future__ import annotations

import math
from typing import NamedTuple, Optional, Sequence

import torch

from . import _lib

__all__ = [
    "ZbError", "Landmarks", "zb_abi_version", "zb_landmark_build", "zb_tile_score_topk",
    "zb_tile_sparse_attn", "zb_dense_attn", "zb_dense_attn_split", "dense_splits", "zb_linear_state", "zb_linear_apply", "zb_linear_attn",
    "zb_affine_fit", "zb_gather_tiles", "zb_last_device_status", "HybridLayer",
    "LAUNCHES_PER_CALL", "zb_key_mean", "zb_linear_state_centered", "zb_block_mass",
    "zb_block_mass_top_fraction", "zb_block_mass_selected_fraction", "zb_spatial_order", "zb_gather_rows",
]

HEAD_DIM = 64

# kernels each entry point launches (for counting launches in a timed region);
# zb_tile_score_topk launches 4 per pass over the heads its workspace holds
# (topk_launches gives the count of one call)
LAUNCHES_PER_CALL = {
    "zb_landmark_build": 1, "zb_tile_score_topk": 4, "zb_tile_sparse_attn": 1, "zb_dense_attn": 1,
    "zb_dense_attn_split": 2,
    "zb_linear_state": 2, "zb_linear_apply": 1, "zb_linear_attn": 3, "zb_affine_fit": 3, "zb_gather_tiles": 1,
    "zb_key_mean": 2, "zb_linear_state_centered": 2, "zb_block_mass": 1, "zb_block_mass_top_fraction": 1,
    "zb_block_mass_selected_fraction": 1, "zb_gather_rows": 1, "zb_spatial_order": 0,
}


def topk_launches(heads: int, n_tokens: int, tile: int, k: int, ws_bytes: int) -> int:
    """Kernels one zb_tile_score_topk call launches: none for k = 0, one fill kernel for
    k = T, else four per pass (digit planes, head summary, int8 score GEMM, select)
    over as many heads as the workspace holds (one head's share is the default
    workspace of a one-head shape)."""
    T = -(-n_tokens // tile)
    if k == 0:
        return 0
    if k == T:
        return 1
    per_pass = min(heads, ws_bytes // topk_workspace_bytes(1, n_tokens, tile))
    return LAUNCHES_PER_CALL["zb_tile_score_topk"] * (-(-heads // per_pass))


class ZbError(RuntimeError):
    """A libzb call returned a non-zero zb_status."""

    def __init__(self, what: str, status: int):
        self.status = status
        name = _lib.STATUS.get(status, str(status))
        super().__init__(f"{what} failed: {name}")


class Landmarks(NamedTuple):
    Qbar: torch.Tensor       # fp64 [H, T, d]
    Kbar: torch.Tensor       # fp64 [H, T, d]
    Kbar_bf16: torch.Tensor  # bf16 [H, T, d]
    Vbar_bf16: torch.Tensor  # bf16 [H, T, d]


def _lib_handle():
    return _lib.load()


def _check(status: int, what: str) -> None:
    if status != 0:
        raise ZbError(what, status)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, ndim: int) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libzb has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out(shape, dtype, device, out: Optional[torch.Tensor], name: str) -> torch.Tensor:
    if out is None:
        return torch.empty(shape, dtype=dtype, device=device)
    _need(out, dtype, name, len(shape))
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(out.shape)}")
    return out


def n_tiles(n_tokens: int, tile: int) -> int:
    return -(-n_tokens // tile)


def zb_abi_version() -> int:
    return int(_lib_handle().zb_abi_version())


def zb_landmark_build(Q: Optional[torch.Tensor], K: torch.Tensor, V: torch.Tensor, tile: int,
                      out: Optional[Landmarks] = None) -> Landmarks:
    """Per-tile means of Q, K, V (see zb.h).  Q may be None (no Qbar)."""
    _need(K, torch.bfloat16, "K", 3)
    _need(V, torch.bfloat16, "V", 3)
    if Q is not None:
        _need(Q, torch.bfloat16, "Q", 3)
    H, N, d = K.shape
    T = n_tiles(N, tile)
    o = out or Landmarks(None, None, None, None)
    Qbar = None if Q is None else _out((H, T, d), torch.float64, K.device, o.Qbar, "Qbar")
    Kbar = _out((H, T, d), torch.float64, K.device, o.Kbar, "Kbar")
    Kb = _out((H, T, d), torch.bfloat16, K.device, o.Kbar_bf16, "Kbar_bf16")
    Vb = _out((H, T, d), torch.bfloat16, K.device, o.Vbar_bf16, "Vbar_bf16")
    st = _lib_handle().zb_landmark_build(_ptr(Q), _ptr(K), _ptr(V), _lib.ZbShape(H, N, d, tile),
                                         _ptr(Qbar), _ptr(Kbar), _ptr(Kb), _ptr(Vb), _stream())
    _check(st, "zb_landmark_build")
    return Landmarks(Qbar, Kbar, Kb, Vb)


def topk_workspace_bytes(heads: int, n_tokens: int, tile: int, head_dim: int = HEAD_DIM) -> int:
    return int(_lib_handle().zb_tile_score_topk_workspace_bytes(_lib.ZbShape(heads, n_tokens, head_dim, tile)))


def zb_tile_score_topk(Qbar: torch.Tensor, Kbar: torch.Tensor, n_tokens: int, tile: int, k: int,
                       out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Indices [H, T, k] (int32, ascending) of the k best key tiles per query tile."""
    _need(Qbar, torch.float64, "Qbar", 3)
    _need(Kbar, torch.float64, "Kbar", 3)
    H, T, d = Kbar.shape
    idx = _out((H, T, k), torch.int32, Kbar.device, out, "idx")
    need = topk_workspace_bytes(H, n_tokens, tile, d) if 0 < k < T else 0
    wsb = _ws(need, Kbar.device, ws) if need else None
    st = _lib_handle().zb_tile_score_topk(_ptr(Qbar), _ptr(Kbar), _lib.ZbShape(H, n_tokens, d, tile),
                                          int(k), _ptr(idx), _ptr(wsb),
                                          0 if wsb is None else wsb.numel() * wsb.element_size(), _stream())
    _check(st, "zb_tile_score_topk")
    return idx


def zb_tile_sparse_attn(Q, K, V, Kbar_bf16, Vbar_bf16, idx, k: int, tile: int,
                        use_landmarks: bool = True, scale: Optional[float] = None,
                        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        want_lse: bool = False, ws: Optional[torch.Tensor] = None,
                        wave_sync: bool = True):
    """Tile-sparse softmax attention with landmarks; returns O (and lse if asked).

    wave_sync passes the call a small workspace (``ws``, or a fresh one) so that
    the work items in flight sweep K/V in step (more L2 reuse); the result is
    the same bit for bit without it."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, n, 3)
    H, N, d = Q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if idx is not None:
        _need(idx, torch.int32, "idx", 3)
    if use_landmarks:
        if Kbar_bf16 is not None:
            _need(Kbar_bf16, torch.bfloat16, "Kbar_bf16", 3)
        if Vbar_bf16 is not None:
            _need(Vbar_bf16, torch.bfloat16, "Vbar_bf16", 3)
    O = _out((H, N, d), torch.bfloat16, Q.device, out, "O")
    if want_lse or lse is not None:
        lse = _out((H, N), torch.float32, Q.device, lse, "lse")
    if wave_sync:
        ws = _ws(int(_lib_handle().zb_tile_sparse_attn_workspace_bytes()), Q.device, ws)
    else:
        ws = None
    st = _lib_handle().zb_tile_sparse_attn(
        _ptr(Q), _ptr(K), _ptr(V), _ptr(Kbar_bf16 if use_landmarks else None),
        _ptr(Vbar_bf16 if use_landmarks else None), _ptr(idx), int(k), 1 if use_landmarks else 0,
        float(scale), _lib.ZbShape(H, N, d, tile), _ptr(O), _ptr(lse), _ptr(ws),
        0 if ws is None else ws.numel() * ws.element_size(), _stream())
    _check(st, "zb_tile_sparse_attn")
    return (O, lse) if lse is not None else O


def zb_dense_attn(Q, K, V, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, want_lse: bool = False, out_fp32: bool = False):
    """Dense softmax attention softmax(scale Q K^T) V on the tensor cores (bf16 or fp32 O)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, n, 3)
    H, Nq, d = Q.shape
    Nk = K.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = _out((H, Nq, d), torch.float32 if out_fp32 else torch.bfloat16, Q.device, out, "O")
    if want_lse or lse is not None:
        lse = _out((H, Nq), torch.float32, Q.device, lse, "lse")
    st = _lib_handle().zb_dense_attn(_ptr(Q), Nq, _ptr(K), _ptr(V), Nk, H, d, float(scale), _ptr(O),
                                     1 if out_fp32 else 0, _ptr(lse), _stream())
    _check(st, "zb_dense_attn")
    return (O, lse) if lse is not None else O


def dense_splits(heads: int, n_q: int, n_kv: int, sms: int, slots_per_sm: int = 2, max_splits: int = 8) -> int:
    """Key splits for zb_dense_attn_split: among the counts that divide n_kv, the one
    whose work items (heads x query tiles x splits, each 1/splits of a row sweep) fill
    the GPU's sms * slots_per_sm attention pipelines in the fewest sweep lengths (ties
    to fewer splits); no split unless that saves at least 5% (each item also loads
    its queries and writes an epilogue, and the parts are merged)."""
    items = heads * -(-n_q // 128)
    slots = max(1, sms * slots_per_sm)
    unsplit = -(-items // slots)
    best, best_cost = 1, unsplit
    for s in range(2, max_splits + 1):
        if n_kv % s:
            continue
        cost = -(-items * s // slots) / s
        if cost < best_cost - 1e-9:
            best, best_cost = s, cost
    return best if best_cost <= 0.95 * unsplit else 1


def dense_split_workspace_bytes(n_q: int, heads: int, splits: int, head_dim: int = HEAD_DIM) -> int:
    return int(_lib_handle().zb_dense_attn_split_workspace_bytes(n_q, heads, head_dim, splits))


def zb_dense_attn_split(Q, K, V, splits: int, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None, want_lse: bool = False, out_fp32: bool = False,
                        ws: Optional[torch.Tensor] = None):
    """Dense softmax attention with the keys split in `splits` equal parts and merged
    (same result as zb_dense_attn; fills the GPU for small query sets)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, n, 3)
    H, Nq, d = Q.shape
    Nk = K.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    O = _out((H, Nq, d), torch.float32 if out_fp32 else torch.bfloat16, Q.device, out, "O")
    if want_lse or lse is not None:
        lse = _out((H, Nq), torch.float32, Q.device, lse, "lse")
    need = dense_split_workspace_bytes(Nq, H, splits, d)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=Q.device)
    st = _lib_handle().zb_dense_attn_split(_ptr(Q), Nq, _ptr(K), _ptr(V), Nk, H, d, float(scale), int(splits), _ptr(O),
                                           1 if out_fp32 else 0, _ptr(lse), _ptr(ws),
                                           0 if ws is None else ws.numel() * ws.element_size(), _stream())
    _check(st, "zb_dense_attn_split")
    return (O, lse) if lse is not None else O


def zb_block_mass(Q, K, lse, block: int = 64, scale: Optional[float] = None,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Dense-softmax mass of every (query block, key block) pair, fp32 [H, Tb, Tb].

    lse: fp32 [H, N], the rows' log-sum-exp from zb_dense_attn(Q, K, V, scale, want_lse=True)."""
    _need(Q, torch.bfloat16, "Q", 3)
    _need(K, torch.bfloat16, "K", 3)
    _need(lse, torch.float32, "lse", 2)
    H, N, d = Q.shape
    if tuple(K.shape) != (H, N, d) or tuple(lse.shape) != (H, N):
        raise ValueError("Q, K must be [H, N, d] and lse [H, N]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Tb = n_tiles(N, block)
    M = _out((H, Tb, Tb), torch.float32, Q.device, out, "M")
    st = _lib_handle().zb_block_mass(_ptr(Q), _ptr(K), _ptr(lse), _lib.ZbShape(H, N, d, block), float(scale),
                                     _ptr(M), _stream())
    _check(st, "zb_block_mass")
    return M


def zb_block_mass_top_fraction(M, m: int, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per query block: the share of its mass held by its m heaviest key blocks, fp32 [H, Tb]."""
    _need(M, torch.float32, "M", 3)
    H, Tb, _ = M.shape
    frac = _out((H, Tb), torch.float32, M.device, out, "frac")
    st = _lib_handle().zb_block_mass_top_fraction(_ptr(M), H, Tb, int(m), _ptr(frac), _stream())
    _check(st, "zb_block_mass_top_fraction")
    return frac


def zb_block_mass_selected_fraction(M, idx, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Per query tile: the share of its mass held by the key tiles of its index list, fp32 [H, T]."""
    _need(M, torch.float32, "M", 3)
    _need(idx, torch.int32, "idx", 3)
    H, T, _ = M.shape
    if tuple(idx.shape[:2]) != (H, T):
        raise ValueError(f"idx must be [{H}, {T}, k], got {tuple(idx.shape)}")
    frac = _out((H, T), torch.float32, M.device, out, "frac")
    st = _lib_handle().zb_block_mass_selected_fraction(_ptr(M), H, T, _ptr(idx), idx.shape[2], _ptr(frac), _stream())
    _check(st, "zb_block_mass_selected_fraction")
    return frac


def linear_state_workspace_bytes(heads: int, n_tokens: int, head_dim: int = HEAD_DIM) -> int:
    return int(_lib_handle().zb_linear_state_workspace_bytes(heads, n_tokens, head_dim))


def affine_fit_workspace_bytes(heads: int, rows: int, head_dim: int = HEAD_DIM) -> int:
    return int(_lib_handle().zb_affine_fit_workspace_bytes(heads, rows, head_dim))


def _ws(nbytes: int, device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is not None and ws.numel() * ws.element_size() >= nbytes:
        return ws
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def zb_linear_state(K, V, S: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None):
    """S = phi(K)^T V [H, d, d] and z = sum phi(K) [H, d] (fp32)."""
    _need(K, torch.bfloat16, "K", 3)
    _need(V, torch.bfloat16, "V", 3)
    H, N, d = K.shape
    S = _out((H, d, d), torch.float32, K.device, S, "S")
    z = _out((H, d), torch.float32, K.device, z, "z")
    need = linear_state_workspace_bytes(H, N, d)
    ws = _ws(need, K.device, ws)
    st = _lib_handle().zb_linear_state(_ptr(K), _ptr(V), H, N, d, _ptr(S), _ptr(z), _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream())
    _check(st, "zb_linear_state")
    return S, z


def key_mean_workspace_bytes(heads: int, n_tokens: int, head_dim: int = HEAD_DIM) -> int:
    return int(_lib_handle().zb_key_mean_workspace_bytes(heads, n_tokens, head_dim))


def zb_key_mean(K, out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """mu = mean of the keys of each head over all tokens, fp32 [H, d] (the linear-centered shift)."""
    _need(K, torch.bfloat16, "K", 3)
    H, N, d = K.shape
    mu = _out((H, d), torch.float32, K.device, out, "mu")
    ws = _ws(key_mean_workspace_bytes(H, N, d), K.device, ws)
    st = _lib_handle().zb_key_mean(_ptr(K), H, N, d, _ptr(mu), _ptr(ws), ws.numel() * ws.element_size(), _stream())
    _check(st, "zb_key_mean")
    return mu


def zb_linear_state_centered(K, V, mu, S: Optional[torch.Tensor] = None, z: Optional[torch.Tensor] = None,
                             ws: Optional[torch.Tensor] = None):
    """S = phi(K - mu)^T V [H, d, d] and z = sum phi(K - mu) [H, d] (fp32), mu fp32 [H, d]."""
    _need(K, torch.bfloat16, "K", 3)
    _need(V, torch.bfloat16, "V", 3)
    _need(mu, torch.float32, "mu", 2)
    H, N, d = K.shape
    if tuple(mu.shape) != (H, d):
        raise ValueError(f"mu must have shape {(H, d)}, got {tuple(mu.shape)}")
    S = _out((H, d, d), torch.float32, K.device, S, "S")
    z = _out((H, d), torch.float32, K.device, z, "z")
    ws = _ws(linear_state_workspace_bytes(H, N, d), K.device, ws)
    st = _lib_handle().zb_linear_state_centered(_ptr(K), _ptr(V), _ptr(mu), H, N, d, _ptr(S), _ptr(z), _ptr(ws),
                                                ws.numel() * ws.element_size(), _stream())
    _check(st, "zb_linear_state_centered")
    return S, z


def zb_linear_apply(Q, S, z, A: Optional[torch.Tensor] = None, b: Optional[torch.Tensor] = None,
                    out: Optional[torch.Tensor] = None, out_fp32: bool = False) -> torch.Tensor:
    """O = (phi(Q) S / (phi(Q) . z)) A + b: bf16 on the tensor cores, or fp32 on the CUDA cores."""
    _need(Q, torch.bfloat16, "Q", 3)
    _need(S, torch.float32, "S", 3)
    _need(z, torch.float32, "z", 2)
    if A is not None:
        _need(A, torch.float32, "A", 3)
    if b is not None:
        _need(b, torch.float32, "b", 2)
    H, N, d = Q.shape
    O = _out((H, N, d), torch.float32 if out_fp32 else torch.bfloat16, Q.device, out, "O")
    st = _lib_handle().zb_linear_apply(_ptr(Q), H, N, d, _ptr(S), _ptr(z), _ptr(A), _ptr(b), _ptr(O),
                                       1 if out_fp32 else 0, _stream())
    _check(st, "zb_linear_apply")
    return O


def linear_attn_workspace_bytes(heads: int, n_tokens: int, head_dim: int = HEAD_DIM) -> int:
    return int(_lib_handle().zb_linear_attn_workspace_bytes(heads, n_tokens, head_dim))


def zb_linear_attn(Q, K, V, A: Optional[torch.Tensor] = None, b: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The whole linear stage in one C call: O = (phi(Q) S / (phi(Q) . z)) A + b, bf16."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.bfloat16, n, 3)
    if A is not None:
        _need(A, torch.float32, "A", 3)
    if b is not None:
        _need(b, torch.float32, "b", 2)
    H, N, d = Q.shape
    O = _out((H, N, d), torch.bfloat16, Q.device, out, "O")
    ws = _ws(linear_attn_workspace_bytes(H, N, d), Q.device, ws)
    st = _lib_handle().zb_linear_attn(_ptr(Q), _ptr(K), _ptr(V), H, N, d, _ptr(A), _ptr(b), _ptr(O), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream())
    _check(st, "zb_linear_attn")
    return O


def zb_affine_fit(X, Y, A: Optional[torch.Tensor] = None, b: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None):
    """Least-squares [A; b] of [X 1] [A; b] = Y per head (vanishing ridge), X, Y fp32 [H, R, d]."""
    _need(X, torch.float32, "X", 3)
    _need(Y, torch.float32, "Y", 3)
    H, R, d = X.shape
    A = _out((H, d, d), torch.float32, X.device, A, "A")
    b = _out((H, d), torch.float32, X.device, b, "b")
    ws = _ws(affine_fit_workspace_bytes(H, R, d), X.device, ws)
    st = _lib_handle().zb_affine_fit(_ptr(X), _ptr(Y), H, R, d, _ptr(A), _ptr(b), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream())
    _check(st, "zb_affine_fit")
    return A, b


def zb_gather_tiles(X, tile: int, tiles: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Whole tiles of X [H, N, d] (tile indices: int32 CUDA tensor) -> [H, n*tile, d]."""
    _need(X, torch.bfloat16, "X", 3)
    _need(tiles, torch.int32, "tiles", 1)
    H, N, d = X.shape
    n = tiles.numel()
    O = _out((H, n * tile, d), torch.bfloat16, X.device, out, "out")
    st = _lib_handle().zb_gather_tiles(_ptr(X), _lib.ZbShape(H, N, d, tile), _ptr(tiles), n, _ptr(O),
                                       _stream())
    _check(st, "zb_gather_tiles")
    return O


def zb_spatial_order(views: int, grid: int = 37, specials: int = 5, win_rows: int = 8, win_cols: int = 16):
    """Token order grouping each view's patches into 2-D windows, and its inverse
    (int32 CPU tensors of views * (specials + grid^2) entries; see zb.h)."""
    n = views * (specials + grid * grid)
    order = torch.empty(n, dtype=torch.int32)
    inverse = torch.empty(n, dtype=torch.int32)
    st = _lib_handle().zb_spatial_order(views, grid, specials, win_rows, win_cols, order.data_ptr(),
                                        inverse.data_ptr())
    _check(st, "zb_spatial_order")
    return order, inverse


def zb_gather_rows(X, rows: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """out[h, r] = X[h, rows[r]] for a bf16 [H, N, d] tensor (rows: int32 CUDA tensor)."""
    _need(X, torch.bfloat16, "X", 3)
    _need(rows, torch.int32, "rows", 1)
    H, N, d = X.shape
    n = rows.numel()
    O = _out((H, n, d), torch.bfloat16, X.device, out, "out")
    st = _lib_handle().zb_gather_rows(_ptr(X), H, N, n, d, _ptr(rows), _ptr(O), _stream())
    _check(st, "zb_gather_rows")
    return O


def zb_last_device_status() -> None:
    """Synchronise the current stream and raise if a kernel recorded a device-side error."""
    st = _lib_handle().zb_last_device_status(_stream())
    _check(st, "device status")


class HybridLayer:
    """Preallocated buffers for one hybrid global-attention layer shape.

    ``sparse(Q, K, V)`` runs the tile-sparse stage (landmarks, selection,
    attention), ``calibrate(Q, K, V)`` fits (A, b) of the linear stage against
    dense attention on whole calibration tiles, ``linear(Q, K, V)`` runs the
    fitted linear stage.  With ``centered=True`` the linear stage is the
    linear-centered variant: keys shifted by their per-head mean before the
    feature map (zb_key_mean, zb_linear_state_centered).  Outputs live in the
    object's buffers and are overwritten by the next call.
    """

    def __init__(self, heads: int, n_tokens: int, tile: int, k: int, calib_tiles: Sequence[int],
                 device="cuda", scale: Optional[float] = None, centered: bool = False,
                 spatial: Optional[Sequence[int]] = None):
        d = HEAD_DIM
        self.centered = centered
        self.heads, self.n_tokens, self.tile, self.k, self.d = heads, n_tokens, tile, k, d
        self.T = n_tiles(n_tokens, tile)
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        dev = torch.device(device)
        H, N, T = heads, n_tokens, self.T
        self.lm = Landmarks(torch.empty(H, T, d, dtype=torch.float64, device=dev),
                            torch.empty(H, T, d, dtype=torch.float64, device=dev),
                            torch.empty(H, T, d, dtype=torch.bfloat16, device=dev),
                            torch.empty(H, T, d, dtype=torch.bfloat16, device=dev))
        self.idx = torch.empty(H, T, k, dtype=torch.int32, device=dev)
        self.ws_topk = torch.empty(max(topk_workspace_bytes(H, N, tile, d), 16), dtype=torch.uint8, device=dev)
        self.ws_attn = torch.empty(int(_lib_handle().zb_tile_sparse_attn_workspace_bytes()), dtype=torch.uint8,
                                   device=dev)
        self.O_sparse = torch.empty(H, N, d, dtype=torch.bfloat16, device=dev)
        self.O_linear = torch.empty(H, N, d, dtype=torch.bfloat16, device=dev)
        self.S = torch.empty(H, d, d, dtype=torch.float32, device=dev)
        self.z = torch.empty(H, d, dtype=torch.float32, device=dev)
        self.ws_lin = torch.empty(max(linear_state_workspace_bytes(H, N, d), 16), dtype=torch.uint8, device=dev)
        self.mu = torch.empty(H, d, dtype=torch.float32, device=dev)
        self.ws_km = torch.empty(max(key_mean_workspace_bytes(H, N, d), 16) if centered else 16, dtype=torch.uint8,
                                 device=dev)
        self.calib = torch.as_tensor(list(calib_tiles), dtype=torch.int32).to(dev)
        R = len(calib_tiles) * tile
        self.R = R
        self.Qc = torch.empty(H, R, d, dtype=torch.bfloat16, device=dev)
        self.Xc = torch.empty(H, R, d, dtype=torch.float32, device=dev)
        self.Yc = torch.empty(H, R, d, dtype=torch.float32, device=dev)
        self.A = torch.empty(H, d, d, dtype=torch.float32, device=dev)
        self.b = torch.empty(H, d, dtype=torch.float32, device=dev)
        self.ws_fit = torch.empty(max(affine_fit_workspace_bytes(H, max(R, d + 1), d), 16), dtype=torch.uint8,
                                  device=dev)
        # the calibration's dense pass splits the keys so that its H x R / 128 work
        # items fill the GPU
        sms = torch.cuda.get_device_properties(dev).multi_processor_count if dev.type == "cuda" else 148
        self.calib_splits = dense_splits(H, R, N, sms)
        self.ws_dense = torch.empty(max(dense_split_workspace_bytes(R, H, self.calib_splits, d), 16),
                                    dtype=torch.uint8, device=dev)
        # spatial tiles: (views, grid, specials, win_rows, win_cols); the sparse stage
        # runs on the tokens gathered into zb_spatial_order's order
        self.spatial = None
        if spatial is not None:
            order, inverse = zb_spatial_order(*spatial)
            if order.numel() != N:
                raise ValueError(f"spatial geometry gives {order.numel()} tokens, the layer has {N}")
            self.spatial = tuple(spatial)
            self.order, self.inverse = order.to(dev), inverse.to(dev)
            self.Qp, self.Kp, self.Vp, self.Op = (torch.empty(H, N, d, dtype=torch.bfloat16, device=dev)
                                                  for _ in range(4))

    # kernel launches of each method (the selection's count depends on the
    # shape and workspace: see launches_per_step)
    LAUNCHES = {
        "sparse": LAUNCHES_PER_CALL["zb_landmark_build"] + LAUNCHES_PER_CALL["zb_tile_sparse_attn"],
        "calibrate": LAUNCHES_PER_CALL["zb_linear_state"] + LAUNCHES_PER_CALL["zb_gather_tiles"]
        + LAUNCHES_PER_CALL["zb_linear_apply"] + LAUNCHES_PER_CALL["zb_affine_fit"],  # + the dense pass
        "linear": LAUNCHES_PER_CALL["zb_linear_apply"],
    }

    def sparse(self, Q, K, V) -> torch.Tensor:
        if self.spatial is not None:
            # spatial tiles: the same stage on the reordered tokens, the output put back
            zb_gather_rows(Q, self.order, out=self.Qp)
            zb_gather_rows(K, self.order, out=self.Kp)
            zb_gather_rows(V, self.order, out=self.Vp)
            Q, K, V = self.Qp, self.Kp, self.Vp
        zb_landmark_build(Q, K, V, self.tile, out=self.lm)
        zb_tile_score_topk(self.lm.Qbar, self.lm.Kbar, self.n_tokens, self.tile, self.k, out=self.idx,
                           ws=self.ws_topk)
        out = self.O_sparse if self.spatial is None else self.Op
        O = zb_tile_sparse_attn(Q, K, V, self.lm.Kbar_bf16, self.lm.Vbar_bf16, self.idx, self.k,
                                self.tile, True, self.scale, out=out, ws=self.ws_attn)
        if self.spatial is not None:
            O = zb_gather_rows(O, self.inverse, out=self.O_sparse)
        return O

    def _state(self, K, V):
        if self.centered:
            zb_key_mean(K, out=self.mu, ws=self.ws_km)
            zb_linear_state_centered(K, V, self.mu, self.S, self.z, self.ws_lin)
        else:
            zb_linear_state(K, V, self.S, self.z, self.ws_lin)

    def calibrate(self, Q, K, V):
        self._state(K, V)
        zb_gather_tiles(Q, self.tile, self.calib, out=self.Qc)
        zb_dense_attn_split(self.Qc, K, V, self.calib_splits, self.scale, out=self.Yc, out_fp32=True,
                            ws=self.ws_dense)
        zb_linear_apply(self.Qc, self.S, self.z, None, None, out=self.Xc, out_fp32=True)
        zb_affine_fit(self.Xc, self.Yc, self.A, self.b, self.ws_fit)
        return self.A, self.b

    def linear(self, Q, K, V, refresh_state: bool = False) -> torch.Tensor:
        if refresh_state:
            self._state(K, V)
        return zb_linear_apply(Q, self.S, self.z, self.A, self.b, out=self.O_linear)

    def save_fit(self, path) -> None:
        """Write the fitted (A, b) of this layer's linear stage to an ``.npz`` file.

        (A, b) is the only state a stage keeps between inputs: a fit made once
        offline on calibration rows serves every later input of the layer.
        """
        import numpy as np
        np.savez(path, A=self.A.detach().cpu().numpy(), b=self.b.detach().cpu().numpy(),
                 heads=self.heads, head_dim=self.d, centered=self.centered)

    def load_fit(self, path) -> None:
        """Read (A, b) written by ``save_fit`` into this layer; ``linear(Q, K, V,
        refresh_state=True)`` then runs the linear stage with it, no calibration."""
        import os
        import numpy as np
        path = os.fspath(path)
        if not os.path.exists(path) and os.path.exists(path + ".npz"):
            path += ".npz"  # numpy's savez adds the suffix when the name has none
        with np.load(path) as f:
            A, b = f["A"], f["b"]
            heads, head_dim, centered = int(f["heads"]), int(f["head_dim"]), bool(f["centered"])
        if (heads, head_dim) != (self.heads, self.d) or A.shape != tuple(self.A.shape) or \
                b.shape != tuple(self.b.shape) or A.dtype != np.float32 or b.dtype != np.float32:
            raise ValueError(f"fit in {path} is for {heads} heads x d = {head_dim} with A {A.shape} "
                             f"{A.dtype}, b {b.shape}; this layer has {self.heads} heads x d = {self.d}")
        if centered != self.centered:
            raise ValueError(f"fit in {path} was made for centered={centered}, this layer has "
                             f"centered={self.centered}")
        self.A.copy_(torch.from_numpy(A))
        self.b.copy_(torch.from_numpy(b))

    def step(self, Q, K, V):
        """One pass of the whole hot path: both stage types on the same input."""
        o_s = self.sparse(Q, K, V)
        self.calibrate(Q, K, V)
        o_l = self.linear(Q, K, V)
        return o_s, o_l

    @property
    def launches_per_step(self) -> int:
        extra = LAUNCHES_PER_CALL["zb_key_mean"] if self.centered else 0
        if self.spatial is not None:
            extra += 4 * LAUNCHES_PER_CALL["zb_gather_rows"]
        topk = topk_launches(self.heads, self.n_tokens, self.tile, self.k, self.ws_topk.numel())
        return (self.LAUNCHES["sparse"] + topk + self.LAUNCHES["calibrate"] + self.dense_launches + extra
                + self.LAUNCHES["linear"])

    @property
    def dense_launches(self) -> int:
        """Kernels of the calibration's dense pass (the dense kernel, and the merge when split)."""
        return LAUNCHES_PER_CALL["zb_dense_attn_split" if self.calib_splits > 1 else "zb_dense_attn"]
