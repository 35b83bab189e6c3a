"""Oracle jobs for the stack parity test, run in worker processes (spawned).

Each job reads one head's Q, K, V (bf16 bit patterns saved as .npy by the
test) and computes, with the fp64 oracle only, what the test compares the
GPU's sampled outputs against.  No torch, no CUDA here.
"""
from __future__ import annotations

import numpy as np

import oracle


def limit_threads(n: int) -> None:
    """Worker initializer: n BLAS threads per worker."""
    from threadpoolctl import threadpool_limits
    threadpool_limits(n)


def _load_head(paths):
    out = []
    for p in paths:
        bits = np.load(p)                                   # uint16 [N, d]
        out.append((bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)[None])
    return out


def sparse_job(paths, tile: int, k: int, tiles, scale: float):
    """Selection rows and tile-sparse output rows of the listed query tiles."""
    q, kk, v = _load_head(paths)
    Qb = oracle.landmark_means(q, tile)
    Kb = oracle.landmark_means(kk, tile)
    idx = oracle.select_tiles(oracle.tile_scores(Qb[:, tiles], Kb), k)[0]
    T = Kb.shape[1]
    full = np.zeros((1, T, k), dtype=np.int64)
    full[0, tiles] = idx
    out = oracle.sparse_attention(q, kk, v, tile, full, scale, query_tiles=tiles)[0]
    return idx, out


def linear_job(paths, tile: int, calib_tiles, tiles, scale: float, chunk: int = 64):
    """Fitted linear output rows of the listed query tiles: fit on the calibration
    tiles against dense attention (evaluated in row chunks)."""
    q, kk, v = _load_head(paths)
    N = q.shape[1]
    rows = oracle.calibration_rows(N, tile, calib_tiles)
    X = oracle.linear_attention(q[:, rows], kk, v)
    Y = np.concatenate([oracle.dense_attention(q[:, rows[c:c + chunk]], kk, v, scale)
                        for c in range(0, len(rows), chunk)], axis=1)
    A, b = oracle.affine_fit(X, Y)
    srows = oracle.calibration_rows(N, tile, tiles)
    return oracle.linear_attention(q[:, srows], kk, v, A, b)[0]
