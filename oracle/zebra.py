"""fp64 CPU oracle for the Zebra3D hybrid global-attention layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  It
shares no code with the CUDA path (``linear_hybrid_attention_b200``) and must
never be reached from it.

Plain NumPy in float64.  Every function states the passage it follows.  The
sources are web pages describing one preprint; they give no formulas, so each
function names both the passage and the reading taken where the pages are
silent.  Sources, by page title:

[ABS]  "Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D
       Reconstruction" -- Abstract: tolerant stages get linear(-centered)
       attention, sensitive stages get tile-sparse attention with landmark
       summaries of the unselected context; a closed-form affine fit makes the
       conversion training-free.
[FIG1] same title -- Figure 1 (a) caption: selected tiles keep full softmax
       interactions, every omitted tile is replaced by a mean-key/mean-value
       landmark.
[HOW]  "Zebra3D speeds up 3D reconstruction by up to 7.1x on 1024 frames
       without training from scratch" -- section "How Zebra3D works":
       tile-sparse attention computes only selected token blocks; linear parts
       are fitted with a closed-form affine map (no gradient descent).
[T20]  same title as [ABS] -- Table 20 caption: in "xL/yS", y is the sparsity
       of attention rows in the non-linear layers.

Readings where the pages are silent (the same list is kept in the design
notes): tiles are contiguous runs of ``tile`` tokens of the flattened
[views x tokens] sequence, the last one ragged; the tile score is the dot
product of the mean query of the query tile and the mean key of the key tile;
the top-k tie-break is the lower key-tile index; a landmark's logit carries a
bias of ln(n_j) (natural log, n_j = tokens in tile j); softmax scale is
1/sqrt(d); the linear feature map is elu(x)+1 on unscaled q and k,
non-causal, with no epsilon; the affine map acts on row vectors, y = x A + b,
fitted by least squares with an intercept; "linear-centered" attention
centres each head's keys by their mean over all tokens before phi, and leaves
the queries as they are.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "tile_lengths", "landmark_means", "tile_scores", "select_tiles",
    "sparse_attention", "dense_attention", "elu_plus_one", "linear_state",
    "linear_apply", "linear_attention", "linear_attention_quadratic", "affine_fit",
    "affine_apply", "calibration_rows", "RIDGE_REL", "key_mean", "linear_state_centered",
    "linear_attention_centered", "block_mass", "top_mass_fraction", "selected_mass_fraction",
    "spatial_order", "inverse_order", "spatial_sparse_attention",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def tile_lengths(n_tokens: int, tile: int) -> np.ndarray:
    """n_j for j = 0..T-1: ``tile`` tokens each, the last tile holds the rest.

    Reading of "spatial tiles" [FIG1]: contiguous runs of the flattened token
    order, T = ceil(N / tile).
    """
    if n_tokens < 1 or tile < 1:
        raise ValueError("n_tokens and tile must be positive")
    T = -(-n_tokens // tile)
    n = np.full(T, tile, dtype=np.int64)
    n[-1] = n_tokens - (T - 1) * tile
    return n


def landmark_means(X, tile: int) -> np.ndarray:
    """Per-tile mean of the rows of X [H, N, d] -> [H, T, d] (fp64).

    [FIG1]: an omitted tile becomes one token whose key is the mean key and
    whose value is the mean value of the tile.  The same pooling of Q gives the
    mean query used for tile scoring.  A sum of at most a few hundred bf16
    values is exact in fp64 (unless the values span more than ~38 binades), so
    the result does not depend on summation order.
    """
    X = _f64(X)
    H, N, d = X.shape
    n = tile_lengths(N, tile)
    T = n.shape[0]
    out = np.empty((H, T, d), dtype=np.float64)
    full = (T - 1) * tile
    if T > 1:
        out[:, : T - 1, :] = X[:, :full, :].reshape(H, T - 1, tile, d).sum(axis=2)
    out[:, T - 1, :] = X[:, full:, :].sum(axis=1)
    out /= n[None, :, None].astype(np.float64)
    return out


def tile_scores(Qbar, Kbar) -> np.ndarray:
    """score[h, i, j] = Qbar[h, i] . Kbar[h, j] (fp64), all query/key tile pairs.

    The pages name the selection ("selected tiles", [FIG1]) but not its
    criterion; the reading taken is the mean-pooled query/key dot product.
    """
    Qbar = _f64(Qbar)
    Kbar = _f64(Kbar)
    return np.matmul(Qbar, np.swapaxes(Kbar, -1, -2))


def select_tiles(scores, k: int) -> np.ndarray:
    """Indices of the k largest scores in each row, ascending -> int64 [..., k].

    Order is (score descending, key-tile index ascending), i.e. equal scores
    go to the lower index; the kept set is then listed in ascending order.
    The budget k is the kept fraction of key tiles (the y of "xL/yS" is the
    dropped fraction [T20]).
    """
    scores = _f64(scores)
    T = scores.shape[-1]
    if not 0 <= k <= T:
        raise ValueError("k must be in [0, T]")
    flat = scores.reshape(-1, T)
    out = np.empty((flat.shape[0], k), dtype=np.int64)
    j = np.arange(T)
    for r in range(flat.shape[0]):
        order = np.lexsort((j, -flat[r]))  # primary: -score, secondary: j
        out[r] = np.sort(order[:k])
    return out.reshape(scores.shape[:-1] + (k,))


def _softmax_rows(logits: np.ndarray) -> np.ndarray:
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / e.sum(axis=-1, keepdims=True)


def sparse_attention(Q, K, V, tile: int, idx, scale: float,
                     use_landmarks: bool = True,
                     query_tiles: Optional[Sequence[int]] = None) -> np.ndarray:
    """Tile-sparse softmax attention with mean-key/value landmarks.

    [FIG1], [HOW]: for a query row r of query tile i, softmax runs over
      * every key of every selected tile j in idx[h, i] with logit s * q_r . k_c,
      * one landmark per unselected tile j (if ``use_landmarks``) with logit
        s * q_r . Kbar_j + ln(n_j) and value Vbar_j,
    and O_r is the softmax-weighted sum of the matching values.  The ln(n_j)
    bias makes a landmark weigh as much as n_j identical keys.

    Q, K, V: [H, N, d]; idx: int [H, T, k] (any order); returns [H, N, d], or
    [H, len(query_tiles) * tile, d] (rows of the listed tiles, in list order;
    rows past N in a ragged tile are zero) when ``query_tiles`` is given.
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    H, N, d = Q.shape
    n = tile_lengths(N, tile)
    T = n.shape[0]
    idx = np.asarray(idx, dtype=np.int64)
    starts = np.arange(T, dtype=np.int64) * tile
    Kbar = landmark_means(K, tile) if use_landmarks else None
    Vbar = landmark_means(V, tile) if use_landmarks else None
    tiles = range(T) if query_tiles is None else list(query_tiles)
    if query_tiles is None:
        O = np.zeros((H, N, d), dtype=np.float64)
    else:
        O = np.zeros((H, len(tiles) * tile, d), dtype=np.float64)
    for h in range(H):
        for slot, i in enumerate(tiles):
            sel = np.unique(idx[h, i])
            rows = slice(starts[i], starts[i] + n[i])
            q = Q[h, rows]
            keys = [np.arange(starts[j], starts[j] + n[j]) for j in sel]
            cols = np.concatenate(keys) if keys else np.zeros(0, dtype=np.int64)
            logit_parts = [scale * q @ K[h, cols].T]
            value_parts = [V[h, cols]]
            if use_landmarks:
                mask = np.ones(T, dtype=bool)
                mask[sel] = False
                lm = np.nonzero(mask)[0]
                logit_parts.append(scale * q @ Kbar[h, lm].T + np.log(n[lm].astype(np.float64))[None, :])
                value_parts.append(Vbar[h, lm])
            logits = np.concatenate(logit_parts, axis=1)
            if logits.shape[1] == 0:
                raise ValueError("query tile with no keys and no landmarks")
            P = _softmax_rows(logits)
            out = P @ np.concatenate(value_parts, axis=0)
            if query_tiles is None:
                O[h, rows] = out
            else:
                O[h, slot * tile: slot * tile + n[i]] = out
    return O


def dense_attention(Q, K, V, scale: float) -> np.ndarray:
    """Dense softmax attention softmax(s * Q K^T) V per head (the unconverted layer).

    Q: [H, Nq, d], K, V: [H, Nk, d] -> [H, Nq, d].
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    out = np.empty(Q.shape[:2] + (V.shape[-1],), dtype=np.float64)
    for h in range(Q.shape[0]):
        out[h] = _softmax_rows(scale * Q[h] @ K[h].T) @ V[h]
    return out


def elu_plus_one(x) -> np.ndarray:
    """phi(x) = elu(x) + 1: x + 1 for x > 0, exp(x) for x <= 0 (always > 0).

    The pages call the tolerant-stage operator linear attention [ABS] but do
    not give its feature map; elu+1 is the reading taken.
    """
    x = _f64(x)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def linear_state(K, V):
    """S = phi(K)^T V  [H, d, d] and z = sum_r phi(k_r)  [H, d] (fp64)."""
    fk = elu_plus_one(K)
    V = _f64(V)
    S = np.matmul(np.swapaxes(fk, -1, -2), V)
    z = fk.sum(axis=-2)
    return S, z


def linear_attention(Q, K, V, A=None, b=None) -> np.ndarray:
    """Non-causal linear attention, associative form, then the affine map.

    O_r = (phi(q_r) S / (phi(q_r) . z)) A + b, with S, z from ``linear_state``.
    A: [H, d, d] (row-vector convention, y = x A), b: [H, d]; None means the
    identity / zero (the unfitted operator, "Linear, no fit" in Table 3 (a) of
    [ABS]'s page).
    """
    S, z = linear_state(K, V)
    return linear_apply(Q, S, z, A, b)


def linear_apply(Q, S, z, A=None, b=None) -> np.ndarray:
    """Output of the linear stage from a given state: (phi(q) S / (phi(q) . z)) A + b."""
    fq = elu_plus_one(Q)
    num = np.matmul(fq, _f64(S))
    den = np.matmul(fq, _f64(z)[..., None])
    return affine_apply(num / den, A, b)


def linear_attention_quadratic(Q, K, V) -> np.ndarray:
    """The same operator in quadratic form: row-normalised (phi(Q) phi(K)^T) V."""
    fq, fk = elu_plus_one(Q), elu_plus_one(K)
    W = np.matmul(fq, np.swapaxes(fk, -1, -2))
    W = W / W.sum(axis=-1, keepdims=True)
    return np.matmul(W, _f64(V))


def key_mean(K) -> np.ndarray:
    """mu_h = (1/N) sum_r k_r, the mean key of each head over all N tokens -> [H, d] (fp64)."""
    K = _f64(K)
    return K.sum(axis=-2) / K.shape[-2]


def linear_state_centered(K, V):
    """State of the linear-centered operator: ``linear_state`` of the centred keys k_r - mu_h.

    [ABS] names "linear-centered" attention for the tolerant stages and Table 3
    (a) of its page compares "Linear, uncentered fit" with "Linear-centered +
    fit"; neither gives a formula.  Reading: the keys of each head are centred
    by their mean over all tokens before the feature map, and the queries are
    left as they are.  Softmax attention is unchanged by subtracting one vector
    from every key (q . (k - mu) = q . k - q . mu is the same for all keys of a
    query), so the dense layer the fit targets stays the same, while phi, not
    being shift-invariant, sees zero-mean keys.
    """
    K = _f64(K)
    return linear_state(K - key_mean(K)[..., None, :], V)


def linear_attention_centered(Q, K, V, A=None, b=None) -> np.ndarray:
    """Linear-centered attention: (phi(q_r) S_c / (phi(q_r) . z_c)) A + b, S_c, z_c of the centred keys."""
    S, z = linear_state_centered(K, V)
    return linear_apply(Q, S, z, A, b)


def affine_apply(X, A=None, b=None) -> np.ndarray:
    """y = x A + b per head (row vectors).  A: [H, d, d], b: [H, d]."""
    X = _f64(X)
    Y = X if A is None else np.matmul(X, _f64(A))
    if b is not None:
        Y = Y + _f64(b)[:, None, :]
    return Y


RIDGE_REL = 1e-8


def affine_fit(X, Y, ridge_rel: float = RIDGE_REL):
    """Closed-form affine map per head: [A; b] minimising ||[X 1][A; b] - Y||_F^2 + lam ||A||_F^2.

    [ABS], [HOW]: the linear stage's output is corrected by an affine map fitted
    in closed form (no gradient descent) against the dense layer's output on
    calibration rows.  X, Y: [H, R, d] -> A [H, d, d], b [H, d].

    Reading: least squares with an intercept and, among its minimisers, the
    one whose A has minimum norm, computed with a vanishing ridge
    lam = ridge_rel * max_i ((X - mean X)^T (X - mean X))_ii on A (not on b).
    The intercept absorbs the means, so this is least squares on the centred
    data, A = argmin ||Xc A - Yc||^2 + lam ||A||^2, b = mean(Y) - mean(X) A,
    which tends to the minimum-norm solution as lam -> 0.  The minimiser is
    not unique for the linear stage: its output rows all satisfy
    O . (S^-1 z) = 1, so the centred calibration matrix has rank d - 1.  The
    ridge only damps directions carrying under sqrt(ridge_rel) of the largest
    singular value.  Solved as an augmented least-squares problem
    [Xc; sqrt(lam) I] A = [Yc; 0] with an fp64 least-squares routine.
    """
    X, Y = _f64(X), _f64(Y)
    H, R, d = X.shape
    A = np.empty((H, d, d), dtype=np.float64)
    b = np.empty((H, d), dtype=np.float64)
    for h in range(H):
        xm = X[h].mean(axis=0)
        ym = Y[h].mean(axis=0)
        Xc = X[h] - xm
        Yc = Y[h] - ym
        lam = ridge_rel * float((Xc * Xc).sum(axis=0).max())
        D = np.concatenate([Xc, np.sqrt(lam) * np.eye(d)], axis=0)
        T = np.concatenate([Yc, np.zeros((d, Y.shape[-1]))], axis=0)
        W, *_ = np.linalg.lstsq(D, T, rcond=None)
        A[h] = W
        b[h] = ym - xm @ W
    return A, b


def block_mass(Q, K, scale: float, block: int) -> np.ndarray:
    """Softmax mass of every (query block, key block) pair of dense attention -> [H, T, T] (fp64).

    M[h, a, b] = sum over query rows r of block a and keys c of block b of
    p_rc, p = softmax over all keys of scale * q_r . k_c.  Blocks are runs of
    ``block`` tokens in sequence order, the last one ragged (the tiling of
    ``tile_lengths``).  The pages measure this with 64 x 64 token blocks on a
    dense pass to show how concentrated attention is ([ABS]'s page, Figure 2
    (b) and Figure 8: mass kept by the heaviest 20% of 64 x 64 blocks).
    """
    Q, K = _f64(Q), _f64(K)
    H, N, _ = Q.shape
    nb = tile_lengths(N, block)
    starts = np.arange(len(nb)) * block
    out = np.zeros((H, len(nb), len(nb)), dtype=np.float64)
    for h in range(H):
        for a in range(len(nb)):
            r0 = a * block
            P = _softmax_rows(scale * Q[h, r0:r0 + nb[a]] @ K[h].T)
            out[h, a] = np.add.reduceat(P.sum(axis=0), starts)
    return out


def top_mass_fraction(M, m: int) -> np.ndarray:
    """Share of each query block's mass held by its m heaviest key blocks -> [H, T].

    Reading: the pages' selection of the heaviest 20% of 64 x 64 token blocks
    (Figure 2 (b), Figure 8) is made per query block, like the method's
    per-query-tile selection, with m = ceil(0.2 T) supplied by the caller.
    """
    M = _f64(M)
    heavy_first = -np.sort(-M, axis=-1)
    return heavy_first[..., :m].sum(axis=-1) / M.sum(axis=-1)


def selected_mass_fraction(M, idx) -> np.ndarray:
    """Share of each query tile's mass held by the key tiles in its index list -> [H, T].

    M: block masses at the tile size ([H, T, T]); idx: [H, T, k] selected key
    tiles (from ``select_tiles``), so this is the dense-softmax mass that the
    method's mean-pooled selection keeps exactly.
    """
    M = _f64(M)
    kept = np.take_along_axis(M, np.asarray(idx, dtype=np.int64), axis=-1)
    return kept.sum(axis=-1) / M.sum(axis=-1)


def calibration_rows(n_tokens: int, tile: int, tiles: Sequence[int]) -> np.ndarray:
    """Token rows of the listed whole calibration tiles, in list order."""
    n = tile_lengths(n_tokens, tile)
    rows = [np.arange(j * tile, j * tile + n[j]) for j in tiles]
    return np.concatenate(rows).astype(np.int64)


def spatial_order(views: int, grid: int = 37, specials: int = 5, win_rows: int = 8, win_cols: int = 16) -> np.ndarray:
    """Token order that groups each view's patch tokens into 2-D windows -> int64 [views * tokens].

    "3D reconstruction drops dense attention layer by layer ...", synopsis:
    exact softmax over selected *spatial* tiles.  Reading: a view holds
    ``specials`` camera/register tokens followed by its grid x grid patch
    tokens in row-major order (patch (y, x) at offset specials + grid*y + x).
    The new order keeps the views in sequence; inside a view the special
    tokens come first, then the patches window by window -- windows of
    win_rows x win_cols patches (those at the right and bottom edges smaller),
    taken in row-major order over the window grid, patches row-major inside a
    window.  Position p of the new sequence holds original token order[p];
    contiguous tiles of the new sequence then cover compact 2-D regions.
    """
    per_view = specials + grid * grid
    one = list(range(specials))
    for wy in range(0, grid, win_rows):
        for wx in range(0, grid, win_cols):
            for y in range(wy, min(wy + win_rows, grid)):
                for x in range(wx, min(wx + win_cols, grid)):
                    one.append(specials + grid * y + x)
    one = np.asarray(one, dtype=np.int64)
    return np.concatenate([v * per_view + one for v in range(views)])


def inverse_order(order) -> np.ndarray:
    """inv with inv[order[p]] = p: position of each original token in the new order."""
    order = np.asarray(order, dtype=np.int64)
    inv = np.empty_like(order)
    inv[order] = np.arange(order.shape[0], dtype=np.int64)
    return inv


def spatial_sparse_attention(Q, K, V, tile: int, order, scale: float, k: int,
                             use_landmarks: bool = True) -> np.ndarray:
    """Tile-sparse attention over spatial tiles: the tokens are put in ``order``
    (``spatial_order``), tiled, selected (mean-pooled scores, top k) and attended
    exactly as in ``sparse_attention``, and each output row goes back to its
    token's original position.  Softmax attention itself does not depend on the
    token order; only which tokens share a tile does.  Returns (O, idx) with
    idx the selection on the reordered tiles."""
    order = np.asarray(order, dtype=np.int64)
    Qp, Kp, Vp = _f64(Q)[:, order], _f64(K)[:, order], _f64(V)[:, order]
    idx = select_tiles(tile_scores(landmark_means(Qp, tile), landmark_means(Kp, tile)), k)
    Op = sparse_attention(Qp, Kp, Vp, tile, idx, scale, use_landmarks=use_landmarks)
    return Op[:, inverse_order(order)], idx
