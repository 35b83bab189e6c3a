"""A stack of hybrid global-attention layers run back to back on one GPU.

"Zebra3D: Efficient Hybrid Foundation Models For Scalable 3D Reconstruction",
Table 20 caption: an "xL/yS" model makes a share x of its global-attention
layers linear and runs the others tile-sparse with a share y of attention rows
dropped; Table 6 lists which of VGGT's layers become linear.  Each layer here
is one ``HybridLayer`` call sequence on that layer's own Q, K, V:

  * a tile-sparse layer: landmarks -> tile selection -> tile-sparse attention;
  * a linear layer: linear state -> calibration (gather whole query tiles,
    dense attention on them, unfitted linear output, closed-form fit) ->
    fitted linear output on all rows.

Host-side scheduling only (the arithmetic is all in the library's kernels).
Each layer's calls split into an input side that needs only the layer's own
Q, K, V (landmarks and selection; linear state and calibration gather) and the
rest.  With ``lookahead`` the input side of layer l + 1 is issued on a second
stream while layer l's attention runs on the caller's stream, so it can fill
the SMs that layer l's last work items leave idle.  Two buffer sets alternate
between layers, and events order every reuse, so the results are the same bit
for bit with and without lookahead.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch

from . import (HybridLayer, zb_affine_fit, zb_dense_attn_split, zb_gather_tiles, zb_landmark_build,
               zb_linear_apply, zb_tile_score_topk, zb_tile_sparse_attn)


class HybridStack:
    """Buffers and streams for ``n_layers`` hybrid layers of one shape.

    ``linear_layers`` are the indices of the linear layers; every other layer
    is tile-sparse with ``k`` kept key tiles per query tile.
    """

    def __init__(self, heads: int, n_tokens: int, tile: int, k: int, calib_tiles: Sequence[int],
                 n_layers: int, linear_layers: Sequence[int], device="cuda", scale: Optional[float] = None):
        self.n_layers = n_layers
        self.linear = frozenset(int(l) for l in linear_layers)
        if any(l < 0 or l >= n_layers for l in self.linear):
            raise ValueError("linear layer index out of range")
        self.bufs = [HybridLayer(heads, n_tokens, tile, k, calib_tiles, device=device, scale=scale)
                     for _ in range(2)]
        self.device = torch.device(device)
        self.side = torch.cuda.Stream(device=self.device)

    def is_linear(self, layer: int) -> bool:
        return layer in self.linear

    # ------------------------------------------------------------- halves ----
    def _front(self, layer: int, buf: HybridLayer, Q, K, V) -> None:
        """Calls that read only the layer's own inputs."""
        if self.is_linear(layer):
            buf._state(K, V)
            zb_gather_tiles(Q, buf.tile, buf.calib, out=buf.Qc)
        else:
            zb_landmark_build(Q, K, V, buf.tile, out=buf.lm)
            zb_tile_score_topk(buf.lm.Qbar, buf.lm.Kbar, buf.n_tokens, buf.tile, buf.k, out=buf.idx,
                               ws=buf.ws_topk)

    def _back(self, layer: int, buf: HybridLayer, Q, K, V) -> torch.Tensor:
        """The rest of the layer; returns its output buffer."""
        if self.is_linear(layer):
            zb_dense_attn_split(buf.Qc, K, V, buf.calib_splits, buf.scale, out=buf.Yc, out_fp32=True, ws=buf.ws_dense)
            zb_linear_apply(buf.Qc, buf.S, buf.z, None, None, out=buf.Xc, out_fp32=True)
            zb_affine_fit(buf.Xc, buf.Yc, buf.A, buf.b, buf.ws_fit)
            return zb_linear_apply(Q, buf.S, buf.z, buf.A, buf.b, out=buf.O_linear)
        return zb_tile_sparse_attn(Q, K, V, buf.lm.Kbar_bf16, buf.lm.Vbar_bf16, buf.idx, buf.k, buf.tile, True,
                                   buf.scale, out=buf.O_sparse, ws=buf.ws_attn)

    def launches(self) -> int:
        """Kernels one pass of the stack launches."""
        n = 0
        for l in range(self.n_layers):
            b = self.bufs[l & 1]
            calib = b.LAUNCHES["calibrate"] + b.dense_launches
            if self.is_linear(l):
                n += calib + b.LAUNCHES["linear"]
            else:
                n += b.launches_per_step - calib - b.LAUNCHES["linear"]
        return n

    # ---------------------------------------------------------------- run ----
    def run(self, inputs: Sequence, lookahead: bool = True,
            on_layer_done: Optional[Callable[[int, torch.Tensor], None]] = None,
            layer_events: Optional[Sequence] = None) -> None:
        """Run every layer once on the caller's current stream.

        ``inputs[l]`` is layer l's (Q, K, V).  ``on_layer_done(l, O)`` is called
        right after layer l's last call is issued, on the caller's stream; what it
        enqueues there may read any of layer l's buffers (``self.bufs[l & 1]``):
        it runs before layer l + 2 reuses them.
        ``layer_events[l]`` (a pair of timing events, serial runs only) brackets
        layer l on the caller's stream."""
        if lookahead and layer_events is not None:
            raise ValueError("per-layer events need lookahead=False")
        main = torch.cuda.current_stream(self.device)
        L = self.n_layers
        if not lookahead:
            for l in range(L):
                Q, K, V = inputs[l]
                buf = self.bufs[l & 1]
                if layer_events is not None:
                    layer_events[l][0].record(main)
                self._front(l, buf, Q, K, V)
                O = self._back(l, buf, Q, K, V)
                if layer_events is not None:
                    layer_events[l][1].record(main)
                if on_layer_done is not None:
                    on_layer_done(l, O)
            return
        front_done = [torch.cuda.Event() for _ in range(L)]
        back_done = [torch.cuda.Event() for _ in range(L)]
        start = torch.cuda.Event()
        start.record(main)
        Q, K, V = inputs[0]
        self._front(0, self.bufs[0], Q, K, V)
        for l in range(L):
            if l + 1 < L:
                # input side of layer l + 1 on the side stream, into the buffer set
                # that layer l - 1 used (free once layer l - 1 is done)
                self.side.wait_event(back_done[l - 1] if l >= 1 else start)
                Qn, Kn, Vn = inputs[l + 1]
                with torch.cuda.stream(self.side):
                    self._front(l + 1, self.bufs[(l + 1) & 1], Qn, Kn, Vn)
                    front_done[l + 1].record(self.side)
            if l >= 1:
                main.wait_event(front_done[l])
            Q, K, V = inputs[l]
            O = self._back(l, self.bufs[l & 1], Q, K, V)
            if on_layer_done is not None:
                on_layer_done(l, O)
            back_done[l].record(main)
        # the side stream's last work is layer L-1's input side, which the main
        # stream has already waited for
