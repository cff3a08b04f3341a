"""Sequence-parallel SQuad-Attention over a process group: one all-to-all between the passes.

Both passes of SQuad-Attention are sequence-local (SQuad paper §3.2): the local pass needs the tokens of
one window, the global pass the tokens of one slot across all windows of one frame. So the n tokens of a
block can be split over R ranks with one exchange between the passes:

* rank r holds a band of whole window rows: latent rows y in [r*H/R, (r+1)*H/R) of every frame, as a
  [B, h, T*(H/R)*W, d] tensor in (t, y, x) order. Its windows are complete, so the local pass runs there.
* an all-to-all regroups the band into frame groups: rank r then holds frames [r*T/R, (r+1)*T/R) of
  every row. Its slot sequences are complete (a slot (t, dy, dx) only reaches tokens of frame t), so the
  global pass runs there with the same window (its temporal extent is the frame group).
* a second all-to-all returns the output to the bands.

The global-then-local order runs the same steps the other way round, and the backward retraces them.
Requirements: T % R == 0, H % hw == W % ww == 0 and (H / hw) % R == 0.

Compute is the library's single-pass forward and backward (`local_only` / `global_only`). Around each
exchange the library's squad_seqpar_reorder moves the blocks between the band, frame-group and
all-to-all layouts, and adds the two passes' dQ and dK shares while moving the second one back; the
exchange itself is torch.distributed.all_to_all_single on those buffers, so on GPUs it is NCCL over
NVLink. The per-rank compute and the reordering can be replaced (`fwd`, `bwd`, `reorder` arguments) for
testing the composition without a GPU. With one rank both exchanges are the identity and the band is
the whole grid, so the library's fused two-pass forward and its backward run directly (no exchange
buffers, no single-pass split).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class SeqParallelSquad:
    def __init__(self, grid, window, group=None, fwd=None, bwd=None, reorder=None):
        self.group = group
        self.R = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        T, H, W = grid
        tw, hw, ww = window
        if tw != T or H % hw or W % ww or T % self.R or (H // hw) % self.R:
            raise ValueError("needs tw == T, a window that divides H x W, T % R == 0 and (H / hw) % R == 0")
        self.grid, self.window = tuple(grid), tuple(window)
        self.Hb, self.Tg = H // self.R, T // self.R
        self.band_grid = (T, self.Hb, W)                   # the local pass's grid on this rank
        self.frame_grid = (self.Tg, H, W)                  # the global pass's grid on this rank
        self.frame_window = (self.Tg, hw, ww)
        # one rank with the library's own compute: the fused launch, no exchange
        self.whole = self.R == 1 and fwd is None and bwd is None
        if fwd is None or bwd is None or reorder is None:
            from .api import squad_attn_bwd, squad_attn_fwd, squad_seqpar_reorder
            fwd = fwd or (lambda q, k, v, g, w, o: squad_attn_fwd(q, k, v, g, w, o))
            bwd = bwd or (lambda q, k, v, out, do, ws, g, w, o: squad_attn_bwd(q, k, v, out, do, ws, g, w, o))
            reorder = reorder or squad_seqpar_reorder
        self._fwd, self._bwd, self._reorder = fwd, bwd, reorder

    # -------------------------------------------------------------------------------- exchange
    def _a2a(self, send):
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=self.group)
        return recv

    def band_to_frames(self, x):
        """[B, h, T*Hb*W, d] (this rank's rows, all frames) -> [B, h, Tg*H*W, d] (its frames, all rows)."""
        send = self._reorder(x, self.grid, self.R, "band", "chunks")       # a chunk per frame group
        recv = self._a2a(send)                                             # a chunk per row band
        return self._reorder(recv, self.grid, self.R, "chunks", "frames")

    def frames_to_band(self, x, add=None):
        """[B, h, Tg*H*W, d] -> [B, h, T*Hb*W, d], the inverse of band_to_frames; plus `add` (a band
        tensor) if given."""
        send = self._reorder(x, self.grid, self.R, "frames", "chunks")     # a chunk per row band
        recv = self._a2a(send)                                             # a chunk per frame group
        return self._reorder(recv, self.grid, self.R, "chunks", "band", add=add)

    # -------------------------------------------------------------------------------- passes
    def _local(self, q, k, v):
        return self._fwd(q, k, v, self.band_grid, self.window, "local_only")

    def _global(self, q, k, v):
        return self._fwd(q, k, v, self.frame_grid, self.frame_window, "global_only")

    def forward(self, q, k, v, order="local_then_global"):
        """q, k, v: this rank's band. Returns (o band, ctx for backward)."""
        if order not in ("local_then_global", "global_then_local"):
            raise ValueError(order)
        if self.whole:
            o, ws = self._fwd(q, k, v, self.grid, self.window, order)
            return o, ("whole", order, q, k, v, o, ws)
        if order == "local_then_global":
            o1, ws1 = self._local(q, k, v)
            qf, kf, o1f = self.band_to_frames(q), self.band_to_frames(k), self.band_to_frames(o1)
            of, ws2 = self._global(qf, kf, o1f)
            return self.frames_to_band(of), (order, q, k, v, o1, ws1, qf, kf, o1f, of, ws2)
        if order == "global_then_local":
            qf, kf, vf = self.band_to_frames(q), self.band_to_frames(k), self.band_to_frames(v)
            o1f, ws1 = self._global(qf, kf, vf)
            o1 = self.frames_to_band(o1f)
            o, ws2 = self._local(q, k, o1)
            return o, (order, q, k, v, o1, o, ws2, qf, kf, vf, o1f, ws1)
        raise ValueError(order)

    def backward(self, ctx, dout):
        """dout: this rank's band of the upstream gradient. Returns (dq, dk, dv) bands."""
        if ctx[0] == "whole":
            _, order, q, k, v, o, ws = ctx
            return self._bwd(q, k, v, o, dout, ws, self.grid, self.window, order)
        order = ctx[0]
        if order == "local_then_global":
            _, q, k, v, o1, ws1, qf, kf, o1f, of, ws2 = ctx
            dqf, dkf, do1f = self._bwd(qf, kf, o1f, of, self.band_to_frames(dout), ws2, self.frame_grid,
                                       self.frame_window, "global_only")
            do1 = self.frames_to_band(do1f)
            dq_l, dk_l, dv = self._bwd(q, k, v, o1, do1, ws1, self.band_grid, self.window, "local_only")
            return self.frames_to_band(dqf, add=dq_l), self.frames_to_band(dkf, add=dk_l), dv
        _, q, k, v, o1, o, ws2, qf, kf, vf, o1f, ws1 = ctx
        dq_l, dk_l, do1 = self._bwd(q, k, o1, o, dout, ws2, self.band_grid, self.window, "local_only")
        dqf, dkf, dvf = self._bwd(qf, kf, vf, o1f, self.band_to_frames(do1), ws1, self.frame_grid,
                                  self.frame_window, "global_only")
        return self.frames_to_band(dqf, add=dq_l), self.frames_to_band(dkf, add=dk_l), self.frames_to_band(dvf)


def band_of(x, grid, rank, R):
    """The band of rows [rank*H/R, (rank+1)*H/R) of every frame of a full [B, h, T*H*W, d] tensor."""
    B, h, _, d = x.shape
    T, H, W = grid
    Hb = H // R
    return x.reshape(B, h, T, H, W, d)[:, :, :, rank * Hb:(rank + 1) * Hb].reshape(B, h, T * Hb * W, d)
