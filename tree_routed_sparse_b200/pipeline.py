"""Batches from host memory through the fused path, with the copies overlapped.

A server holds each batch (Q, K, V and the predictor weights, or budgets) in pinned host memory
and wants the attention output back in host memory. HostPipeline runs every submitted batch
through alhr.build_tree and alhr.forward on a compute stream while the next batch's inputs are
copied in on a second stream and the previous batch's output is copied out on a third; device
buffers are double-buffered (or single-buffered when two sets do not fit: the copies then wait
for the kernels) and the streams are ordered by events, so a buffer is refilled only after the
kernels that read it are done and an output buffer is reused only after it was copied out.
Every batch is still copied in full and read back in full.
"""
from __future__ import annotations

import torch

from . import alhr


class HostPipeline:
    """Double-buffered host -> device -> host runner of the fused path.

    like: a dict of host tensors with the shapes and dtypes of one batch (keys Q, K, V, and W
    and/or budget_override, None when absent). kw: the keyword arguments of alhr.forward
    (q_start, window, max_keys, score_bits, value_bound, score_norm, bucket_log).
    flush: an optional device buffer that is overwritten on the compute stream before every
    batch's kernels (to start each batch with a cold L2; part of the batch's time).
    buffers: 2 (copies overlap the neighbouring batches' kernels) or 1 (half the device memory).
    """

    def __init__(self, like: dict, device=None, flush: torch.Tensor | None = None,
                 buffers: int = 2, **kw):
        if buffers not in (1, 2):
            raise ValueError(f"buffers {buffers}: 1 or 2")
        self.nbuf = buffers
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.kw = kw
        self.vb = kw.get("value_bound", 16)
        self.keys = [k for k in ("Q", "K", "V", "W", "budget_override") if like.get(k) is not None]
        B, H, n, d = like["K"].shape
        nq = like["Q"].shape[2]
        self.bufs = [{k: torch.empty(like[k].shape, dtype=like[k].dtype, device=self.device)
                      for k in self.keys} for _ in range(self.nbuf)]
        tb = alhr.tree_bytes(n, d, self.vb)
        self.trees = [torch.empty((B, H, tb), dtype=torch.uint8, device=self.device)
                      for _ in range(self.nbuf)]
        self.outs = [torch.empty((B, H, nq, d), dtype=torch.float32, device=self.device)
                     for _ in range(self.nbuf)]
        self.copy_in = torch.cuda.Stream(self.device)
        self.compute = torch.cuda.Stream(self.device)
        self.copy_out = torch.cuda.Stream(self.device)
        ev = lambda: [torch.cuda.Event() for _ in range(self.nbuf)]
        self.in_done, self.comp_done, self.out_done = ev(), ev(), ev()
        self.flush = flush
        self.step = 0

    def submit(self, host: dict, host_out: torch.Tensor) -> None:
        """Queue one batch: `host` holds pinned input tensors (as `like`), `host_out` a pinned
        float32 [B, H, nq, d] tensor that receives the output. Returns at once; both must stay
        untouched until synchronize()."""
        b = self.step % self.nbuf
        buf = self.bufs[b]
        with torch.cuda.stream(self.copy_in):
            if self.step >= self.nbuf:
                self.copy_in.wait_event(self.comp_done[b])  # the batch before has read buffer b
            for k in self.keys:
                buf[k].copy_(host[k], non_blocking=True)
            self.in_done[b].record(self.copy_in)
        with torch.cuda.stream(self.compute):
            self.compute.wait_event(self.in_done[b])
            if self.step >= self.nbuf:
                self.compute.wait_event(self.out_done[b])  # output b of the batch before copied out
            if self.flush is not None:
                self.flush.fill_(self.step & 0xFF)
            alhr.build_tree(buf["K"], self.trees[b], value_bound=self.vb)
            alhr.forward(buf["Q"], buf["K"], buf["V"], self.trees[b], W=buf.get("W"),
                         budget_override=buf.get("budget_override"), out=self.outs[b],
                         **self.kw)
            self.comp_done[b].record(self.compute)
        with torch.cuda.stream(self.copy_out):
            self.copy_out.wait_event(self.comp_done[b])
            host_out.copy_(self.outs[b], non_blocking=True)
            self.out_done[b].record(self.copy_out)
        self.step += 1

    def synchronize(self) -> None:
        for s in (self.copy_in, self.compute, self.copy_out):
            s.synchronize()
