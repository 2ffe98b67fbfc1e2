"""Data-parallel block calibration over calibration samples.

The block-wise objective ("【ICLR 2024】OmniQuant: ...", section 框架) is a mean over the
calibration samples, and its parameters (the LWC logits and the LET vectors, a few MB for a
LLaMA-7B block) are shared by all of them. So ranks that each take a different sample, run the
block step to its gradient, and average their gradient vectors follow the gradient of the mean
over their samples; every rank then applies the same AdamW update and keeps an identical copy
of the parameters. One process per GPU; the exchange is one all-reduce of the block's
parameter-gradient vector and one of the loss per step, over a torch.distributed process group
(NCCL over NVLink / NVSwitch on a multi-GPU node, gloo on the host). The update is the
library's AdamW kernel with the block's two learning rates, the same arithmetic the block step
applies itself when it updates in place.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def world_size(group=None) -> int:
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def allreduce_mean_(tensors, group=None):
    """In place: each tensor becomes the mean over the ranks of the group (a sum, then one
    division by the world size, so every rank holds bitwise the same values). Every rank must
    call it with the same tensors in the same order."""
    world = world_size(group)
    if world == 1:
        return tensors
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        t.div_(world)
    return tensors


class DataParallelBlock:
    """One rank's share of a block's data-parallel calibration.

    ``blk`` is this rank's ``omq.Block`` with the same weights and initial parameters on every
    rank. ``step(x, y_ref)`` runs the block step on this rank's sample without updating,
    averages the gradient vector and the loss over the group, and applies AdamW to both
    parameter segments (LWC logits at ``blk.lr_lwc``, LET vectors at ``blk.lr_let``)."""

    def __init__(self, blk, group=None):
        self.blk = blk
        self.group = group
        self.n_lwc = blk.theta_slices["s1"][0]     # the LWC logits precede the LET vectors

    def step(self, x, y_ref, stream=None):
        """One data-parallel step. With ``stream`` given, the whole step (the block kernels,
        the all-reduce and the update) is ordered on that stream: it becomes the current
        stream for the duration, since a collective orders itself against the current stream
        of its caller, not against the stream its inputs were produced on."""
        if stream is not None and stream != torch.cuda.current_stream(stream.device):
            with torch.cuda.stream(stream):
                return self._step(x, y_ref)
        return self._step(x, y_ref)

    def _step(self, x, y_ref):
        from . import omq
        blk = self.blk
        blk.step(x, y_ref, update=False)
        allreduce_mean_([blk.d_theta, blk.loss], self.group)
        blk.t += 1
        n = self.n_lwc
        omq.adamw_step(blk.theta[:n], blk.d_theta[:n], blk.adam_m[:n], blk.adam_v[:n],
                       blk.lr_lwc, blk.t)
        omq.adamw_step(blk.theta[n:], blk.d_theta[n:], blk.adam_m[n:], blk.adam_v[n:],
                       blk.lr_let, blk.t)
        return blk.loss

    def calibrate(self, xs, y_refs, epochs: int):
        """``epochs`` passes over this rank's samples xs [S, M, D] with targets y_refs
        [S, M, D] (every rank the same S): step i of a pass takes this rank's sample i, so the
        group advances on world-size samples per step. Returns the averaged loss of every step
        (device tensor [epochs * S])."""
        S = xs.shape[0]
        counts = torch.tensor([S], dtype=torch.int64, device=xs.device)
        if world_size(self.group) > 1:
            lo, hi = counts.clone(), counts.clone()
            dist.all_reduce(lo, op=dist.ReduceOp.MIN, group=self.group)
            dist.all_reduce(hi, op=dist.ReduceOp.MAX, group=self.group)
            if int(lo.item()) != int(hi.item()):
                raise ValueError("every rank must hold the same number of samples")
        losses = torch.empty(epochs * S, dtype=torch.float32, device=xs.device)
        for e in range(epochs):
            for i in range(S):
                losses[e * S + i:e * S + i + 1].copy_(self.step(xs[i], y_refs[i]))
        return losses
