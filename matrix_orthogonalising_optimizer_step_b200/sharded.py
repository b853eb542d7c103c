"""Ownership-sharded data-parallel Muon step and the global S_max, over
torch.distributed (NCCL on GPUs).

Why this shape ("MuonClip: speed, then stability", §08 "A matrix-aware
optimizer becomes a collective-communication problem"): Newton-Schulz needs
the whole matrix (orthogonalising pieces of a matrix separately is a different
operation), so the unit of work is a whole matrix, and the per-head maximum of
QK-Clip must cover the whole data-parallel batch, or the clip would depend on
how samples were assigned to ranks; the rescaled weights must then agree on
every replica.

Layout.  Every rank keeps every weight (a replica), in one flat buffer laid out
by owner: rank r's segment holds the matrices r owns (mc_shard_plan), each at a
256-byte-aligned offset, and all segments have one padded length.  Gradients
use the same layout in a buffer of the gradient dtype.  Momenta exist only on
the owner.

Step (``ShardedMuon.step``):
  1. reduce-scatter (sum) of the gradient buffer: rank r receives the summed
     gradients of the matrices it owns;
  2. the Muon step of the owned matrices on this GPU (``muon_step`` of the C
     ABI), in place on their slots of the weight buffer;
  3. all-gather of the weight buffer, in place: every replica gets every
     updated matrix.

The gradients are summed, not averaged: the Newton-Schulz input is divided by
its Frobenius norm, and momentum is linear in the gradients, so a constant
factor on every gradient leaves the update unchanged (below the norm floor eps
aside); this saves a scaling pass.

QK-Clip (``global_smax``): each rank computes S_max over its own batch, one
all-reduce (max) of H floats makes it global, and every rank then runs the
same clip on the same weights, which keeps the replicas identical.

Each matrix's result does not depend on which other matrices share its call,
so the sharded step is the single-GPU step on the summed gradients, bit for
bit.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

from . import muon_step, shard_plan

_ALIGN = 256


def _dist():
    import torch.distributed as dist
    return dist


def _round_up(x: int, a: int) -> int:
    return (x + a - 1) // a * a


class ShardedMuon:
    """Flat replicated weights, owner-laid-out gradients and owner-only momenta
    for ``shapes`` (a list of (rows, cols)), plus the sharded step.

    ``weights[i]`` and ``grads[i]`` are views into the flat buffers: let the
    model read its parameters from ``weights`` and write (accumulate) its local
    gradients into ``grads``.  ``moms[i]`` is an fp32 tensor on the owner of
    matrix i and None elsewhere.  ``local_step`` defaults to the C-ABI Muon
    step; it is called as ``local_step(Ws, Gs, Ms, **hparams)`` on the owned
    matrices.
    """

    def __init__(self, shapes: Sequence, *, w_dtype, g_dtype, device, group=None, ns_steps: int = 5,
                 local_step: Optional[Callable] = None):
        import torch
        dist = _dist()
        self.group = group
        if dist.is_available() and dist.is_initialized():
            self.world = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
        else:
            self.world, self.rank = 1, 0
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        self.owner, self.load = shard_plan(self.shapes, self.world, ns_steps)
        self.local_step = local_step if local_step is not None else muon_step
        wes = torch.empty((), dtype=w_dtype).element_size()
        ges = torch.empty((), dtype=g_dtype).element_size()

        # byte offsets of each matrix inside its owner's segment
        w_off, g_off = [0] * len(self.shapes), [0] * len(self.shapes)
        w_used, g_used = [0] * self.world, [0] * self.world
        for i, (r, c) in enumerate(self.shapes):
            o = self.owner[i]
            w_off[i] = w_used[o]
            g_off[i] = g_used[o]
            w_used[o] = _round_up(w_used[o] + r * c * wes, _ALIGN)
            g_used[o] = _round_up(g_used[o] + r * c * ges, _ALIGN)
        self.w_seg = max(max(w_used), _ALIGN)
        self.g_seg = max(max(g_used), _ALIGN)

        self.w_flat = torch.zeros(self.world * self.w_seg, dtype=torch.uint8, device=device)
        g_flat_bytes = torch.zeros(self.world * self.g_seg, dtype=torch.uint8, device=device)
        self.g_flat = g_flat_bytes.view(g_dtype)
        if self.world > 1:
            self.g_red = torch.zeros(self.g_seg // ges, dtype=g_dtype, device=device)
        else:
            self.g_red = self.g_flat
        g_red_bytes = self.g_red.view(torch.uint8)

        self.weights, self.grads, self._red = [], [], []
        for i, (r, c) in enumerate(self.shapes):
            o = self.owner[i]
            wb = o * self.w_seg + w_off[i]
            gb = o * self.g_seg + g_off[i]
            self.weights.append(self.w_flat[wb:wb + r * c * wes].view(w_dtype).view(r, c))
            self.grads.append(g_flat_bytes[gb:gb + r * c * ges].view(g_dtype).view(r, c))
            if o == self.rank:
                self._red.append(g_red_bytes[g_off[i]:g_off[i] + r * c * ges].view(g_dtype).view(r, c))
            else:
                self._red.append(None)
        self.owned = [i for i, o in enumerate(self.owner) if o == self.rank]
        self.moms = [torch.zeros(s, dtype=torch.float32, device=device) if self.owner[i] == self.rank else None
                     for i, s in enumerate(self.shapes)]

    def step(self, **hparams) -> None:
        """Reduce-scatter the gradients, update the owned matrices, all-gather
        the weights.  ``hparams`` go to ``local_step`` (mu, nesterov, lr, wd,
        ns_steps, a, b, c, eps, rms_scale, coeffs, stream, ...)."""
        dist = _dist()
        if self.world > 1:
            dist.reduce_scatter_tensor(self.g_red, self.g_flat, op=dist.ReduceOp.SUM, group=self.group)
        if self.owned:
            self.local_step([self.weights[i] for i in self.owned], [self._red[i] for i in self.owned],
                            [self.moms[i] for i in self.owned], **hparams)
        if self.world > 1:
            mine = self.w_flat[self.rank * self.w_seg:(self.rank + 1) * self.w_seg]
            dist.all_gather_into_tensor(self.w_flat, mine, group=self.group)


def global_smax(smax, group=None):
    """All-reduce (max) of a per-head S_max tensor in place, so that the clip
    covers the whole data-parallel batch; returns it."""
    dist = _dist()
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(smax, op=dist.ReduceOp.MAX, group=group)
    return smax
