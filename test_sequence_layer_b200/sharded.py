"""Sequence-sharded Mesa forward over torch.distributed ranks.

Each rank holds one consecutive slice of every sequence (rank order =
sequence order) and computes the output of its slice. The only exchange is
one all-gather of the slices' state summaries (see mesa_chunk_state and
mesa_state_prefix in mesa.h): every rank scans its slice from a zero state to
(Delta, D), the summaries of all ranks are gathered, and each rank forms the
state entering its slice and runs the forward from it.

Method: "MesaNet: Sequence Modeling by Locally Optimal Test-Time Training"
(gist.science), Technical summary > Method > Mesa layer, "Parallelisation"
(the layer carries H_t, G_t from chunk to chunk).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import mesa


def gather_slice_summaries(H, G, decay, group=None):
    """All-gather of one summary per rank, stacked in rank order:
    ([W, *H.shape], [W, *G.shape], [W, *decay.shape]). Works on any backend
    that implements all_gather (NCCL for device tensors, gloo for host ones)."""
    W = dist.get_world_size(group) if dist.is_initialized() else 1
    if W == 1:                                         # one slice: the gather is the identity
        return tuple(t.unsqueeze(0) for t in (H, G, decay))
    out = []
    for t in (H, G, decay):
        t = t.contiguous()
        parts = [torch.empty_like(t) for _ in range(W)]
        dist.all_gather(parts, t, group=group)
        out.append(torch.stack(parts))
    return tuple(out)


def forward_sequence_sharded(q, k, v, gamma, beta, lam, *, group=None, chunk=64, cg_steps=15, tol=0.0,
                             return_iters=False, workspace=None, stream=None):
    """The forward of this rank's slice [B,H,T_r,*] of sequences split over the
    ranks of `group` in rank order (without an initialised process group: one
    slice). Returns out [B,H,T_r,dv] (plus iters). `workspace` (optional)
    serves both the slice scan and the forward, which run one after the other
    on `stream`: at least mesa.workspace_size() bytes."""
    r = dist.get_rank(group) if dist.is_initialized() else 0
    H_s, G_s, d_s = mesa.chunk_state(k, v, gamma, beta, chunk=chunk, workspace=workspace, stream=stream)
    H_all, G_all, d_all = gather_slice_summaries(H_s, G_s, d_s, group)
    H_in, G_in = mesa.state_prefix(H_all, G_all, d_all, r, stream=stream)
    return mesa.forward(q, k, v, gamma, beta, lam, chunk=chunk, cg_steps=cg_steps, tol=tol, H_in=H_in, G_in=G_in,
                        return_iters=return_iters, workspace=workspace, stream=stream)
