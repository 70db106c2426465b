"""Probe-parallel CD-RGE across processes, one per GPU.

The pith.science review ("What carries the argument") describes the
distributed scheme: the model is broadcast to the workers once, each worker
computes a few perturbed forward losses, and only scalar losses travel.  Here
every rank holds the same theta, evaluates a contiguous slice of the n_pert
probes (zo_probe_losses_slice), the 2 x n_pert scalar losses are all-gathered
(torch.distributed; NCCL on GPUs, gloo on CPU), and every rank then computes
the same coefficients and applies the same update, so the replicas stay
bit-identical without ever re-broadcasting theta.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def probe_slice(n_pert: int, rank: int, world: int):
    """(first probe, count) of rank's contiguous share; the first n % world
    ranks take one extra probe."""
    base, extra = divmod(n_pert, world)
    count = base + (1 if rank < extra else 0)
    begin = rank * base + min(rank, extra)
    return begin, count


def gather_losses(lp_local: torch.Tensor, lm_local: torch.Tensor, n_pert: int, group=None):
    """All-gather every rank's slice of L+ / L- into full [n_pert] tensors
    (same device as the inputs).  Slices are padded to a common length for
    the collective and re-assembled in rank order."""
    world = dist.get_world_size(group)
    counts = [probe_slice(n_pert, r, world)[1] for r in range(world)]
    m = max(counts)
    dev = lp_local.device
    # gloo gathers host tensors: device slices travel through host memory
    via = torch.device("cpu") if dist.get_backend(group) == "gloo" else dev
    mine = torch.zeros(2, m, dtype=lp_local.dtype, device=via)
    mine[0, :lp_local.numel()] = lp_local.to(via)
    mine[1, :lm_local.numel()] = lm_local.to(via)
    parts = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(parts, mine, group=group)
    lp = torch.cat([p[0, :c] for p, c in zip(parts, counts)]).to(dev)
    lm = torch.cat([p[1, :c] for p, c in zip(parts, counts)]).to(dev)
    return lp, lm


def cdrge_step_sharded(ctx, theta, step_seed, n_pert, eps, eta, tokens, targets, coeffs,
                       group=None, stream=None):
    """One CD-RGE update with the probes split over the ranks of `group`.
    Returns the gathered (L+, L-) device tensors."""
    import zero_order_recurrent_b200 as zo
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    begin, count = probe_slice(n_pert, rank, world)
    lp_local = torch.empty(max(count, 1), device=theta.device)
    lm_local = torch.empty(max(count, 1), device=theta.device)
    if count:
        zo.zo_probe_losses_slice(ctx, theta, step_seed, begin, count, eps, tokens, targets,
                                 lp_local, lm_local, stream=stream)
    lp, lm = gather_losses(lp_local[:count], lm_local[:count], n_pert, group)
    zo.zo_coeffs(ctx, lp, lm, n_pert, eps, eta, coeffs, stream=stream)
    zo.zo_update(ctx, theta, step_seed, n_pert, coeffs, stream=stream)
    return lp, lm
