"""Data-parallel sharding of one Muon step across ranks.

Every matrix's step is independent (the MONA pass is elementwise, the
orthogonalisation is per matrix), so the step partitions by whole matrices:
each rank updates the matrices it owns -- its share of the optimizer state
(G_prev, A, M) lives only there -- and one exchange brings every replica's
weights up to date.  The exchange is one broadcast per rank of the flattened
weights it owns (NCCL over NVLink on GPUs, gloo in the CPU tests).

partition() balances the algorithmic Newton-Schulz flops per rank
(3 s^2 l + s^3 per quintic step for an s x l wide view), longest first onto the
least-loaded rank, ties to the lower rank: deterministic, so every rank
computes the same assignment without communicating.
"""
import torch

import muon_family_optimizer_b200 as mo


def matrix_cost(rows, cols, ns_steps=5):
    s, l = min(rows, cols), max(rows, cols)
    return ns_steps * (3.0 * s * s * l + float(s) ** 3)


def partition(shapes, world_size, ns_steps=5):
    """Owner rank of each matrix: list (one entry per rank) of sorted matrix indices."""
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    order = sorted(range(len(shapes)), key=lambda j: (-matrix_cost(*shapes[j], ns_steps), j))
    load = [0.0] * world_size
    owned = [[] for _ in range(world_size)]
    for j in order:
        r = min(range(world_size), key=lambda q: (load[q], q))
        owned[r].append(j)
        load[r] += matrix_cost(*shapes[j], ns_steps)
    return [sorted(o) for o in owned]


def owners(assignment):
    """Matrix index -> owner rank."""
    out = {}
    for r, idx in enumerate(assignment):
        for j in idx:
            out[j] = r
    return out


def gather_weights(weights, assignment, group=None):
    """Bring every rank's copy of each W (list of tensors, same order on all
    ranks) up to date from its owner: one broadcast per rank of the flat
    concatenation of the weights it owns."""
    import torch.distributed as dist
    for r, idx in enumerate(assignment):
        if not idx:
            continue
        flat = torch.cat([weights[j].reshape(-1) for j in idx])
        dist.broadcast(flat, src=r, group=group)
        off = 0
        for j in idx:
            n = weights[j].numel()
            if dist.get_rank(group) != r:
                weights[j].copy_(flat[off:off + n].view_as(weights[j]))
            off += n


def sharded_step(params, w_dtype, ns_dtype, hp, schedule, workspace, rank, world_size, group=None,
                 d_status=None, stream=None, step_fn=None):
    """One step over all matrices on `world_size` ranks: muon_step_batched on
    this rank's share, then the weight exchange.  params: the full list (same
    order and shapes on every rank; only the owned entries' G, G_prev, A, M are
    read or written).  step_fn(owned_params) replaces the library call (tests)."""
    shapes = [tuple(p["W"].shape) for p in params]
    assignment = partition(shapes, world_size)
    mine = [params[j] for j in assignment[rank]]
    if mine:
        if step_fn is not None:
            step_fn(mine)
        else:
            mo.muon_step_batched(mine, w_dtype, ns_dtype, hp, schedule, workspace, d_status=d_status,
                                 stream=stream)
    gather_weights([p["W"] for p in params], assignment, group=group)
    return assignment
