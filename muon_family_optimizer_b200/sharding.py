"""Data-parallel sharding of one Muon step across ranks.

Every matrix's step is independent (the MONA pass is elementwise, the
orthogonalisation is per matrix), so the step partitions by whole matrices:
each rank updates the matrices it owns -- its share of the optimizer state
(G_prev, A, M) lives only there -- and one exchange brings every replica's
weights up to date.  The exchange is one all-gather (NCCL over NVLink on
GPUs, gloo in the CPU tests): every rank packs the weights it owns into a
flat buffer padded to the largest rank's share, and after the all-gather
copies the other ranks' weights out of the gathered buffer.

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


def exchange_numel(weights, assignment):
    """Elements per rank of the padded all-gather: the largest rank's share."""
    return max([sum(weights[j].numel() for j in idx) for idx in assignment] + [1])


def gather_weights(weights, assignment, group=None, buffers=None):
    """Bring every rank's copy of each W (list of tensors, same order, shapes
    and dtype on all ranks) up to date from its owner with one all-gather.

    `assignment` lists the matrices of each rank of `group` (indexed by the
    rank within the group).  `buffers` = (send, recv) may be passed to reuse
    the flat buffers (send: exchange_numel elements, recv: world times that);
    they are allocated otherwise.  The collective and the copies are ordered
    on the current stream (torch's NCCL backend waits for it)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    me = dist.get_rank(group)
    if len(assignment) != world:
        raise ValueError(f"assignment has {len(assignment)} ranks, the group {world}")
    if world == 1:
        return
    per = exchange_numel(weights, assignment)
    ref = weights[0]
    if buffers is None:
        send = torch.empty(per, dtype=ref.dtype, device=ref.device)
        recv = torch.empty(world * per, dtype=ref.dtype, device=ref.device)
    else:
        send, recv = buffers
        if send.numel() < per or recv.numel() < world * per:
            raise ValueError("exchange buffers too small")
        send, recv = send[:per], recv[:world * per]
    off = 0
    for j in assignment[me]:
        n = weights[j].numel()
        send[off:off + n].copy_(weights[j].reshape(-1))
        off += n
    dist.all_gather_into_tensor(recv, send, group=group)
    for r, idx in enumerate(assignment):
        if r == me:
            continue
        off = r * per
        for j in idx:
            n = weights[j].numel()
            weights[j].copy_(recv[off:off + n].view_as(weights[j]))
            off += n


def sharded_step(params, w_dtype, ns_dtype, hp, schedule, workspace, rank, world_size, group=None,
                 d_status=None, stream=None, step_fn=None, buffers=None):
    """One step over all matrices on `world_size` ranks: muon_step_batched on
    this rank's share, then the weight exchange.  params: the full list (same
    order and shapes on every rank; only the owned entries' G, G_prev, A, M are
    read or written).  rank / world_size: this rank and the size of `group`
    (the default group when None).  The step runs on `stream` (torch's current
    stream when None) and the exchange is ordered after it on the same stream.
    step_fn(owned_params) replaces the library call (tests)."""
    import torch.distributed as dist
    if dist.is_initialized():
        if dist.get_rank(group) != rank or dist.get_world_size(group) != world_size:
            raise ValueError("rank / world_size do not match the process group")
    shapes = [tuple(p["W"].shape) for p in params]
    assignment = partition(shapes, world_size)
    mine = [params[j] for j in assignment[rank]]
    if mine:
        if step_fn is not None:
            step_fn(mine)
        else:
            mo.muon_step_batched(mine, w_dtype, ns_dtype, hp, schedule, workspace, d_status=d_status,
                                 stream=stream)
    if world_size > 1:
        if stream is not None and params[0]["W"].is_cuda:
            with torch.cuda.stream(stream):
                gather_weights([p["W"] for p in params], assignment, group=group, buffers=buffers)
        else:
            gather_weights([p["W"] for p in params], assignment, group=group, buffers=buffers)
    return assignment
