"""Multi-rank host logic of the sharded step, on CPU with gloo (world size 2 and
3, and two 2-rank subgroups of a 4-rank world).

Each rank updates the matrices partition() gives it (the per-matrix step is the
fp64 oracle here: the CUDA library is not needed to test the exchange), then
gather_weights() brings every replica's W up to date with one all-gather.
Every rank's W, and the owned optimizer state, must equal a single-process
oracle step of all matrices.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from muon_family_optimizer_b200 import sharding

QUINTIC = (3.4445, -4.7750, 2.0315)
HP = dict(mu=0.95, eta=0.02, gamma=1.0, beta_a=0.9, alpha=0.5, **{"lambda": 0.1})
SHAPES = [(48, 48), (48, 48), (48, 160), (160, 48), (32, 96), (96, 32), (16, 16)]


def _state(seed=5):
    g = torch.Generator().manual_seed(seed)
    out = []
    for r, c in SHAPES:
        out.append({k: torch.randn(r, c, generator=g, dtype=torch.float64) * s
                    for k, s in (("W", 0.02), ("G", 1.0), ("G_prev", 1.0), ("A", 1e-2), ("M", 1e-1))})
    return out


def _oracle_step(p):
    ref = oracle.muon_step(p["W"].numpy(), p["G"].numpy(), p["G_prev"].numpy(), p["A"].numpy(), p["M"].numpy(),
                           mu=HP["mu"], eta=HP["eta"], lam=HP["lambda"], gamma=HP["gamma"], beta_a=HP["beta_a"],
                           alpha=HP["alpha"], coeffs=[QUINTIC] * 5)
    for k in ("W", "G_prev", "A", "M"):
        p[k].copy_(torch.from_numpy(ref[k]))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue, subgroups=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        oracle.set_num_threads(1)
        params = _state()
        group = None
        grank, gworld = rank, world
        if subgroups:
            # two subgroups {0, 2} and {1, 3}: every rank creates both, then steps in its own
            groups = [dist.new_group([0, 2]), dist.new_group([1, 3])]
            group = groups[rank % 2]
            grank, gworld = dist.get_rank(group), dist.get_world_size(group)
        assignment = sharding.sharded_step(params, None, None, HP, None, None, grank, gworld, group=group,
                                           step_fn=lambda mine: [_oracle_step(p) for p in mine])
        queue.put((grank, assignment, {j: {k: v.numpy().copy() for k, v in p.items()} for j, p in enumerate(params)}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,subgroups", [(2, False), (3, False), (4, True)])
def test_sharded_step_matches_single_process(world, subgroups):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, queue, subgroups)) for r in range(world)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = _state()
    for p in ref:
        _oracle_step(p)
    for rank, assignment, params in results:
        owner = sharding.owners(assignment)
        assert sorted(owner) == list(range(len(SHAPES)))
        for j, p in params.items():
            # every replica's weights are the full step's
            assert np.array_equal(p["W"], ref[j]["W"].numpy()), (rank, j)
            # optimizer state is updated only by the owner
            if owner[j] == rank:
                for k in ("A", "M", "G_prev"):
                    assert np.array_equal(p[k], ref[j][k].numpy()), (rank, j, k)


def test_partition_balanced_and_deterministic():
    from muon_family_optimizer_b200 import synthetic as syn
    shapes = syn.WORKLOADS["llama3_8b"]["shapes"]
    for world in (1, 2, 4, 8):
        a = sharding.partition(shapes, world)
        assert a == sharding.partition(shapes, world)
        assert sorted(j for idx in a for j in idx) == list(range(len(shapes)))
        loads = [sum(sharding.matrix_cost(*shapes[j]) for j in idx) for idx in a]
        biggest = max(sharding.matrix_cost(*s) for s in shapes)
        # greedy longest-first: no rank exceeds the mean by more than one matrix
        assert max(loads) - sum(loads) / world <= biggest
    with pytest.raises(ValueError):
        sharding.partition(shapes, 0)


def test_exchange_numel_is_the_largest_share():
    ws = [torch.zeros(r, c) for r, c in SHAPES]
    a = sharding.partition(SHAPES, 3)
    assert sharding.exchange_numel(ws, a) == max(sum(r * c for r, c in (SHAPES[j] for j in idx)) for idx in a)
    assert sharding.exchange_numel(ws, [[], []] + [list(range(len(SHAPES)))]) == sum(r * c for r, c in SHAPES)


def test_partition_edge_cases():
    assert sharding.partition([], 4) == [[], [], [], []]
    assert sharding.partition([(8, 8)], 3) == [[0], [], []]
