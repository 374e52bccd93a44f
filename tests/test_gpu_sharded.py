"""The sharded step through the real library on one GPU.

sharding.sharded_step at world size 1 (inside an NCCL process group of one
rank, as bench.py runs it under torchrun) must be exactly the library's step:
the partition gives every matrix to rank 0 and no exchange is needed.  The
multi-rank exchange itself is tested with gloo on CPU (test_sharding_gloo.py).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import muon_family_optimizer_b200 as mo
import oracle
from conftest import rel_fro
from muon_family_optimizer_b200 import sharding
from muon_family_optimizer_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

QUINTIC = (3.4445, -4.7750, 2.0315)
HP = dict(mu=0.95, eta=0.02, gamma=1.0, beta_a=0.9, alpha=0.5, **{"lambda": 0.1})
SHAPES = [(256, 256), (192, 520), (520, 192), (64, 1024)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _state():
    out = []
    for j, (r, c) in enumerate(SHAPES):
        out.append(dict(W=syn.initial_weight("gpt2_small", j, r, c).to(torch.bfloat16).cuda(),
                        G=syn.gradient("gpt2_small", j, 0, r, c).to(torch.bfloat16).cuda(),
                        G_prev=syn.gradient("gpt2_small", j, 8, r, c).to(torch.bfloat16).cuda(),
                        A=torch.zeros(r, c, device="cuda"), M=torch.zeros(r, c, device="cuda")))
    return out


def test_sharded_step_world_one_is_the_library_step():
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    from datetime import timedelta
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0),
                            timeout=timedelta(seconds=60))
    try:
        params = _state()
        host = [{k: v.double().cpu().numpy() for k, v in p.items()} for p in params]
        ref = _state()
        sched = mo.quintic_schedule(5)
        ws = torch.empty(mo.muon_workspace_size(params, mo.BF16, sched), dtype=torch.uint8, device="cuda")
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        stream = torch.cuda.Stream()
        a = sharding.sharded_step(params, mo.BF16, mo.BF16, HP, sched, ws, 0, 1, d_status=status, stream=stream)
        assert a == [list(range(len(SHAPES)))]
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        mo.muon_step_batched(ref, mo.BF16, mo.BF16, HP, sched, ws)
        torch.cuda.synchronize()
        for p, q, h in zip(params, ref, host):
            for k in ("W", "G_prev", "A", "M"):
                assert torch.equal(p[k], q[k]), k
            o = oracle.muon_step(h["W"], h["G"], h["G_prev"], h["A"], h["M"], mu=HP["mu"], eta=HP["eta"],
                                 lam=HP["lambda"], gamma=HP["gamma"], beta_a=HP["beta_a"], alpha=HP["alpha"],
                                 coeffs=[QUINTIC] * 5, round_to=oracle.ROUND_BF16)
            assert rel_fro(p["W"].double().cpu().numpy(), o["W"]) <= 2.0 ** -8
        with pytest.raises(ValueError):   # rank / world size must match the group
            sharding.sharded_step(params, mo.BF16, mo.BF16, HP, sched, ws, 0, 2)
    finally:
        dist.destroy_process_group()
