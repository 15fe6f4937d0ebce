"""The sharded Muon step (ownership of whole matrices by Newton-Schulz FLOPs,
owner-only momentum, owner broadcast of the updated weights over NCCL) with
the library's CUDA step as the local step.

Every GPU call in this environment has one GPU, so the step runs at world
size 1 here: the plan, the local CUDA step and the NCCL broadcasts all run,
and the result must be the plain MuonStep's, bit for bit, and the oracle's
within the stated tolerance.  The exchange between two or three ranks is
covered on CPU (tests/test_multirank_cpu.py, gloo).
"""
import datetime
import math
import socket

import pytest
import torch

import newton_schulz_matrix_b200 as nsm
import oracle
import synth
from parity_util import Q5, rel, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_sharded_step_at_world_size_one_is_the_plain_step():
    import torch.distributed as dist

    from newton_schulz_matrix_b200.distributed import ShardedMuonStep

    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.moe_layer(experts=4, device=DEV)   # 8 up/gate, 4 down (transposed), 4 shared 2048^2
        params, grads, moms = [], [], []
        for g in w.groups:
            params += [x.float() for x in g.W]       # fp32 W so that O is observable exactly
            grads += g.G
            moms += g.M
        hp = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, scale_coef=0.2, eps=1e-7, coeffs=Q5)
        W0 = [p.clone() for p in params]
        M0 = [m.clone() for m in moms]
        sharded = ShardedMuonStep(params, grads, {i: m for i, m in enumerate(moms)}, **hp)
        assert sharded.owned() == list(range(len(params)))
        sharded()
        torch.cuda.synchronize()
        assert int(sharded.local.status.abs().sum()) == 0

        Wp = [x.clone() for x in W0]
        Mp = [x.clone() for x in M0]
        nsm.MuonStep(Wp, grads, Mp, **hp)()
        torch.cuda.synchronize()
        for a, b in zip(params + moms, Wp + Mp):
            assert torch.equal(a, b)

        for i in (0, 8, 12):                          # up, down (tall), shared
            r, c = params[i].shape
            Wr, Mr, Or = oracle.muon_step(to_np(W0[i]), to_np(grads[i]), to_np(M0[i]), **hp)
            assert rel(to_np(moms[i]), Mr) < 1e-6
            step = hp["lr"] * hp["scale_coef"] * math.sqrt(max(r, c))
            O = ((1 - hp["lr"] * hp["weight_decay"]) * to_np(W0[i]) - to_np(params[i])) / step
            assert rel(O, Or) < 2e-2
    finally:
        dist.destroy_process_group()
