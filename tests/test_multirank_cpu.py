"""Multi-process host logic on CPU with the gloo backend (world size 2-3):
the bench's cross-rank timing reduction and weak-scaling value, and the
sharded step's ownership plan and weight exchange, with injected local
updates in place of the CUDA step: rank-tagged ones that show where each
weight came from, and the fp64 oracle's own Muon step."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from newton_schulz_matrix_b200.distributed import ShardedMuonStep, lpt_owners, ns_cost


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _bench_worker(rank, world, port, q):
    _init(rank, world, port)
    import bench
    ms = bench.max_over_ranks(100.0 + 10 * rank, dist, torch.device("cpu"))
    v = bench.whole_job_tflops(world, 513.2e12, ms)
    q.put((rank, ms, v))
    dist.barrier()
    dist.destroy_process_group()


def _sharded_worker(rank, world, port, q):
    _init(rank, world, port)
    torch.manual_seed(0)  # identical initial weights on every rank
    shapes = [(64, 32), (16, 16), (128, 64), (32, 96), (8, 8), (64, 64), (48, 16)]
    params = [torch.randn(*s) for s in shapes]
    grads = [torch.randn(*s) for s in shapes]
    start = [p.clone() for p in params]
    owner = lpt_owners([ns_cost(s) for s in shapes], world)
    moms = {i: torch.zeros(*shapes[i]) for i in range(len(shapes)) if owner[i] == rank}

    def fake_local(ps, gs, ms, **hp):
        def run():
            for p, g in zip(ps, gs):
                p.add_(g, alpha=1.0 + rank)   # rank-specific, so the broadcast source is visible
        return run

    step = ShardedMuonStep(params, grads, moms, local_step_factory=fake_local, lr=0.02)
    assert step.owned() == [i for i, r in enumerate(owner) if r == rank]
    step()
    ok = all(torch.equal(params[i], start[i] + grads[i] * (1.0 + owner[i])) for i in range(len(shapes)))
    q.put((rank, ok, owner))
    dist.barrier()
    dist.destroy_process_group()


def _idle_rank_worker(rank, world, port, q):
    """Three ranks, two matrices: one rank owns nothing and only receives."""
    _init(rank, world, port)
    torch.manual_seed(1)
    shapes = [(32, 64), (48, 48)]
    params = [torch.randn(*s) for s in shapes]
    grads = [torch.randn(*s) for s in shapes]
    start = [p.clone() for p in params]
    owner = lpt_owners([ns_cost(s) for s in shapes], world)
    moms = {i: torch.zeros(*shapes[i]) for i in range(len(shapes)) if owner[i] == rank}

    def fake_local(ps, gs, ms, **hp):
        def run():
            for p, g in zip(ps, gs):
                p.sub_(g)
        return run

    step = ShardedMuonStep(params, grads, moms, local_step_factory=fake_local)
    step()
    step()  # a second step: the idle rank keeps taking the same collective steps
    ok = all(torch.equal(params[i], (start[i] - grads[i]) - grads[i]) for i in range(len(shapes)))
    q.put((rank, ok, step.owned()))
    dist.barrier()
    dist.destroy_process_group()


def _oracle_step_worker(rank, world, port, q):
    """Each owner runs the method's own update (the fp64 oracle's Muon step on
    its matrices) as the local step; after the exchange every rank must hold
    the full set of updated weights that one process computing every matrix
    gets, and each owner the new momentum of its own matrices."""
    _init(rank, world, port)
    import numpy as np

    import oracle
    import synth
    hp = dict(lr=0.02, momentum=0.95, nesterov=True, weight_decay=0.1, scale_coef=0.2, eps=1e-7,
              coeffs=[oracle.QUINTIC] * 5)
    shapes = [(24, 40), (40, 24), (16, 16), (32, 72), (8, 20)]
    params = [synth.gaussian(r, c, 10 + i).double() for i, (r, c) in enumerate(shapes)]
    grads = [synth.gaussian(r, c, 20 + i).double() for i, (r, c) in enumerate(shapes)]
    moms0 = [synth.gaussian(r, c, 30 + i, std=0.1).double() for i, (r, c) in enumerate(shapes)]
    want = [oracle.muon_step(p.numpy(), g.numpy(), m.numpy(), **hp) for p, g, m in zip(params, grads, moms0)]
    owner = lpt_owners([ns_cost(s) for s in shapes], world)
    moms = {i: moms0[i].clone() for i in range(len(shapes)) if owner[i] == rank}

    def oracle_local(ps, gs, ms, **h):
        def run():
            for p, g, m in zip(ps, gs, ms):
                W, M, _ = oracle.muon_step(p.numpy(), g.numpy(), m.numpy(), **hp)
                p.copy_(torch.from_numpy(W))
                m.copy_(torch.from_numpy(M))
        return run

    step = ShardedMuonStep(params, grads, moms, local_step_factory=oracle_local, **hp)
    step()
    ok_w = all(np.array_equal(params[i].numpy(), want[i][0]) for i in range(len(shapes)))
    ok_m = all(np.array_equal(moms[i].numpy(), want[i][1]) for i in moms)
    q.put((rank, ok_w and ok_m, owner))
    dist.barrier()
    dist.destroy_process_group()


def _spawn(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out)


def test_bench_timing_takes_the_slowest_rank():
    out = _spawn(_bench_worker)
    for rank, ms, v in out:
        assert ms == 110.0
        assert v == pytest.approx(2 * 513.2e12 / 0.110 / 1e12)


def test_sharded_step_exchanges_owned_updates():
    out = _spawn(_sharded_worker)
    assert [ok for _, ok, _ in out] == [True, True]
    assert out[0][2] == out[1][2]  # both ranks computed the same plan


def test_lpt_balances_the_kimi_k2_set():
    shapes = [(2048, 7168)] * 648 + [(7168, 18432)] * 3
    costs = [ns_cost(s) for s in shapes]
    for world in (2, 4, 8):
        owner = lpt_owners(costs, world)
        load = [0.0] * world
        for c, r in zip(costs, owner):
            load[r] += c
        assert max(load) / (sum(load) / world) < 1.02
        assert sorted(set(owner)) == list(range(world))
    assert lpt_owners([5, 5, 5], 1) == [0, 0, 0]
    with pytest.raises(ValueError):
        lpt_owners([1.0], 0)


def test_sharded_step_with_a_rank_that_owns_nothing():
    out = _spawn(_idle_rank_worker, world=3)
    assert [ok for _, ok, _ in out] == [True, True, True]
    owned = [o for _, _, o in out]
    assert sorted(i for o in owned for i in o) == [0, 1]
    assert [] in owned


def test_sharded_step_exchanges_the_methods_updates():
    out = _spawn(_oracle_step_worker)
    assert [ok for _, ok, _ in out] == [True, True]
    assert sorted(set(out[0][2])) == [0, 1]  # both ranks own matrices
