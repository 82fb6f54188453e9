"""Replica-parallel host logic on 2 gloo ranks (CPU): per-rank seeds, the
max-over-ranks timing reduction and the whole-job throughput, plus a rank
that fails between steps being seen by the other through a short timeout."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from paged_kv_cache_321_b200 import replicas
    from workloads import SPECS, make_workload

    r, w, lr = replicas.world_from_env()
    dist = replicas.init("gloo", timeout_s=30)
    spec = SPECS["tiny"]
    wl = make_workload(spec, seed_offset=replicas.replica_seed_offset(spec.seed_offset, r))
    times = [1.0 + r, 5.0 - r]  # rank 0: (1, 5), rank 1: (2, 4)
    mx = replicas.max_over_ranks(times, dist)
    thr = replicas.job_throughput(100.0, w, mx[0])
    q.put((r, w, float(wl.q[0, 0]), mx, thr))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, q0, mx0, thr0), (r1, w1, q1, mx1, thr1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert q0 != q1  # independent replicas draw different requests
    assert mx0 == mx1 == [2.0, 5.0]  # element-wise max over ranks
    assert thr0 == thr1 == pytest.approx(100.0 * 2 / 2.0)


def _failing_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    from paged_kv_cache_321_b200 import replicas

    dist = replicas.init("gloo", timeout_s=5)
    dist.barrier()
    if rank == 1:
        os._exit(3)  # leaves between steps, with nothing in flight
    try:
        replicas.max_over_ranks([1.0], dist)
        q.put((rank, "no error"))
    except Exception as e:  # the survivor's next collective ends with an error
        q.put((rank, type(e).__name__))


def test_rank_leaving_between_steps_is_detected():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    rank, what = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert rank == 0 and what != "no error"
    assert procs[1].exitcode == 3
