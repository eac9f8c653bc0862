"""Multi-replica host logic of bench.py on CPU: two gloo ranks (world size 2).

The attention path has no exchange step, so N GPUs run N independent replicas; the
process group only provides the barrier and the max-over-ranks timing.  These tests run
that logic with the gloo backend in spawned processes, and check that a rank which
leaves before a barrier surfaces as an error on the other rank instead of a hang.
"""
import os
import socket
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)


def _replica(rank, world, port, q):
    _env(rank, world, port)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo", timeout_s=30)
    bench.barrier(w)
    local_ms = 10.0 + 5.0 * r               # rank 1 is the slower replica
    job_ms = bench.max_over_ranks(local_ms, w)
    value = bench.whole_job_tflops(1e12, 4, w, job_ms)
    q.put((r, w, job_ms, value))
    dist.destroy_process_group()


def _leaver(rank, world, port, q):
    _env(rank, world, port)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world, backend="gloo", timeout_s=5)
    bench.barrier(w)
    if r == 1:
        os._exit(0)                          # leaves between steps, before the next barrier
    t0 = time.time()
    try:
        bench.barrier(w)
        bench.max_over_ranks(1.0, w)
        q.put(("no error", time.time() - t0))
    except Exception as e:                   # noqa: BLE001 - any error ends the wait
        q.put((type(e).__name__, time.time() - t0))
    try:
        dist.destroy_process_group()
    except Exception:                        # noqa: BLE001
        pass


def _spawn(fn, world, timeout):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = []
    deadline = time.time() + timeout
    for p in procs:
        p.join(max(1.0, deadline - time.time()))
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    while not q.empty():
        out.append(q.get())
    return out, [p.exitcode for p in procs]


def test_two_replicas_max_time_and_whole_job_value():
    out, codes = _spawn(_replica, 2, timeout=120)
    assert codes == [0, 0], codes
    assert sorted(o[0] for o in out) == [0, 1]
    for r, w, job_ms, value in out:
        assert w == 2
        assert job_ms == 15.0                # the slower replica's time, on every rank
        # two replicas x 4 steps x 1 TFLOP each, in 15 ms
        assert value == pytest.approx(2 * 4 * 1.0 / 15e-3)


def test_rank_that_leaves_is_an_error_not_a_hang():
    out, codes = _spawn(_leaver, 2, timeout=120)
    assert codes[1] == 0
    assert len(out) == 1, out
    what, waited = out[0]
    assert what != "no error"
    assert waited < 60.0
