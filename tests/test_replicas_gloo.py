"""The multi-GPU path of the bench is N independent replicas (the DSA hot path has
no exchange step on one GPU).  Its host plumbing -- process group, barriers, the
maximum step time over ranks, the whole-job rate and per-replica seeds -- runs
here as two gloo ranks on the CPU."""
import os
import socket

import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from long_context_sparse_fp8_b200 import replicas as R
    r, w, dev = R.setup(timeout_s=30, cpu=True)
    R.barrier(w, dev)
    step_ms = 1.5 + r                      # rank 1 is the slow one
    m = R.max_over_ranks(step_ms, w, dev)
    rate = R.job_throughput(32, m, w)
    seed = R.replica_seed(1234, r)
    R.barrier(w, dev)
    R.teardown(w)
    q.put((r, w, dev.type, m, rate, seed))


def test_two_replicas_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=120) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 and r[2] == "cpu" for r in res)
    # every rank sees the slowest rank's time; the job rate counts both replicas
    assert all(r[3] == 2.5 for r in res)
    assert all(abs(r[4] - 32 * 2 / 2.5e-3) < 1e-6 for r in res)
    assert res[0][5] != res[1][5]


def test_single_process_needs_no_group():
    from long_context_sparse_fp8_b200 import replicas as R
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    r, w, dev = R.setup(cpu=True)
    assert (r, w, dev.type) == (0, 1, "cpu")
    assert R.max_over_ranks(3.0, w, dev) == 3.0
    assert R.job_throughput(32, 2.0, 1) == 16000.0
