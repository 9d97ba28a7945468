"""Multi-process tests (gloo on CPU, world size 2) of the replica orchestration
that bench.py --gpus N uses: the path has no exchange step, so N GPUs run N
replicas; the ranks line up around the timed region, the slowest rank's time
is taken, and the job's throughput is N replicas' work over that time. A rank
that dies before the barrier must make the others fail within the process
group's timeout instead of hanging."""

import multiprocessing as mp
import os
import socket

import pytest


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def worker(rank, world, port, mode, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from precision_attention_fmha_b200 import replicas

    w, r, _ = replicas.setup("gloo", timeout_s=8)
    if mode == "ok":
        replicas.barrier(w)
        slowest = replicas.max_over_ranks(10.0 + 5.0 * r, w, device="cpu")  # rank r took 10 + 5r ms
        thr = replicas.job_throughput(1000.0, w, slowest)
        replicas.barrier(w)
        q.put((r, slowest, thr))
        replicas.teardown(w)
        return
    # mode == "rank1_dies": rank 1 leaves between steps, before the barrier
    if r == 1:
        os._exit(3)
    try:
        replicas.barrier(w)
        q.put((r, "no error"))
    except Exception as e:  # the barrier must end with an error, not hang
        q.put((r, "error: " + type(e).__name__))
    q.close()
    q.join_thread()  # flush the result before leaving without the group's teardown
    os._exit(0)


def run(world, mode, timeout=60):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank hung"
    out = []
    while not q.empty():
        out.append(q.get())
    return sorted(out, key=lambda t: t[0]), [p.exitcode for p in procs]


def test_two_replicas_take_the_slowest_rank_and_sum_the_work():
    out, codes = run(2, "ok")
    assert codes == [0, 0]
    assert [o[0] for o in out] == [0, 1]
    for _, slowest, thr in out:
        assert slowest == 15.0                      # max over ranks of 10 and 15 ms
        assert thr == pytest.approx(2 * 1000.0 / 15e-3)  # both replicas' work over the slowest time


def test_a_rank_that_dies_makes_the_other_fail_not_hang():
    out, codes = run(2, "rank1_dies")
    assert codes[1] == 3
    assert len(out) == 1 and out[0][0] == 0 and out[0][1].startswith("error")


def test_single_process_needs_no_group(monkeypatch):
    from precision_attention_fmha_b200 import replicas

    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert replicas.setup("gloo") == (1, 0, 0)
    assert replicas.max_over_ranks(3.5, 1) == 3.5
    assert replicas.job_throughput(100.0, 1, 10.0) == pytest.approx(1e4)
    replicas.barrier(1)
    replicas.teardown(1)
