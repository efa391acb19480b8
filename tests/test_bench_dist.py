"""The N>1 path of bench.py on CPU: world-size-2 gloo ranks (127.0.0.1).

The kernels are row-independent, so bench.py runs one replica per GPU and uses
torch.distributed only for barriers and the timing reduction: whole-job units are
summed over ranks and the elapsed time is the maximum over ranks. This checks that
reduction, and that every rank takes the same collective steps.
"""
import os
import socket
import time

import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist

    r, w, local = bench.init_dist()
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    units, ms = bench.aggregate(1000.0 * (rank + 1), 10.0 + 5.0 * rank, w)
    bench.barrier(w)
    out[rank] = (units, ms)
    dist.destroy_process_group()


def test_aggregate_sums_units_and_takes_max_time_over_two_ranks():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == (3000.0, 15.0) and out[1] == (3000.0, 15.0)


def test_single_rank_aggregate_is_identity():
    assert bench.aggregate(123.0, 4.5, 1) == (123.0, 4.5)


def _rank_main_failing(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank), BI_PG_TIMEOUT_S="5")
    r, w, _ = bench.init_dist()
    if rank == 1:
        os._exit(0)  # this rank leaves between steps, before the next collective
    t0 = time.time()
    try:
        bench.barrier(w)
        out[rank] = ("no error", time.time() - t0)
    except Exception as e:  # the surviving rank learns of it from its collective
        out[rank] = (type(e).__name__, time.time() - t0)


def test_a_rank_that_leaves_ends_the_others_collective_with_an_error():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_failing, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    kind, seconds = out[0]
    assert kind != "no error" and seconds < 60, (kind, seconds)
