"""Host logic of the multi-process bench on CPU: two ranks over gloo (127.0.0.1).

Each rank of `bench.py --gpus N` processes its own replica of the workload (the (batch, head)
slices are independent, so there is no data-path collective); the only collectives are the
barriers around the timed region and the max over ranks of the elapsed time.
"""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world, backend="gloo")
    d.barrier()
    elapsed = 2.0 + 3.0 * rank          # rank 1 is the slow one
    worst = d.max(elapsed)
    d.barrier()
    d.close()
    out.put((rank, d.world, worst))


def test_two_ranks_take_the_max_elapsed_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 2, 5.0), (1, 2, 5.0)]
