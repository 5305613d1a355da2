"""The N>1 reduction of bench.py (max of times, sum of work over ranks),
exercised with two gloo ranks on the CPU."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    res = bench.aggregate({"time_s": 1.0 + rank, "work": 10.0 * (rank + 1)}, world)
    out[rank] = (res["time_s"], res["work"])
    dist.destroy_process_group()


def test_aggregate_two_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == (2.0, 30.0) and out[1] == (2.0, 30.0)


def test_aggregate_single_rank_is_identity():
    import bench
    assert bench.aggregate({"time_s": 3.0, "work": 7.0}, 1) == {"time_s": 3.0, "work": 7.0}
