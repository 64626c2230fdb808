"""Host logic of the multi-rank bench path, as two gloo ranks on CPU: every
rank joins the barrier, and the reported time is the max over ranks."""
import os

import pytest
import torch
import torch.multiprocessing as mp


def _worker(rank, world, store_path, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    # a file rendezvous: no TCP port that another process could take between
    # choosing it and binding it
    torch.distributed.init_process_group("gloo", init_method=f"file://{store_path}", rank=rank,
                                         world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    ms = 10.0 + 5.0 * rank
    out[rank] = bench.max_over_ranks(ms, world, torch.device("cpu"))
    torch.distributed.destroy_process_group()


def test_max_over_ranks_gloo_world2(tmp_path):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    store = str(tmp_path / "rendezvous")
    procs = [ctx.Process(target=_worker, args=(r, 2, store, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert dict(out) == {0: 15.0, 1: 15.0}
