"""The multi-GPU benchmark path (independent replicas, one per rank) on CPU:
two gloo ranks aggregate their timings the way `bench.py --gpus N` does --
max over ranks of the device time, sum over ranks of the bytes streamed."""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    local_ms = [10.0, 12.5][rank]          # rank 1 is the slow one
    local_bytes = 7.0e9                     # bytes each replica streams over the timed steps
    ms, nbytes, gbs = bench.replica_throughput(dist, "cpu", local_ms, local_bytes, steps=5)
    out[rank] = (ms, nbytes, gbs)
    dist.barrier()
    dist.destroy_process_group()


def test_two_replicas_aggregate_max_time_and_total_bytes():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    for rank in (0, 1):
        ms, nbytes, gbs = out[rank]
        assert ms == 12.5
        assert nbytes == 14.0e9
        assert abs(gbs - 14.0e9 / (12.5 / 5 * 1e-3) / 1e9) < 1e-9


def test_single_process_is_identity():
    import bench
    ms, nbytes, gbs = bench.replica_throughput(None, "cpu", 4.0, 2.0e9, steps=2)
    assert (ms, nbytes) == (4.0, 2.0e9) and abs(gbs - 1000.0) < 1e-9
