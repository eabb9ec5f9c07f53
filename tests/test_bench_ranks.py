"""The multi-rank logic of bench.py (one process per GPU under torchrun) on CPU: two gloo
ranks with different timings must both see the slowest rank's time, and the whole-job
rate counts every rank's units over that time."""
import os
import socket
import tempfile

import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = [12.5, 20.25, 7.0][rank]
    slowest = bench.max_over_ranks(ms, world, "cpu")
    e2e = bench.max_over_ranks(ms / 1000.0 + rank, world, "cpu")
    rate = bench.whole_job_rate(1000, 4, world, slowest / 1e3)
    with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
        f.write(f"{slowest!r} {e2e!r} {rate!r}")
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_rate_on_gloo():
    for world in (2, 3):
        with tempfile.TemporaryDirectory() as d:
            mp.start_processes(_rank_main, args=(world, _free_port(), d), nprocs=world,
                               join=True, start_method="spawn")
            got = [open(os.path.join(d, f"r{r}.txt")).read().split() for r in range(world)]
        want_ms = max([12.5, 20.25, 7.0][:world])
        for slowest, e2e, rate in got:
            assert float(slowest) == want_ms
            assert float(e2e) == max(ms / 1000.0 + r for r, ms in enumerate([12.5, 20.25, 7.0][:world]))
            assert float(rate) == 1000 * 4 * world / (want_ms / 1e3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_rate(10, 2, 1, 0.5) == 40.0
