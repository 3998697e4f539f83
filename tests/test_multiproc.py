"""Host logic of the multi-GPU benchmark path, on CPU with gloo, world size 2:
rank/world discovery from the launcher's environment, the barrier, and the
max-over-ranks reduction of the timed region (the layer runs as independent
replicas, so there is no data-path collective to test)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    bench.dist_init(w, "gloo")
    bench.barrier(w)
    # each rank reports a different elapsed time; everyone must get the max
    got = bench.max_over_ranks(10.0 + 5.0 * rank, w, torch.device("cpu"))
    # tokens of all ranks over the slowest rank's time
    value = 1000 * w / (got / 1e3)
    # the CUDA-graph timed region is used only if every rank captured: rank 1
    # reports a failed capture, so both ranks fall back to eager steps
    use_graph = bench.max_over_ranks(0.0 if rank == 0 else 1.0, w, torch.device("cpu")) == 0
    q.put((rank, got, value, use_graph))
    bench.barrier(w)
    torch.distributed.destroy_process_group()


def test_max_over_ranks_and_job_throughput_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [g for _, g, _, _ in res] == [15.0, 15.0]
    assert all(abs(v - 2000 / 0.015) < 1e-6 for _, _, v, _ in res)
    assert [u for _, _, _, u in res] == [False, False]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1)
    assert not torch.distributed.is_initialized()
