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


def _ep_worker(rank, world, port, E, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    from dropless_top_mixture_b200 import ep
    g = torch.Generator().manual_seed(100 + rank)
    counts = torch.randint(0, 50, (E,), generator=g, dtype=torch.int32)
    allc = ep.exchange_counts(counts)
    mine = list(ep.owned_experts(E, world, rank))
    q.put((rank, allc.numpy().tolist(), mine, ep.receive_rows_max(300, 4, world)))
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


def test_expert_parallel_count_exchange_world3():
    """Expert parallelism's host side over gloo: every rank receives every
    rank's per-expert counts in rank order, the experts split into
    contiguous blocks, and receive buffers are sized for every token of every
    rank landing on one rank."""
    E, world = 12, 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ep_worker, args=(r, world, port, E, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    expect = [torch.randint(0, 50, (E,), generator=torch.Generator().manual_seed(100 + r),
                            dtype=torch.int32).tolist() for r in range(world)]
    for rank, allc, mine, rows_max in res:
        assert allc == expect
        assert mine == list(range(rank * 4, rank * 4 + 4))
        assert rows_max == 3 * 300 * 4


def test_expert_parallel_split_and_sizing():
    """The expert split is contiguous and covers every expert once; an
    expert count that does not divide over the ranks is refused; receive
    buffers hold the dropless worst case (every token of every rank)."""
    from dropless_top_mixture_b200 import ep
    for E, G in ((64, 8), (12, 3), (7, 1), (128, 4)):
        seen = []
        for r in range(G):
            blk = list(ep.owned_experts(E, G, r))
            assert blk == list(range(r * E // G, (r + 1) * E // G))
            seen += blk
        assert seen == list(range(E))
    with pytest.raises(ValueError):
        ep.owned_experts(10, 4, 0)
    assert ep.receive_rows_max(T_max=300, k=4, G=3) == 3 * 300 * 4
