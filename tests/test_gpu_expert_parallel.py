"""Expert parallelism's device path, with G ranks emulated on one GPU.

Each emulated rank routes its own tokens; the counts of all ranks form
counts_all; every rank's plan, dispatch into the owners' receive buffers,
the owners' grouped GEMMs and every rank's combine run as they would on G
GPUs, except that the G buffer sets live on one device and the ranks run one
after another (no kernel waits on another rank's). The plan is checked row
by row against a host restatement of the receive layout, the receive
buffers bitwise against x, and every rank's output against the oracle
layer on that rank's tokens."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from dropless_top_mixture_b200.workloads import adversarial_logits
from tests._util import assert_close_layer, np64

pytestmark = pytest.mark.gpu


def _moe():
    from dropless_top_mixture_b200 import moe
    return moe


def _expected_rows(counts_all, idx_s, slot_s, offsets_s, me, El):
    """Owner and row of each of rank me's (t, j): the owner's buffer is
    expert-major, senders in rank order within an expert."""
    G, E = counts_all.shape
    tot = counts_all.sum(axis=0)
    rank = idx_s // El
    row = np.empty_like(idx_s)
    for (t, j), e in np.ndenumerate(idx_s):
        r = e // El
        below_experts = tot[r * El:e].sum()
        below_senders = counts_all[:me, e].sum()
        row[t, j] = below_experts + below_senders + (slot_s[t, j] - offsets_s[e])
    return rank, row


@pytest.mark.parametrize("G,E,k,T,dtype", [(4, 16, 4, [300, 257, 1, 500], torch.bfloat16),
                                           (2, 8, 2, [129, 64], torch.float32),
                                           (8, 64, 8, [64] * 8, torch.bfloat16)])
def test_expert_parallel_emulated(G, E, k, T, dtype):
    moe = _moe()
    d, F = 256, 256
    El = E // G
    dev = "cuda"
    g = torch.Generator().manual_seed(G * 100 + E)
    W1 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(dtype)
    W3 = (torch.randn(E, F, d, generator=g) * d ** -0.5).to(dtype)
    W2 = (torch.randn(E, d, F, generator=g) * F ** -0.5).to(dtype)
    xs = [torch.randn(t, d, generator=g).to(dtype) for t in T]
    lgs = [adversarial_logits(t, E, "normal", seed=s + 7).numpy() for s, t in enumerate(T)]
    lgs[0][:, 1] -= 50.0  # expert 1 gets nothing from rank 0
    routes = [moe.moe_route(k, logits=torch.from_numpy(lg).to(dev)) for lg in lgs]
    counts_all = torch.stack([r.counts for r in routes])
    rows_max = G * max(T) * k
    recv = [torch.full((rows_max, d), float("nan"), dtype=dtype, device=dev) for _ in range(G)]
    ye = [torch.full((rows_max, d), float("nan"), dtype=dtype, device=dev) for _ in range(G)]
    recv_table = torch.tensor([b.data_ptr() for b in recv], dtype=torch.int64, device=dev)
    ye_table = torch.tensor([b.data_ptr() for b in ye], dtype=torch.int64, device=dev)
    plans = [moe.moe_ep_plan(counts_all, s, routes[s]) for s in range(G)]
    ca = counts_all.cpu().numpy().astype(np.int64)
    for s in range(G):
        rk, rw = _expected_rows(ca, routes[s].idx.cpu().numpy(), routes[s].slot.cpu().numpy(),
                                routes[s].offsets.cpu().numpy(), s, El)
        assert np.array_equal(plans[s].dst_rank.cpu().numpy(), rk)
        assert np.array_equal(plans[s].dst_row.cpu().numpy(), rw)
        tot = ca.sum(axis=0)[s * El:(s + 1) * El]
        assert np.array_equal(plans[s].recv_offsets.cpu().numpy(),
                              np.concatenate([[0], np.cumsum(tot)]))
    for s in range(G):
        moe.moe_dispatch_ep(xs[s].to(dev), plans[s], recv_table, rows_max)
    torch.cuda.synchronize()
    # every received row is the sender's token row, bit for bit
    for s in range(G):
        rk = plans[s].dst_rank.cpu().numpy()
        rw = plans[s].dst_row.cpu().numpy()
        for (t, j), r in np.ndenumerate(rk):
            assert torch.equal(recv[r][rw[t, j]].cpu(), xs[s][t])
    for r in range(G):
        rows = int(plans[r].recv_offsets[-1].item())
        if rows:
            moe.moe_grouped_swiglu(recv[r][:rows], W1[r * El:(r + 1) * El].to(dev),
                                   W3[r * El:(r + 1) * El].to(dev), W2[r * El:(r + 1) * El].to(dev),
                                   plans[r].recv_offsets, Ye=ye[r][:rows])
    outs = [moe.moe_combine_ep(ye_table, plans[s], routes[s].gate, d, dtype, rows_max)
            for s in range(G)]
    torch.cuda.synchronize()
    assert moe.moe_get_status() == 0
    for s in range(G):
        ref = O.moe_layer(xs[s], k, W1, W3, W2, logits=lgs[s])
        assert np.array_equal(routes[s].idx.cpu().numpy(), ref["idx"])
        assert_close_layer(np64(outs[s]), ref["out"], f"rank {s}")


def test_expert_parallel_bad_row_is_flagged_not_written():
    moe = _moe()
    d, k, G = 64, 2, 2
    x = torch.randn(3, d, device="cuda").to(torch.bfloat16)
    plan = moe.EPPlan(dst_rank=torch.tensor([[0, 1], [1, 5], [0, 0]], dtype=torch.int32, device="cuda"),
                      dst_row=torch.tensor([[0, 1], [2, 0], [99, 3]], dtype=torch.int32, device="cuda"),
                      recv_offsets=torch.zeros(2, dtype=torch.int32, device="cuda"))
    bufs = [torch.zeros(8, d, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    table = torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device="cuda")
    moe.moe_dispatch_ep(x, plan, table, 8)
    torch.cuda.synchronize()
    st = moe.moe_get_status(clear=True)
    assert st & moe.MOE_DEVERR_BAD_INDEX  # rank 5 and row 99 are out of range
    assert torch.equal(bufs[0][0], x[0]) and torch.equal(bufs[1][1], x[0])
    assert torch.equal(bufs[1][2], x[1]) and torch.equal(bufs[0][3], x[2])
    assert moe.moe_get_status() == 0
