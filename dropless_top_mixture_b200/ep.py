"""Expert parallelism of the MoE layer across GPUs of one node.

"olmoforge" README, capability table: row-wise expert parallelism writes each
token row straight into its expert's input buffer on whichever GPU holds
the expert; "专家池 8→128 只慢 5%…" (Olmo-core 3, 关键数字): the experts are
spread over the GPUs. Rank r of a group of G owns experts r*El .. (r+1)*El-1
(El = E / G) and their weights. One forward step:

  1. moe_route on the rank's own tokens (all E experts);
  2. exchange_counts: every rank's per-expert counts gathered into
     counts_all [G, E] (one all-gather);
  3. moe_ep_plan: each (token, choice)'s owner and row in the owner's
     expert-major receive buffer, and this rank's receive offsets;
  4. moe_dispatch_ep: the rows written straight into the owners' receive
     buffers (peer stores over NVLink, no all-to-all buffer in between);
  5. the owner's grouped SwiGLU GEMMs on its receive buffer;
  6. moe_combine_ep: each token's k outputs gathered back from the owners
     (peer loads) and summed with their gates.

The ranks order the steps with group barriers: a receive buffer is complete
when every rank's dispatch has finished, and an output buffer is readable
when its owner's GEMMs have. The peers' buffers are mapped into each process
with CUDA IPC handles; every launch is one of this library's kernels.
"""
from __future__ import annotations

from typing import List, Optional

import torch
import torch.distributed as dist

from . import moe


def exchange_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """All ranks' per-expert counts [E] gathered into [G, E] (row s = rank
    s's), in rank order, on the device of ``counts``."""
    G = dist.get_world_size(group)
    parts = [torch.empty_like(counts) for _ in range(G)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts)


def owned_experts(E: int, G: int, rank: int) -> range:
    """The experts rank ``rank`` of ``G`` holds (a contiguous block)."""
    if E % G:
        raise ValueError(f"{E} experts do not split evenly over {G} ranks")
    el = E // G
    return range(rank * el, (rank + 1) * el)


def receive_rows_max(T_max: int, k: int, G: int) -> int:
    """Rows a receive buffer must hold in the worst case: every rank's tokens
    all routed to this rank's experts (dropless: nothing is cut)."""
    return G * T_max * k


def _ipc_table(buf: torch.Tensor, group) -> List[int]:
    """Device addresses, in this process, of every rank's buffer ``buf``
    (this rank's own address for its own)."""
    from cuda.bindings import runtime as rt

    err, handle = rt.cudaIpcGetMemHandle(buf.data_ptr())
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaIpcGetMemHandle: {err}")
    blobs = [None] * dist.get_world_size(group)
    dist.all_gather_object(blobs, bytes(handle.reserved), group=group)
    me = dist.get_rank(group)
    addrs = []
    for r, blob in enumerate(blobs):
        if r == me:
            addrs.append(buf.data_ptr())
            continue
        h = rt.cudaIpcMemHandle_t()
        h.reserved = blob
        err, ptr = rt.cudaIpcOpenMemHandle(h, rt.cudaIpcMemLazyEnablePeerAccess)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaIpcOpenMemHandle (rank {r}): {err}")
        addrs.append(int(ptr))
    return addrs


class ExpertParallelLayer:
    """The layer forward with experts partitioned over the ranks of
    ``group`` (one GPU per rank). ``W1``, ``W3`` [El, F, d] and ``W2``
    [El, d, F] are this rank's experts; ``T_max`` bounds any rank's tokens
    per call."""

    def __init__(self, E: int, k: int, W1: torch.Tensor, W3: torch.Tensor, W2: torch.Tensor,
                 T_max: int, group=None):
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.E, self.k = E, k
        self.experts = owned_experts(E, self.G, self.rank)
        if W1.shape[0] != len(self.experts):
            raise ValueError("W1 must hold exactly this rank's experts")
        self.W1, self.W3, self.W2 = W1, W3, W2
        self.F, self.d = W1.shape[1], W1.shape[2]
        self.dev = W1.device
        self.rows_max = receive_rows_max(T_max, k, self.G)
        self.recv = torch.empty((self.rows_max, self.d), dtype=W1.dtype, device=self.dev)
        self.ye = torch.empty((self.rows_max, self.d), dtype=W1.dtype, device=self.dev)
        self.H = torch.empty((self.rows_max, self.F), dtype=W1.dtype, device=self.dev)
        self.recv_table = torch.tensor(_ipc_table(self.recv, group), dtype=torch.int64,
                                       device=self.dev)
        self.ye_table = torch.tensor(_ipc_table(self.ye, group), dtype=torch.int64,
                                     device=self.dev)

    def forward(self, x: torch.Tensor, logits: Optional[torch.Tensor] = None,
                Wr: Optional[torch.Tensor] = None) -> torch.Tensor:
        rt = moe.moe_route(self.k, logits=logits, x=None if logits is not None else x,
                           Wr=Wr)
        counts_all = exchange_counts(rt.counts, self.group)
        plan = moe.moe_ep_plan(counts_all, self.rank, rt)
        dist.barrier(group=self.group)        # receive buffers free to be written
        moe.moe_dispatch_ep(x, plan, self.recv_table, self.rows_max)
        dist.barrier(group=self.group)        # every rank's rows have landed
        rows = int(plan.recv_offsets[-1].item())
        if rows:
            moe.moe_grouped_swiglu(self.recv[:rows], self.W1, self.W3, self.W2,
                                   plan.recv_offsets, H=self.H[:rows], Ye=self.ye[:rows])
        dist.barrier(group=self.group)        # every owner's outputs are written
        out = moe.moe_combine_ep(self.ye_table, plan, rt.gate, self.d, x.dtype, self.rows_max)
        dist.barrier(group=self.group)        # nobody still reads this rank's outputs
        return out


__all__ = ["exchange_counts", "owned_experts", "receive_rows_max", "ExpertParallelLayer"]
