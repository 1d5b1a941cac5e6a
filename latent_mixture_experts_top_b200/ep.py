"""Expert-parallel forward of the LatentMoE layer over several ranks.

"Shaping Latent MoE", Figure 6: the routed experts sit inside W_down / W_up,
so under expert parallelism every token crosses to the ranks that own its
experts, and back, in the latent width l rather than d; "LatentMoE
Explained", Figure 12 and its discussion of the all-to-all that runs twice
per expert layer.  Each rank owns a contiguous slice of the N' experts
(LatentMoELayer(..., ep_rank=r, ep_world=W)); router, projections and shared
experts are replicated.  One forward per rank:

    dispatch (library)   x -> z rows in dispatch order + rows per expert
    exchange             counts, then rows, to the ranks owning the experts
    experts (library)    received rows -> expert outputs, same order
    exchange back        outputs return in the order they were sent
    combine (library)    gate-weighted combine, W_up, shared experts -> y

Every computation runs in the library's kernels; this module only moves the
buffers between ranks (torch.distributed all-to-alls: NCCL between GPUs,
gloo in the CPU tests) and keeps the split bookkeeping.  ``backend`` is
anything with the three phase methods; CudaBackend is the library's.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class CudaBackend:
    """The library's three phases for one expert-parallel rank."""

    def __init__(self, layer):
        assert layer.ep_world > 1, "an expert-parallel handle (ep_world > 1)"
        self.layer = layer
        self.world = layer.ep_world

    def dispatch(self, x: torch.Tensor):
        from . import lmoe
        T = x.shape[0]
        L = self.layer
        send = torch.empty((T * L.k_active, L.l), dtype=torch.bfloat16, device=x.device)
        counts = torch.empty((L.n_routed,), dtype=torch.int32, device=x.device)
        lmoe.lmoe_ep_dispatch(L.handle, x, T, send, counts)
        return send, counts

    def experts(self, recv: torch.Tensor, recv_counts: torch.Tensor) -> torch.Tensor:
        from . import lmoe
        out = torch.empty_like(recv)
        lmoe.lmoe_ep_experts(self.layer.handle, recv, recv_counts.contiguous(), recv.shape[0], out)
        return out

    def combine(self, back: torch.Tensor, T: int) -> torch.Tensor:
        from . import lmoe
        y = torch.empty((T, self.layer.cfg.d), dtype=torch.bfloat16, device=back.device)
        lmoe.lmoe_ep_combine(self.layer.handle, back, y, T)
        return y


def split_sizes(counts_by_rank: torch.Tensor) -> list[int]:
    """Rows per rank from a [W][N'/W] count matrix (a host sync)."""
    return [int(v) for v in counts_by_rank.sum(dim=1).tolist()]


def forward(backend, x: torch.Tensor, world: int, group=None) -> torch.Tensor:
    """One expert-parallel forward of this rank's tokens x; every rank of
    ``group`` (world ranks) calls it with its own x, in the same order."""
    send, counts = backend.dispatch(x)
    n_local = counts.numel() // world
    counts2 = counts.view(world, n_local)
    # row q of this rank's counts goes to rank q: afterwards recv_counts[s] is
    # what source s sends for each of this rank's experts
    recv_counts = torch.empty_like(counts2)
    dist.all_to_all_single(recv_counts, counts2, group=group)
    send_split, recv_split = split_sizes(counts2), split_sizes(recv_counts)
    recv = send.new_empty((sum(recv_split), send.shape[1]))
    dist.all_to_all_single(recv, send[:sum(send_split)], recv_split, send_split, group=group)
    out = backend.experts(recv, recv_counts)
    back = send.new_empty((sum(send_split), send.shape[1]))
    dist.all_to_all_single(back, out, send_split, recv_split, group=group)
    return backend.combine(back, x.shape[0])


def forward_emulated(backends, xs):
    """All ranks' forwards in one process, the two exchanges done by copies
    (no collective, no kernel waits on another): backends[r] and xs[r] are
    rank r's.  The same phases and layouts as forward()."""
    world = len(backends)
    sends, counts = zip(*[b.dispatch(x) for b, x in zip(backends, xs)])
    n_local = counts[0].numel() // world
    counts2 = [c.view(world, n_local) for c in counts]
    sizes = [split_sizes(c) for c in counts2]           # sizes[s][q]: rows s -> q
    starts = [[sum(sz[:q]) for q in range(world)] for sz in sizes]
    outs = []
    for q in range(world):
        recv = torch.cat([sends[s][starts[s][q]:starts[s][q] + sizes[s][q]] for s in range(world)])
        recv_counts = torch.stack([counts2[s][q] for s in range(world)])
        outs.append(backends[q].experts(recv, recv_counts))
    ys = []
    for s in range(world):
        parts = []
        for q in range(world):
            before = sum(sizes[p][q] for p in range(s))   # source s's block within rank q's rows
            parts.append(outs[q][before:before + sizes[s][q]])
        back = torch.cat(parts)
        ys.append(backends[s].combine(back, xs[s].shape[0]))
    return ys
