"""Expert parallelism: the exchange plumbing of latent_mixture_experts_top_b200.ep
with world-size-2 gloo ranks on CPU.

The library's phases need a GPU, so here each rank's phases are played by the
fp64 oracle (dispatch: router, top-K', dispatch order and z rows; experts:
the rank's own experts, row by row, in the received layout; combine: slot-order
combine, W_up, shared experts).  What runs for real is ep.forward -- the
count exchange, the split sizes and the two row all-to-alls -- and the layout
contract between the three phases.  Each rank's y must equal the oracle's
single-process forward of the same tokens ("Shaping Latent MoE", Figure 6:
experts split across devices, tokens exchanged at width l).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle

D, ALPHA, M, N, K, NS, MS = 64, 2, 32, 8, 3, 1, 32


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _layer(seed=0):
    rng = np.random.default_rng(seed)
    l = D // ALPHA
    w = lambda *shape: rng.normal(0.0, 0.2, size=shape)
    return oracle.Layer(w_router=w(N, D), b_router=None, w_down=w(l, D), w_up=w(D, l),
                        w_gate=w(N, M, l), w_upx=w(N, M, l), w_out=w(N, l, M),
                        s_gate=w(NS, MS, D), s_up=w(NS, MS, D), s_out=w(NS, D, MS), k_active=K)


def _tokens(rank):
    rng = np.random.default_rng(100 + rank)
    return rng.normal(0.0, 1.0, size=(20 if rank == 0 else 13, D))


class OracleBackend:
    """The three phases of one rank, computed by the oracle, with the
    library's layouts: send rows in dispatch order (experts ascending, tokens
    ascending), received rows source-major and expert-grouped, returned rows
    in send order."""

    def __init__(self, L, rank, world):
        self.L, self.rank, self.world = L, rank, world
        self.nl = N // world

    def dispatch(self, x):
        L = self.L
        x = x.numpy()
        s = oracle.router_logits(L, x)
        ids, self.g = oracle.select(s, K)
        off, perm, self.pos = oracle.dispatch(ids, N)
        z = np.stack([oracle.down(L, x, t) for t in range(x.shape[0])])
        self.x = x
        send = torch.from_numpy(np.ascontiguousarray(z[perm // K]))
        return send, torch.from_numpy(np.diff(off).astype(np.int32))

    def experts(self, recv, recv_counts):
        rc = recv_counts.numpy()
        assert rc.shape == (self.world, self.nl) and rc.sum() == recv.shape[0]
        out = np.empty(tuple(recv.shape))
        i = 0
        for s in range(self.world):
            for e in range(self.nl):
                for _ in range(rc[s, e]):
                    out[i] = oracle.expert(self.L, self.rank * self.nl + e, recv[i].numpy())
                    i += 1
        return torch.from_numpy(out)

    def combine(self, back, T):
        b = back.numpy()
        y = np.empty((T, D))
        for t in range(T):
            u = sum(self.g[t, k] * b[self.pos[t * K + k]] for k in range(K))
            y[t] = oracle.up(self.L, u) + oracle.shared(self.L, self.x, t)
        return torch.from_numpy(y)


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    from latent_mixture_experts_top_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        L = _layer()
        x = torch.from_numpy(_tokens(rank))
        y = ep.forward(OracleBackend(L, rank, world), x, world)
        y_ref, _, _ = oracle.forward(L, x.numpy())
        out.put((rank, float(np.abs(y.numpy() - y_ref).max() / np.abs(y_ref).max())))
    finally:
        dist.destroy_process_group()


def test_expert_parallel_exchange_two_ranks_matches_single_process_oracle():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(out.get(timeout=5) for _ in range(world))
    assert set(res) == {0, 1}
    for r, err in res.items():
        assert err < 1e-12, (r, err)


def test_emulated_exchange_matches_the_collective_layout():
    """ep.forward_emulated (the single-process copy of the exchange the GPU
    test uses) against the oracle, with two ranks of different token counts."""
    from latent_mixture_experts_top_b200 import ep
    L = _layer(1)
    world = 2
    xs = [torch.from_numpy(_tokens(r)) for r in range(world)]
    ys = ep.forward_emulated([OracleBackend(L, r, world) for r in range(world)], xs)
    for x, y in zip(xs, ys):
        y_ref, _, _ = oracle.forward(L, x.numpy())
        assert np.abs(y.numpy() - y_ref).max() / np.abs(y_ref).max() < 1e-12


def test_split_sizes():
    from latent_mixture_experts_top_b200 import ep
    c = torch.tensor([[1, 2, 0], [4, 0, 0]], dtype=torch.int32)
    assert ep.split_sizes(c) == [3, 4]
