"""The allocation-free dispatch (lmoe_dispatch_noalloc) against lmoe_route.

lmoe_dispatch_noalloc serves callers that may not call cudaMalloc where they
need the dispatch (for example a serving loop whose device memory is all
reserved by its own pool allocator, or a plugin whose host framework forbids
allocation in its execute callback).  Its scratch is a fixed file-scope device
array shared by every call, so the GPU test makes two calls in a row, of
different sizes, and checks each against the handle-based entry point.  This
file is named to be collected last.
"""
import ctypes as C

import pytest
import torch

from latent_mixture_experts_top_b200 import configs, synth


def _lib():
    from latent_mixture_experts_top_b200 import lmoe
    return lmoe


@pytest.mark.gpu
def test_dispatch_noalloc_matches_route_on_two_calls_in_a_row():
    lm = _lib()
    cfg = configs.README_ACC
    inp = synth.make_inputs(cfg, 0, "cuda")
    layer = lm.LatentMoELayer(cfg, inp)
    N, K = layer.n_routed, layer.k_active
    x = inp["x"]
    for T, start in ((cfg.T, 0), (1000, 1234)):      # second call smaller: stale scratch must not leak
        xs = x[start:start + T].contiguous()
        ids, _, offsets_ref, perm_ref = layer.route(xs)
        offsets = torch.full((N + 1,), -7, dtype=torch.int32, device="cuda")
        perm = torch.full((T * K,), -7, dtype=torch.int32, device="cuda")
        lm.lmoe_dispatch_noalloc(ids, T, K, N, offsets, perm)
        torch.cuda.synchronize()
        assert torch.equal(offsets, offsets_ref)
        assert torch.equal(perm, perm_ref)
    layer.close()


def test_dispatch_noalloc_rejects_sizes_beyond_its_scratch():
    """Host-side checks, before any CUDA call (no GPU needed)."""
    from latent_mixture_experts_top_b200 import build
    lib = C.CDLL(build.build())
    f = lib.lmoe_dispatch_noalloc
    f.argtypes = [C.c_void_p, C.c_int32, C.c_int32, C.c_int32, C.c_void_p, C.c_void_p,
                  C.c_void_p]
    dummy = C.c_void_p(16)   # never dereferenced: every call below is rejected first
    assert f(dummy, 65537, 1, 8, dummy, dummy, None) == -4        # T over the limit
    assert f(dummy, 65536, 5, 8, dummy, dummy, None) == -4        # T*K' over the limit
    assert f(dummy, 16, 2, 1025, dummy, dummy, None) == -7        # N' over the limit
    assert f(dummy, 16, 0, 8, dummy, dummy, None) == -1           # K' < 1
    assert f(dummy, 16, 9, 8, dummy, dummy, None) == -1           # K' > N'
    assert f(dummy, 16, 2, 8, None, dummy, None) == -2            # offsets NULL
    assert f(None, 16, 2, 8, dummy, dummy, None) == -2            # ids NULL with T > 0


@pytest.mark.gpu
def test_dispatch_noalloc_at_its_limits_n1024():
    """N' = 1024 experts and T*K' = LMOE_NOALLOC_MAX_PAIRS: the largest sizes
    the fixed scratch serves (here the scatter kernel needs more than 48 KB of
    shared memory).  Random distinct in-range ids per row; offsets and perm
    must equal the oracle's dispatch bit for bit."""
    import numpy as np
    import oracle
    lm = _lib()
    T, K, N = 16384, 16, 1024
    assert T * K == 262144
    g = torch.Generator(device="cuda").manual_seed(11)
    ids = torch.rand(T, N, device="cuda", generator=g).argsort(dim=1)[:, :K].to(torch.int32)
    ids = ids.contiguous()
    offsets = torch.full((N + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((T * K,), -7, dtype=torch.int32, device="cuda")
    lm.lmoe_dispatch_noalloc(ids, T, K, N, offsets, perm)
    torch.cuda.synchronize()
    off_ref, perm_ref, _ = oracle.dispatch(ids.cpu().numpy(), N)
    np.testing.assert_array_equal(offsets.cpu().numpy(), off_ref)
    np.testing.assert_array_equal(perm.cpu().numpy(), perm_ref)


@pytest.mark.gpu
def test_dispatch_noalloc_skips_out_of_range_ids():
    """Caller-given ids outside [0, N') are skipped, not used as indices: they
    are not counted in offsets, perm from offsets[N'] on holds -1, and every
    in-range pair is placed as the dispatch places it.  A row naming one
    expert twice places both pairs at one position; one position of that
    expert's range is left at -1."""
    import numpy as np
    lm = _lib()
    T, K, N = 300, 4, 16
    rng = np.random.default_rng(5)
    ids = np.stack([rng.choice(N, size=K, replace=False) for _ in range(T)]).astype(np.int32)
    ids[5, 2] = -1
    ids[17, 0] = N
    ids[200, 3] = 1 << 30
    ids[299, 1] = -(1 << 30)

    def expected(ids_np):
        flat = np.arange(T * K)
        e = ids_np.reshape(-1)
        v = (e >= 0) & (e < N)
        cnt = np.bincount(e[v], minlength=N)
        off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
        order = np.lexsort((flat[v], e[v]))
        perm = np.full(T * K, -1, dtype=np.int32)
        perm[:v.sum()] = flat[v][order]
        return off, perm

    def run(ids_np):
        d_ids = torch.from_numpy(ids_np).cuda()
        offsets = torch.full((N + 1,), -7, dtype=torch.int32, device="cuda")
        perm = torch.full((T * K,), -7, dtype=torch.int32, device="cuda")
        lm.lmoe_dispatch_noalloc(d_ids, T, K, N, offsets, perm)
        torch.cuda.synchronize()
        return offsets.cpu().numpy(), perm.cpu().numpy()

    off, perm = run(ids)
    off_x, perm_x = expected(ids)
    np.testing.assert_array_equal(off, off_x)
    np.testing.assert_array_equal(perm, perm_x)
    assert off[N] == T * K - 4 and (perm[off[N]:] == -1).all()

    dup = ids.copy()
    dup[40] = [3, 3, 7, 9]
    off, perm = run(dup)
    off_x, perm_x = expected(dup)
    np.testing.assert_array_equal(off, off_x)      # both pairs of row 40 counted
    for e in range(N):
        got = perm[off[e]:off[e + 1]]
        want = perm_x[off_x[e]:off_x[e + 1]]
        if e != 3:
            np.testing.assert_array_equal(got, want)
            continue
        pair = {40 * K, 40 * K + 1}
        assert (got == -1).sum() == 1
        assert len(pair & set(got.tolist())) == 1
        rest = [p for p in got.tolist() if p != -1 and p not in pair]
        assert rest == [p for p in want.tolist() if p not in pair]
