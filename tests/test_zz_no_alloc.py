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
