"""Expert parallelism on one GPU: two expert-parallel ranks emulated in one
process (ep.forward_emulated moves the rows between them with copies; no
kernel waits on another), each running the library's three phases on its
half of the experts.  Each rank's y must match the fp64 oracle on the rank's
tokens (bf16 tolerance), and the single-GPU forward of the same tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from latent_mixture_experts_top_b200 import configs, synth
from tests import parity_util as pu
from tests.test_parity_gpu import MID_PAIR

pytestmark = pytest.mark.gpu


def _lm():
    from latent_mixture_experts_top_b200 import lmoe
    return lmoe


def _run(cfg, Ts, seed=0):
    from latent_mixture_experts_top_b200 import ep
    lm = _lm()
    world = len(Ts)
    inp = synth.make_inputs(cfg, seed, "cuda", T=sum(Ts))
    full = lm.LatentMoELayer(cfg, inp, max_tokens=max(Ts))
    ranks = [lm.LatentMoELayer(cfg, inp, max_tokens=max(Ts), ep_rank=r, ep_world=world)
             for r in range(world)]
    starts = np.cumsum([0] + list(Ts))
    xs = [inp["x"][starts[r]:starts[r + 1]].contiguous() for r in range(world)]
    ys = ep.forward_emulated([ep.CudaBackend(L) for L in ranks], xs)
    torch.cuda.synchronize()
    for L in ranks:
        assert lm.lmoe_device_status(L.handle) == 0
    Lo = pu.oracle_layer(inp, cfg.k_active, cfg.activation)
    for r in range(world):
        if Ts[r] == 0:
            assert ys[r].shape == (0, cfg.d)
            continue
        y_full = full.forward(xs[r])
        ids, gates, offsets, perm = ranks[r].route(xs[r])
        x_np = synth.to_numpy(xs[r])
        s_ref = oracle.router_logits(Lo, x_np)
        ids_g = ids.cpu().numpy()
        _, flipped = pu.check_routing(ids_g, gates.cpu().numpy(), s_ref, cfg.k_active)
        tok = np.arange(Ts[r])
        y_ref = pu.reference_y(Lo, x_np, tok, ids_g, flipped)
        err = pu.rel_err(pu.y_to_numpy(ys[r]), y_ref)
        same = torch.equal(ys[r], y_full)
        dev = float((ys[r].float() - y_full.float()).abs().max() / y_full.float().abs().max())
        print(f"{cfg.name} EP rank {r}/{world}: rel err {err:.3e}, vs single-GPU "
              f"{'bit-identical' if same else f'{dev:.2e}'}")
        assert err <= pu.TOL_BF16
        assert dev <= 1e-2
    with pytest.raises(lm.LmoeError) as e:
        lm.lmoe_forward(ranks[0].handle, xs[0], torch.empty_like(xs[0]), Ts[0])
    assert e.value.code == -7
    for L in ranks + [full]:
        L.close()


def test_expert_parallel_two_ranks_readme_acc():
    """README acc layer, experts split 128 / 128, ranks with 512 and 300
    tokens (single-CTA down GEMM on the received rows)."""
    _run(configs.README_ACC, [512, 300])


def test_expert_parallel_two_ranks_pair_down_gemm():
    """A layer whose received rows average > 256 per expert, so the down GEMM
    runs on CTA pairs over the received segments."""
    _run(MID_PAIR, [1100, 777])


def test_expert_parallel_rank_with_no_tokens():
    """A rank with no tokens still serves its experts for the other."""
    _run(MID_PAIR, [600, 0])
