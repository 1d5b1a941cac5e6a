"""GPU parity of the layer backward (lmoe_backward) against the fp64 oracle.

Inputs and the cotangent dy come from latent_mixture_experts_top_b200.synth.
The routing is checked as in the forward parity tests; the oracle then takes
the library's own ids (identical off near-ties), so that both sides
differentiate the same piecewise-smooth branch.  Every array -- dx and each
weight gradient -- is compared as max|g - g_ref| / max|g_ref| against the
mode's tolerance: 1e-5 for fp32 (fp32 accumulation of sums over at most a
few thousand terms of one sign-mixed product), 2e-2 for bf16.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from latent_mixture_experts_top_b200 import configs, synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _lmoe():
    from latent_mixture_experts_top_b200 import lmoe
    return lmoe


def _backward_case(cfg, T=None, max_tokens=None, seed=0, tol=None, warm_seed=None):
    lm = _lmoe()
    T = cfg.T if T is None else T
    inp = synth.make_inputs(cfg, seed, "cuda", T=T)
    dy = synth.make_cotangent(cfg, seed, "cuda", T=T)
    layer = lm.LatentMoELayer(cfg, inp, max_tokens=max_tokens or cfg.T, training=True)
    x = inp["x"]
    if warm_seed is not None:
        # an earlier call on other tokens leaves its rows in the workspace
        xw = synth.make_inputs(cfg, warm_seed, "cuda", T=max_tokens or cfg.T)["x"]
        dyw = synth.make_cotangent(cfg, warm_seed, "cuda", T=max_tokens or cfg.T)
        layer.backward(xw, dyw)
    dx, grads = layer.backward(x, dy)
    ids, gates, offsets, perm = layer.route(x)
    torch.cuda.synchronize()
    assert lm.lmoe_device_status(layer.handle) == 0
    L = pu.oracle_layer(inp, cfg.k_active, cfg.activation)
    x_np = synth.to_numpy(x)
    ids_g = ids.cpu().numpy()
    s_ref = oracle.router_logits(L, x_np)
    pu.check_routing(ids_g, gates.cpu().numpy(), s_ref, cfg.k_active)
    dy_np = dy.float().cpu().numpy().astype(np.float64)
    ref = oracle.backward(L, x_np, dy_np, ids=ids_g, want=tuple(grads))
    tol = tol or (pu.TOL_F32 if cfg.dtype == "f32" else pu.TOL_BF16)
    errs = {"dx": pu.rel_err(dx.float().cpu().numpy().astype(np.float64), ref["dx"])}
    for k, v in grads.items():
        errs[k] = pu.rel_err(v.cpu().numpy().astype(np.float64), ref[k])
    print(cfg.name, T, {k: f"{v:.2e}" for k, v in errs.items()})
    layer.close()
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, bad
    return errs


def test_backward_tiny_f32_swiglu():
    _backward_case(configs.TINY_F32)


def test_backward_tiny_f32_relu2():
    _backward_case(configs.TINY_RELU2_F32)


def test_backward_tiny_f32_ragged_tokens():
    """T = 37 tokens in a workspace for 64: partial tiles everywhere."""
    _backward_case(configs.TINY_F32, T=37, max_tokens=64)


# bf16 cases: a mid-size layer that spans several tiles of every GEMM with
# ragged tails (T*K' = 2400 rows over 32 experts), both expert activations,
# with a router bias; and the README acc layer's full shape at T = 256.
MID_BF16 = configs.LayerConfig("mid_bf16_T300_d512_l256_m256_N32_K8_bias", T=300, d=512, m=256,
                               n_experts=16, top_k=4, alpha=2, n_shared=1, m_shared=256,
                               variant="acc", router_bias_std=0.5)
MID_RELU2_BF16 = replace(MID_BF16, name="mid_relu2_bf16_T300_d512_l256_m192_N32_K8", m=192,
                         m_shared=192, activation="relu2", router_bias_std=0.0)


def test_backward_bf16_mid_swiglu_bias():
    _backward_case(MID_BF16)


def test_backward_bf16_mid_relu2():
    _backward_case(MID_RELU2_BF16)


def test_backward_bf16_after_a_larger_call():
    """A call on fewer tokens after one on more: the expert row ranges move,
    and rows the earlier call wrote must not leak into the weight gradients."""
    _backward_case(MID_BF16, T=200, max_tokens=300, warm_seed=7)


def test_backward_bf16_readme_acc_shape():
    _backward_case(configs.README_ACC, T=256, max_tokens=256)


def test_backward_zero_tokens_gives_zero_gradients():
    lm = _lmoe()
    cfg = configs.TINY_F32
    inp = synth.make_inputs(cfg, 0, "cuda")
    layer = lm.LatentMoELayer(cfg, inp, training=True)
    x = inp["x"][:0]
    dx, grads = layer.backward(x, x.clone())
    torch.cuda.synchronize()
    for v in grads.values():
        assert not torch.any(v)
    layer.close()


def test_backward_needs_a_training_handle():
    lm = _lmoe()
    cfg = configs.TINY_F32
    inp = synth.make_inputs(cfg, 0, "cuda")
    layer = lm.LatentMoELayer(cfg, inp)   # training off
    with pytest.raises(lm.LmoeError) as e:
        layer.backward(inp["x"], inp["x"].clone())
    assert e.value.code == -7
    layer.close()
