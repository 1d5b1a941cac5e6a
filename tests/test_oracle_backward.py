"""Pins of the oracle's backward (CPU only).

The pages give no gradient formulas; the backward is the derivative of the
forward the other pins fix.  So it is pinned against that forward itself, by
central finite differences in fp64 along random directions, one parameter
group at a time (x, each weight, the router bias), for both expert
activations.  Also: a closed form (K' = 1 makes every gate 1, so nothing
reaches the router), and additivity over token subsets.  A mutation test
plants mistakes in the backward and requires one of these pins to fail.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

D, LAT, M, N, K, NS, MS, T = 16, 8, 12, 6, 3, 2, 10, 7
EPS = 1e-6


def _layer(rng, activation="swiglu", k=K, bias=True, params=None):
    f = lambda *s: rng.standard_normal(s) * 0.35
    p = params or dict(w_router=f(N, D), b_router=f(N) if bias else None,
                       w_down=f(LAT, D), w_up=f(D, LAT), w_gate=f(N, M, LAT),
                       w_upx=f(N, M, LAT), w_out=f(N, LAT, M), s_gate=f(NS, MS, D),
                       s_up=f(NS, MS, D), s_out=f(NS, D, MS))
    return p, oracle.Layer(**p, k_active=k, activation=activation)


def _objective(params, x, dy, activation, k):
    layer = oracle.Layer(**params, k_active=k, activation=activation)
    y, ids, _ = oracle.forward(layer, x)
    return float(np.sum(y * dy)), ids


def _fd_check(activation, group, seed, k=K):
    rng = np.random.default_rng(seed)
    params, layer = _layer(rng, activation, k)
    x = rng.standard_normal((T, D))
    dy = rng.standard_normal((T, D))
    g = oracle.backward(layer, x, dy)
    if group == "x":
        v = rng.standard_normal(x.shape)
        fp, ids_p = _objective(params, x + EPS * v, dy, activation, k)
        fm, ids_m = _objective(params, x - EPS * v, dy, activation, k)
        analytic = float(np.sum(g["dx"] * v))
    else:
        v = rng.standard_normal(params[group].shape)
        pp = dict(params); pp[group] = params[group] + EPS * v
        pm = dict(params); pm[group] = params[group] - EPS * v
        fp, ids_p = _objective(pp, x, dy, activation, k)
        fm, ids_m = _objective(pm, x, dy, activation, k)
        analytic = float(np.sum(g[group] * v))
    assert np.array_equal(ids_p, ids_m), "the probe moved the selection; pick another seed"
    numeric = (fp - fm) / (2 * EPS)
    scale = max(1.0, abs(numeric))
    assert abs(numeric - analytic) <= 1e-6 * scale, (group, numeric, analytic)


GROUPS = ["x", "w_router", "b_router", "w_down", "w_up", "w_gate", "w_upx", "w_out",
          "s_gate", "s_up", "s_out"]


@pytest.mark.parametrize("activation", ["swiglu", "relu2"])
@pytest.mark.parametrize("group", GROUPS)
def test_backward_matches_finite_differences(activation, group):
    if activation == "relu2" and group in ("w_gate", "s_gate"):
        # two-matrix experts never read the gate weights: gradient exactly 0
        rng = np.random.default_rng(3)
        _, layer = _layer(rng, activation)
        g = oracle.backward(layer, rng.standard_normal((T, D)), rng.standard_normal((T, D)))
        assert not np.any(g[group])
        return
    _fd_check(activation, group, seed=11)


def test_backward_finite_differences_second_seed():
    for group in ("x", "w_router", "w_out", "w_upx"):
        _fd_check("swiglu", group, seed=29)


def test_single_active_expert_sends_nothing_to_the_router():
    """K' = 1: the renormalised gate is identically 1, so ds = 0."""
    rng = np.random.default_rng(5)
    _, layer = _layer(rng, k=1)
    g = oracle.backward(layer, rng.standard_normal((T, D)), rng.standard_normal((T, D)))
    assert not np.any(g["w_router"]) and not np.any(g["b_router"])
    assert np.any(g["w_out"])


def test_weight_gradients_add_over_token_subsets():
    rng = np.random.default_rng(8)
    _, layer = _layer(rng)
    x = rng.standard_normal((T, D))
    dy = rng.standard_normal((T, D))
    full = oracle.backward(layer, x, dy)
    a, b = np.arange(0, 3), np.arange(3, T)
    ga = oracle.backward(layer, x, dy[a], tokens=a)
    gb = oracle.backward(layer, x, dy[b], tokens=b)
    for k in oracle.GRAD_NAMES:
        np.testing.assert_allclose(ga[k] + gb[k], full[k], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.concatenate([ga["dx"], gb["dx"]]), full["dx"],
                               rtol=1e-12, atol=1e-12)


# ---- the pins above must catch plausible mistakes in the backward
SRC = os.path.join(os.path.dirname(oracle.__file__), "lmoe_oracle.c")
MUTATIONS = {
    "dsilu_missing_term": ("return sg * (1.0 + a * (1.0 - sg));", "return sg;"),
    "gate_grad_without_mean": ("DS[n * K + k] = g[k] * (dg[k] - gdg);",
                               "DS[n * K + k] = g[k] * dg[k];"),
    "slot_grad_without_gate": ("for (int j = 0; j < l; ++j) dok[j] = g[k] * du[j];",
                               "for (int j = 0; j < l; ++j) dok[j] = du[j];"),
    "relu2_grad_without_two": ("db[c] = dh * 2.0 * (b[c] > 0.0 ? b[c] : 0.0);",
                               "db[c] = dh * (b[c] > 0.0 ? b[c] : 0.0);"),
    "up_grad_transposed": ("for (int i = 0; i < d; ++i) acc += elem(L->w_up, L->dtype, (size_t)i * l + j) * dyr[i];",
                           "for (int i = 0; i < d; ++i) acc += elem(L->w_up, L->dtype, (size_t)j * d + i) * dyr[i];"),
    "down_grad_dropped": ("dxs[i] += acc;\n      }\n      for (int j = 0; j < ns; ++j)",
                          "dxs[i] += 0.0 * acc;\n      }\n      for (int j = 0; j < ns; ++j)"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_backward_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(lib), str(mutated), "-lm"])
    oracle._swap_library(str(lib))
    try:
        caught = False
        for act in ("swiglu", "relu2"):
            for group in GROUPS:
                if act == "relu2" and group in ("w_gate", "s_gate"):
                    continue
                try:
                    _fd_check(act, group, seed=11)
                except AssertionError:
                    caught = True
                    break
            if caught:
                break
        assert caught, f"no pin caught mutation {name}"
    finally:
        oracle._swap_library(None)
