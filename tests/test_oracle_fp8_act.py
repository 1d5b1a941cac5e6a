"""Pins of the oracle's quantised-activation readings (act_fp8: E4M3;
act_fp4: NVFP4), CPU only.

The pages put the experts in FP8 ("LatentMoE Explained": an expert is about
22 MB in FP8; the models are pretrained in NVFP4) but print no recipe for the
activations.  The reading taken: the routed experts multiply E4M3 activations
-- each token's z and each expert's hidden vector h are quantised with the
rule of the weight rows (power-of-two scale, E4M3 round-to-nearest-even,
saturating; pinned in tests/test_oracle_fp8.py) -- while the router, W_down,
the combine, W_up and the shared experts are unchanged.  Here the oracle's
forward with act_fp8 is held to the definition recomposed with numpy from the
pinned quantiser and the pinned router: a missing, misplaced or extra
quantisation step fails.  The NVFP4 reading is the same with the NVFP4 row
quantiser (pinned in tests/test_oracle_nvfp4.py) in place of E4M3.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle

D, L_, M, N, K, NS, MS = 64, 32, 48, 6, 2, 1, 32


def _weights(seed, activation):
    rng = np.random.default_rng(seed)
    w = lambda *s: rng.normal(0.0, 0.3, size=s)
    kw = dict(w_router=w(N, D), b_router=None, w_down=w(L_, D), w_up=w(D, L_),
              w_gate=w(N, M, L_), w_upx=w(N, M, L_), w_out=w(N, L_, M), s_gate=w(NS, MS, D),
              s_up=w(NS, MS, D), s_out=w(NS, D, MS), k_active=K, activation=activation)
    x = rng.normal(0.0, 1.0, size=(9, D))
    return kw, x


def _q(v, mode="e4m3"):
    v = np.asarray(v, dtype=np.float64)[None, :]
    return (oracle.fp8_rows(v) if mode == "e4m3" else oracle.nvfp4_rows(v))[0][0]


def _bf16(a):
    """float64 -> bf16 bit patterns, rounded to nearest even through float32."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _widen(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _silu(a):
    return a / (1.0 + np.exp(-a))


def _recompose(kw, x, act_fp8, mode="e4m3", rnd=False):
    r = (lambda v: _widen(_bf16(v))) if rnd else (lambda v: v)
    Lp = oracle.Layer(**kw)                        # unquantised: router and ids only
    s = oracle.router_logits(Lp, x)
    ids, g = oracle.select(s, K)
    relu2 = kw["activation"] == "relu2"
    y = np.zeros((x.shape[0], D))
    for t in range(x.shape[0]):
        z = kw["w_down"] @ x[t]
        if act_fp8:
            z = _q(r(z), mode)
        u = np.zeros(L_)
        for k in range(K):
            e = ids[t, k]
            b = kw["w_upx"][e] @ z
            h = np.maximum(b, 0.0) ** 2 if relu2 else _silu(kw["w_gate"][e] @ z) * b
            if act_fp8:
                h = _q(r(h), mode)
            u += g[t, k] * (kw["w_out"][e] @ h)
        y[t] = kw["w_up"] @ u
        for j in range(NS):
            b = kw["s_up"][j] @ x[t]
            h = np.maximum(b, 0.0) ** 2 if relu2 else _silu(kw["s_gate"][j] @ x[t]) * b
            y[t] += kw["s_out"][j] @ h
    return y


def _flag(mode):
    return {"act_fp8": True} if mode == "e4m3" else {"act_fp4": True}


@pytest.mark.parametrize("mode", ["e4m3", "nvfp4"])
@pytest.mark.parametrize("activation", ["swiglu", "relu2"])
def test_act_fp8_forward_is_the_quantised_recomposition(activation, mode):
    kw, x = _weights(1, activation)
    y, _, _ = oracle.forward(oracle.Layer(**kw, **_flag(mode)), x)
    y_ref = _recompose(kw, x, True, mode)
    np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-12 * np.abs(y_ref).max())
    # and it is not the unquantised layer
    y0 = _recompose(kw, x, False)
    assert np.abs(y - y0).max() > 1e-4 * np.abs(y0).max()


@pytest.mark.parametrize("mode", ["e4m3", "nvfp4"])
def test_bf16_layer_quantises_the_bf16_rounding_of_each_row(mode):
    """In a bf16 layer z and h are bf16 vectors: their codes are decided on
    the bf16 values (the precision the layer holds them in)."""
    kw, x = _weights(6, "swiglu")
    bits = {k: (_bf16(v) if isinstance(v, np.ndarray) else v) for k, v in kw.items()}
    xb = _bf16(x)
    y, _, _ = oracle.forward(oracle.Layer(**bits, **_flag(mode)), xb)
    wide = {k: (_widen(v) if isinstance(v, np.ndarray) else v) for k, v in bits.items()}
    y_ref = _recompose(wide, _widen(xb), True, mode, rnd=True)
    np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-12 * np.abs(y_ref).max())
    # a float64 layer with act_bf16 is the same layer
    y64, _, _ = oracle.forward(oracle.Layer(**wide, **_flag(mode), act_bf16=True), _widen(xb))
    np.testing.assert_allclose(y64, y_ref, rtol=0, atol=1e-12 * np.abs(y_ref).max())
    # and the rounding decides some codes: without it the result differs
    y_unrounded = _recompose(wide, _widen(xb), True, mode, rnd=False)
    assert np.abs(y_unrounded - y_ref).max() > 1e-9 * np.abs(y_ref).max()


def test_act_fp8_off_leaves_the_layer_unchanged():
    kw, x = _weights(2, "swiglu")
    y, _, _ = oracle.forward(oracle.Layer(**kw, act_fp8=False), x)
    np.testing.assert_allclose(y, _recompose(kw, x, False), rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode,hi", [("e4m3", 0.1), ("nvfp4", 0.4)])
def test_act_fp8_error_is_that_of_a_few_roundings(mode, hi):
    kw, x = _weights(3, "swiglu")
    y8, _, _ = oracle.forward(oracle.Layer(**kw, **_flag(mode)), x)
    y, _, _ = oracle.forward(oracle.Layer(**kw), x)
    rel = np.abs(y8 - y).max() / np.abs(y).max()
    assert 1e-4 < rel < hi, rel


def test_nvfp4_activations_need_whole_blocks():
    kw, x = _weights(5, "swiglu")          # m = 48, l = 32: whole 16-blocks
    oracle.forward(oracle.Layer(**kw, act_fp4=True), x)
    kw["w_gate"], kw["w_upx"], kw["w_out"] = kw["w_gate"][:, :40], kw["w_upx"][:, :40], kw["w_out"][:, :, :40]
    with pytest.raises(ValueError):
        oracle.forward(oracle.Layer(**kw, act_fp4=True), x)


@pytest.mark.parametrize("mode", ["e4m3", "nvfp4"])
def test_backward_refuses_quantised_activations(mode):
    kw, x = _weights(4, "swiglu")
    with pytest.raises(Exception):
        oracle.backward(oracle.Layer(**kw, **_flag(mode)), x, np.ones((x.shape[0], D)))


SRC = os.path.join(os.path.dirname(oracle.__file__), "lmoe_oracle.c")
MUTATIONS = {
    "no_hidden_quantisation": ("  if (quant_hidden) q_act(L, quant_hidden, a, hid);\n", "\n"),
    "no_z_quantisation": ("      if (L->act_quant) q_act(L, L->act_quant, z, l);  /* the experts read z quantised */\n",
                          "\n"),
    "shared_quantised_too": ("(size_t)j * d * L->m_shared, d, L->m_shared, d, xv, sh, scratch, 0);",
                             "(size_t)j * d * L->m_shared, d, L->m_shared, d, xv, sh, scratch, L->act_quant);"),
    "quantised_after_down": ("  if (quant_hidden) q_act(L, quant_hidden, a, hid);\n  matvec(Wo, L->dtype, off_out, out_w, hid, a, out);",
                             "  matvec(Wo, L->dtype, off_out, out_w, hid, a, out);\n  if (quant_hidden) q_act(L, quant_hidden, out, out_w);"),
    "no_bf16_rounding": ("  if (L->dtype == ODT_BF16 || (L->act_quant & OQ_BF16_ROWS))\n    for (int i = 0; i < n; ++i) v[i] = round_bf16(v[i]);\n",
                         "\n"),
    "modes_swapped": ("  if (mode == OQ_E4M3) q_vec_e4m3(v, n);\n  else if (mode == OQ_NVFP4) q_vec_nvfp4(v, n);",
                      "  if (mode == OQ_NVFP4) q_vec_e4m3(v, n);\n  else if (mode == OQ_E4M3) q_vec_nvfp4(v, n);"),
}


@pytest.mark.parametrize("mode", ["e4m3", "nvfp4"])
@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_act_fp8_pins_catch_mutation(name, mode, tmp_path):
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
        with pytest.raises(AssertionError):
            test_act_fp8_forward_is_the_quantised_recomposition("swiglu", mode)
            test_bf16_layer_quantises_the_bf16_rounding_of_each_row(mode)
    finally:
        oracle._swap_library(None)
