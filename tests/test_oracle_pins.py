"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own loop: each checks it against a
hand-derived closed form, a brute-force enumeration, a special case that
reduces to a textbook layer, or an invariant of the definition
("LatentMoE Explained": Figure 3, Figure 8, Figure 9 and the MoE / LatentMoE
code modules; Latent-MoE README, "Usage").
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _layer_from_json(g):
    f64 = lambda k: np.array(g[k], dtype=np.float64)
    d = len(g["x"][0])
    act = g.get("activation", "swiglu")
    if "s_up" in g:
        sg = f64("s_gate") if "s_gate" in g else None
        su, so = f64("s_up"), f64("s_out")
    else:  # no shared expert
        sg, su, so = (np.zeros((0, 1, d)), np.zeros((0, 1, d)), np.zeros((0, d, 1)))
    return oracle.Layer(w_router=f64("w_router"), b_router=None, w_down=f64("w_down"),
                        w_up=f64("w_up"), w_gate=f64("w_gate") if "w_gate" in g else None,
                        w_upx=f64("w_upx"), w_out=f64("w_out"), s_gate=sg, s_up=su,
                        s_out=so, k_active=g["k_active"], activation=act)


def rand_layer(rng, d, l, m, N, K, ns, ms, dtype=np.float64, bias=False, wstd=0.3,
               activation="swiglu"):
    r = lambda *s: (rng.standard_normal(s) * wstd).astype(dtype)
    return oracle.Layer(
        w_router=r(N, d), b_router=(rng.standard_normal(N) * 0.5 if bias else None),
        w_down=r(l, d), w_up=r(d, l), w_gate=r(N, m, l), w_upx=r(N, m, l),
        w_out=r(N, l, m), s_gate=r(ns, ms, d), s_up=r(ns, ms, d), s_out=r(ns, d, ms),
        k_active=K, activation=activation)


def silu(a):
    return a / (1.0 + np.exp(-a))


def ffn(Wg, Wu, Wo, v, activation="swiglu"):
    """Independent numpy expert FFN in matrix form (test-side, for reductions):
    SwiGLU W_o (silu(W_g v) * W_u v), or the pages' squared-ReLU Expert class
    W_o (relu(W_u v))**2 with two matrices."""
    if activation == "relu2":
        return Wo @ (np.maximum(Wu @ v, 0.0) ** 2)
    return Wo @ (silu(Wg @ v) * (Wu @ v))


# --------------------------------------------------------------- golden cases

def test_golden_hand_case_b():
    g = _golden("hand_case_b.json")
    L = _layer_from_json(g)
    x = np.array(g["x"], dtype=np.float64)
    y, ids, gates = oracle.forward(L, x)
    assert ids.tolist() == g["expect_ids"]
    np.testing.assert_allclose(gates, g["expect_gates"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(y, g["expect_y"], rtol=0, atol=g["atol"])


def test_golden_hand_case_relu2():
    g = _golden("hand_case_relu2.json")
    L = _layer_from_json(g)
    y, ids, gates = oracle.forward(L, np.array(g["x"], dtype=np.float64))
    assert ids.tolist() == g["expect_ids"]
    np.testing.assert_allclose(y, g["expect_y"], rtol=0, atol=g["atol"])


def test_golden_silu_sign_and_gate_role():
    g = _golden("hand_case_silu.json")
    L = _layer_from_json(g)
    y, ids, gates = oracle.forward(L, np.array(g["x"], dtype=np.float64))
    assert ids.tolist() == [[0], [0]]
    np.testing.assert_allclose(gates, 1.0, rtol=0, atol=0)
    np.testing.assert_allclose(y, g["expect_y"], rtol=0, atol=g["atol"])


# ------------------------------------------------------------- routing pins

@pytest.mark.parametrize("N,K", [(2, 1), (5, 2), (7, 3), (8, 8), (10, 4)])
def test_topk_brute_force(N, K):
    """The selected set is the K-subset of maximal logit sum (lexicographic
    tie-break), listed by (logit desc, index asc)."""
    rng = np.random.default_rng(N * 100 + K)
    s = rng.standard_normal((40, N))
    s[::5, 1:3] = s[::5, 0:1]           # exact ties on every fifth row
    s[1::7] = np.round(s[1::7])         # many ties
    ids, gates = oracle.select(s, K)
    for t in range(s.shape[0]):
        best = None
        for sub in itertools.combinations(range(N), K):  # lexicographic order
            tot = sum(s[t, e] for e in sub)
            if best is None or tot > best[0]:
                best = (tot, sub)
        assert sorted(ids[t].tolist()) == list(best[1])
        order = sorted(best[1], key=lambda e: (-s[t, e], e))
        assert ids[t].tolist() == order
        p = np.exp(s[t] - s[t].max())
        p /= p.sum()
        np.testing.assert_allclose(gates[t], p[order] / p[order].sum(), rtol=1e-14)


def test_topk_ties_go_to_lower_index():
    s = np.array([[2.0, 1.0, 1.0, 0.0], [1.0, 2.0, 2.0, 0.0], [0.0, 0.0, 0.0, 0.0]])
    ids, g = oracle.select(s, 2)
    assert ids.tolist() == [[0, 1], [1, 2], [0, 1]]
    e = math.e
    np.testing.assert_allclose(g[0], [e / (1 + e), 1 / (1 + e)], rtol=1e-15)
    np.testing.assert_allclose(g[1], [0.5, 0.5], rtol=0, atol=0)
    np.testing.assert_allclose(g[2], [0.5, 0.5], rtol=0, atol=0)


def test_zero_router_selects_first_experts_uniformly():
    rng = np.random.default_rng(1)
    L = rand_layer(rng, 8, 4, 6, 9, 3, 1, 5)
    L._keep["w_router"][:] = 0.0
    x = rng.standard_normal((5, 8))
    _, ids, gates = oracle.forward(L, x)
    assert (ids == np.array([0, 1, 2])).all()
    np.testing.assert_allclose(gates, 1.0 / 3.0, rtol=1e-15)


def test_gates_sum_to_one_and_are_non_increasing():
    rng = np.random.default_rng(2)
    s = rng.standard_normal((200, 64)) * 3
    for K in (1, 6, 24, 64):
        ids, g = oracle.select(s, K)
        np.testing.assert_allclose(g.sum(1), 1.0, rtol=1e-14)
        assert (np.diff(g, axis=1) <= 1e-15).all()
        if K == 1:
            np.testing.assert_allclose(g, 1.0, rtol=0, atol=0)
        assert (np.diff(np.take_along_axis(s, ids.astype(np.int64), 1), axis=1) <= 0).all()


def test_router_bias_enters_before_softmax():
    """With a bias b, routing equals routing of the unbiased logits plus b."""
    rng = np.random.default_rng(3)
    L = rand_layer(rng, 8, 4, 6, 9, 3, 1, 5, bias=True)
    x = rng.standard_normal((10, 8))
    s = oracle.router_logits(L, x)
    s_plain = x @ L._keep["w_router"].T        # textbook matrix product
    np.testing.assert_allclose(s, s_plain + L.b_router, rtol=1e-13, atol=1e-13)
    _, ids, g = oracle.forward(L, x)
    ids2, g2 = oracle.select(s_plain + L.b_router, 3)
    assert (ids == ids2).all()
    np.testing.assert_allclose(g, g2, rtol=1e-14)


# ------------------------------------------------------- whole-layer pins

@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_dense_limit_K_equals_N(act):
    """K' = N': no selection is left, y = W_up sum_e softmax(s)_e E_e(z) + shared."""
    rng = np.random.default_rng(4)
    d, l, m, N, ns, ms = 12, 6, 10, 5, 2, 7
    L = rand_layer(rng, d, l, m, N, N, ns, ms, activation=act)
    k = L._keep
    x = rng.standard_normal((6, d))
    y, _, _ = oracle.forward(L, x)
    for t in range(x.shape[0]):
        s = k["w_router"] @ x[t]
        p = np.exp(s - s.max()); p /= p.sum()
        z = k["w_down"] @ x[t]
        u = sum(p[e] * ffn(k["w_gate"][e], k["w_upx"][e], k["w_out"][e], z, act)
                for e in range(N))
        ref = k["w_up"] @ u + sum(ffn(k["s_gate"][j], k["s_up"][j], k["s_out"][j], x[t], act)
                                  for j in range(ns))
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12)


def test_alpha_one_relu2_is_the_pages_moe_class():
    """alpha = 1, identity projections, squared-ReLU experts: the layer is the
    MoE class of the article's code (router on x, topk of the softmax,
    renormalise, experts down(relu(up(x))**2), shared experts added)."""
    rng = np.random.default_rng(15)
    d, m, N, K, ns = 10, 8, 7, 3, 2
    L = rand_layer(rng, d, d, m, N, K, ns, m, activation="relu2")
    k = L._keep
    k["w_down"][:] = np.eye(d)
    k["w_up"][:] = np.eye(d)
    x = rng.standard_normal((9, d))
    y, ids, _ = oracle.forward(L, x)
    for t in range(x.shape[0]):
        scores = k["w_router"] @ x[t]
        probs = np.exp(scores - scores.max()); probs /= probs.sum()
        top = np.argsort(-probs, kind="stable")[:K]
        w = probs[top] / probs[top].sum()
        expert = lambda up, down, v: down @ (np.maximum(up @ v, 0.0) ** 2)
        ref = sum(w[i] * expert(k["w_upx"][e], k["w_out"][e], x[t]) for i, e in enumerate(top))
        ref = ref + sum(expert(k["s_up"][j], k["s_out"][j], x[t]) for j in range(ns))
        assert sorted(ids[t].tolist()) == sorted(top.tolist())
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12)


def test_alpha_one_identity_projections_is_standard_moe():
    """alpha = 1 with W_down = W_up = I is the standard d-space MoE layer
    ("LatentMoE Explained", the MoE code module, with SwiGLU experts)."""
    rng = np.random.default_rng(5)
    d, m, N, K, ns, ms = 10, 8, 7, 3, 2, 6
    L = rand_layer(rng, d, d, m, N, K, ns, ms)
    k = L._keep
    k["w_down"][:] = np.eye(d)
    k["w_up"][:] = np.eye(d)
    x = rng.standard_normal((9, d))
    y, ids, _ = oracle.forward(L, x)
    for t in range(x.shape[0]):
        scores = k["w_router"] @ x[t]
        probs = np.exp(scores - scores.max()); probs /= probs.sum()
        top = np.argsort(-probs, kind="stable")[:K]
        w = probs[top] / probs[top].sum()
        ref = sum(w[i] * ffn(k["w_gate"][e], k["w_upx"][e], k["w_out"][e], x[t])
                  for i, e in enumerate(top))
        ref = ref + sum(ffn(k["s_gate"][j], k["s_up"][j], k["s_out"][j], x[t])
                        for j in range(ns))
        assert sorted(ids[t].tolist()) == sorted(top.tolist())
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12)


def test_combine_then_up_equals_per_expert_up():
    """W_up sum_k g_k E_k(z) = sum_k g_k W_up E_k(z)  ("W_up wrapped their sum")."""
    rng = np.random.default_rng(6)
    L = rand_layer(rng, 16, 8, 12, 11, 4, 1, 9)
    x = rng.standard_normal((5, 16))
    y, ids, gates = oracle.forward(L, x)
    for t in range(x.shape[0]):
        z = oracle.down(L, x, t)
        alt = sum(gates[t, k] * oracle.up(L, oracle.expert(L, int(ids[t, k]), z))
                  for k in range(L.K))
        alt = alt + oracle.shared(L, x, t)
        np.testing.assert_allclose(y[t], alt, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_mask_form_over_all_experts(act):
    """y equals the sum over ALL experts with zero gates off the top-K'."""
    rng = np.random.default_rng(7)
    d, l, m, N, K = 12, 4, 6, 9, 3
    L = rand_layer(rng, d, l, m, N, K, 1, 5, activation=act)
    k = L._keep
    x = rng.standard_normal((8, d))
    y, ids, gates = oracle.forward(L, x)
    for t in range(x.shape[0]):
        gate_full = np.zeros(N)
        gate_full[ids[t]] = gates[t]
        z = k["w_down"] @ x[t]
        u = sum(gate_full[e] * ffn(k["w_gate"][e], k["w_upx"][e], k["w_out"][e], z, act)
                for e in range(N))
        ref = k["w_up"] @ u + ffn(k["s_gate"][0], k["s_up"][0], k["s_out"][0], x[t], act)
        np.testing.assert_allclose(y[t], ref, rtol=1e-12, atol=1e-12)


def test_token_permutation_invariance():
    rng = np.random.default_rng(8)
    L = rand_layer(rng, 12, 6, 8, 10, 3, 1, 6, dtype=np.float32)
    x = rng.standard_normal((20, 12)).astype(np.float32)
    P = rng.permutation(20)
    y, ids, g = oracle.forward(L, x)
    yp, idsp, gp = oracle.forward(L, x[P])
    np.testing.assert_array_equal(yp, y[P])
    np.testing.assert_array_equal(idsp, ids[P])
    off, perm, pos = oracle.dispatch(ids, 10)
    offp, permp, posp = oracle.dispatch(idsp, 10)
    np.testing.assert_array_equal(off, offp)
    for e in range(10):
        a = {(int(P.tolist().index(q // 3)), q % 3) for q in perm[off[e]:off[e + 1]]}
        b = {(q // 3, q % 3) for q in permp[offp[e]:offp[e + 1]]}
        assert a == b


def test_bf16_inputs_widen_exactly():
    """bf16 bit patterns give the same result as the same values in float32."""
    rng = np.random.default_rng(9)
    L32 = rand_layer(rng, 16, 8, 8, 6, 2, 1, 8, dtype=np.float32)
    bf = {}
    for k, v in L32._keep.items():
        bits = (v.view(np.uint32) + 0x8000) >> 16   # any rounding: we only need bf16 values
        bf[k] = bits.astype(np.uint16)
        L32._keep[k][...] = (bf[k].astype(np.uint32) << 16).view(np.float32)
    Lbf = oracle.Layer(b_router=None, k_active=2, **bf)
    x = rng.standard_normal((4, 16)).astype(np.float32)
    xb = ((x.view(np.uint32) + 0x8000) >> 16).astype(np.uint16)
    x[...] = (xb.astype(np.uint32) << 16).view(np.float32)
    y32, _, _ = oracle.forward(L32, x)
    ybf, _, _ = oracle.forward(Lbf, xb)
    np.testing.assert_array_equal(y32, ybf)


def test_given_ids_matches_own_routing():
    rng = np.random.default_rng(10)
    L = rand_layer(rng, 12, 6, 8, 10, 4, 1, 6)
    x = rng.standard_normal((7, 12))
    y, ids, g = oracle.forward(L, x)
    y2, ids2, g2 = oracle.forward(L, x, ids=ids)
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(g, g2)
    tok = np.array([6, 0, 3])
    y3, _, _ = oracle.forward(L, x, tokens=tok)
    np.testing.assert_array_equal(y3, y[tok])


# ------------------------------------------------------------ dispatch pins

@pytest.mark.parametrize("T,K,N", [(1, 1, 1), (37, 4, 16), (64, 6, 256), (200, 3, 5)])
def test_dispatch_is_the_unique_stable_grouping(T, K, N):
    rng = np.random.default_rng(T * K + N)
    ids = np.stack([rng.permutation(N)[:K] for _ in range(T)]).astype(np.int32)
    if T >= 64:                 # a hot expert (0) in every row; others starve
        for row in ids:
            if 0 not in row:
                row[0] = 0
    off, perm, pos = oracle.dispatch(ids, N)
    counts = np.bincount(ids.ravel(), minlength=N)
    np.testing.assert_array_equal(np.diff(off), counts)
    assert off[0] == 0 and off[-1] == T * K
    assert sorted(perm.tolist()) == list(range(T * K))
    np.testing.assert_array_equal(pos[perm], np.arange(T * K))
    flat = ids.ravel()
    for e in range(N):
        seg = perm[off[e]:off[e + 1]]
        assert (flat[seg] == e).all()
        assert (np.diff(seg // K) > 0).all()   # token ascending, each token once
