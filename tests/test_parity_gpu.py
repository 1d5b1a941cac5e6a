"""GPU parity: the CUDA library through its C ABI against the fp64 oracle.

Inputs come from latent_mixture_experts_top_b200.synth (seeded, on the GPU);
the oracle gets host copies of the same rounded values.  Tolerances (from
the layer's arithmetic): fp32 mode 1e-5 and bf16 mode 2e-2 on
max|y - y_ref| / max|y_ref|; routing and dispatch exact (see parity_util).
"""
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


_INPUT_CACHE = {}


def _inputs(cfg, seed=0):
    key = (cfg.name, seed)
    if key not in _INPUT_CACHE:
        _INPUT_CACHE.clear()   # keep at most one big weight set on the device
        torch.cuda.empty_cache()
        _INPUT_CACHE[key] = synth.make_inputs(cfg, seed, "cuda")
    return _INPUT_CACHE[key]


def _run(cfg, inp, x=None, max_tokens=None):
    lm = _lmoe()
    layer = lm.LatentMoELayer(cfg, inp, max_tokens=max_tokens)
    x = inp["x"] if x is None else x
    y = layer.forward(x)
    ids, gates, offsets, perm = layer.route(x)
    torch.cuda.synchronize()
    assert lm.lmoe_device_status(layer.handle) == 0
    return layer, y, ids, gates, offsets, perm


def _check_layer(cfg, n_sample, seed=0):
    """n_sample: compare that many sampled tokens, every token (>= T), or
    "tiles": the tokens that put a compared row into every expert's first and
    last grouped-GEMM M-tile (128- and 256-row tiles), plus a random spread."""
    inp = _inputs(cfg, seed)
    layer, y, ids, gates, offsets, perm = _run(cfg, inp)
    L = pu.oracle_layer(inp, cfg.k_active, cfg.activation)
    x_np = synth.to_numpy(inp["x"])
    s_ref = oracle.router_logits(L, x_np)
    ids_g, gates_g = ids.cpu().numpy(), gates.cpu().numpy()
    near, flipped = pu.check_routing(ids_g, gates_g, s_ref, cfg.k_active)
    pu.check_dispatch(ids_g, offsets.cpu().numpy(), perm.cpu().numpy(), cfg.n_routed)
    if not flipped.any():   # then the oracle's own dispatch must agree too
        ids_ref, _ = oracle.select(s_ref, cfg.k_active)
        pu.check_dispatch_against_oracle_ids(ids_ref, ids_g, offsets.cpu().numpy(),
                                             perm.cpu().numpy(), cfg.n_routed)
    if n_sample == "tiles":
        cover = pu.tile_cover_tokens(offsets.cpu().numpy(), perm.cpu().numpy(), cfg.k_active)
        tok = np.union1d(cover, pu.sample_tokens(cfg.T, 64))
    elif n_sample < cfg.T:
        tok = pu.sample_tokens(cfg.T, n_sample)
    else:
        tok = np.arange(cfg.T)
    y_ref = pu.reference_y(L, x_np, tok, ids_g, flipped)
    err = pu.rel_err(pu.y_to_numpy(y)[tok], y_ref)
    tol = pu.TOL_F32 if cfg.dtype == "f32" else pu.TOL_BF16
    print(f"{cfg.name}: rel err {err:.3e} (tol {tol}) over {len(tok)} tokens, "
          f"near-tie {near.sum()}, flipped {flipped.sum()}")
    assert err <= tol
    layer.close()
    return err


def test_parity_tiny_f32_all_tokens():
    _check_layer(configs.TINY_F32, n_sample=10 ** 9)


def test_parity_readme_acc_all_tokens():
    _check_layer(configs.README_ACC, n_sample=10 ** 9)


def test_parity_readme_eff_all_tokens():
    _check_layer(configs.README_EFF, n_sample=10 ** 9)


def test_parity_decode_all_tokens():
    _check_layer(configs.DECODE, n_sample=10 ** 9)


def test_parity_prefill_biased_router():
    """Every expert's first and last 128-row (gate/up) and 256-row (down, CTA
    pairs) M-tile holds a compared row."""
    _check_layer(configs.PREFILL, n_sample="tiles")


# A mid-size layer whose experts average 275 rows (T K / N = 1100 * 8 / 32),
# so that the expert down GEMM runs on CTA pairs over 256-row M-tiles: with
# the router bias the counts spread, giving full pair tiles, ragged ones and
# tiles whose second CTA has no rows; T = 1100 also leaves the dense GEMMs a
# ragged last pair tile.  Every token is compared.
MID_PAIR = configs.LayerConfig("mid_pair_T1100_d512_l256_m256_N32_K8_bias", T=1100, d=512,
                               m=256, n_experts=16, top_k=4, alpha=2, n_shared=1, m_shared=256,
                               variant="acc", router_bias_std=0.5)


def test_parity_pair_down_gemm_all_tokens():
    assert MID_PAIR.T * MID_PAIR.k_active >= 256 * MID_PAIR.n_routed
    _check_layer(MID_PAIR, n_sample=10 ** 9)


# K' = 72 > 64: routing takes the four-launch path (top-K', histogram scan,
# scatter, then the permutation) instead of the fused two-launch one.
WIDE_K_F32 = configs.LayerConfig("wide_k_f32_T64_d256_l128_N128_K72", T=64, d=256, m=256,
                                 n_experts=64, top_k=36, alpha=2, n_shared=1, m_shared=256,
                                 variant="acc", dtype="f32")
WIDE_K_BF16 = configs.LayerConfig("wide_k_bf16_T300_d256_l128_N128_K72", T=300, d=256, m=256,
                                  n_experts=64, top_k=36, alpha=2, n_shared=1, m_shared=256,
                                  variant="acc")


@pytest.mark.parametrize("cfg", [WIDE_K_F32, WIDE_K_BF16], ids=["f32", "bf16"])
def test_parity_wide_k_four_launch_routing(cfg):
    assert cfg.k_active == 72
    _check_layer(cfg, n_sample=10 ** 9)


# The method's degenerate cases and the largest expert count, every token
# compared: K' = 1 (the gate is 1), K' = N' (every expert: the dense limit),
# alpha = 1 (l = d, no compression), and N' = 1024 (the library's maximum;
# top-K' keys 32 per lane).
EDGE = [
    configs.LayerConfig("k1_f32_T64_d256_l128_N16_K1", T=64, d=256, m=256, n_experts=16, top_k=1,
                        alpha=2, n_shared=1, m_shared=256, variant="eff", dtype="f32",
                        n_routed_override=16),
    configs.LayerConfig("k1_bf16_T200_d256_l128_N32_K1", T=200, d=256, m=256, n_experts=32,
                        top_k=1, alpha=2, n_shared=1, m_shared=256, variant="eff",
                        n_routed_override=32),
    configs.LayerConfig("dense_f32_T64_d256_l128_N16_K16", T=64, d=256, m=256, n_experts=16,
                        top_k=16, alpha=2, n_shared=1, m_shared=256, variant="eff", dtype="f32",
                        n_routed_override=16),
    configs.LayerConfig("dense_bf16_T200_d256_l128_N32_K32", T=200, d=256, m=256, n_experts=32,
                        top_k=32, alpha=2, n_shared=1, m_shared=256, variant="eff",
                        n_routed_override=32),
    configs.LayerConfig("alpha1_f32_T64_d128_l128_N8_K2", T=64, d=128, m=128, n_experts=8, top_k=2,
                        alpha=1, n_shared=1, m_shared=128, variant="acc", dtype="f32"),
    configs.LayerConfig("alpha1_bf16_T300_d256_l256_N32_K4", T=300, d=256, m=256, n_experts=32,
                        top_k=4, alpha=1, n_shared=1, m_shared=256, variant="acc"),
    configs.LayerConfig("n1024_bf16_T512_d256_l128_N1024_K8", T=512, d=256, m=128, n_experts=512,
                        top_k=4, alpha=2, n_shared=1, m_shared=256, variant="acc"),
]


@pytest.mark.parametrize("cfg", EDGE, ids=lambda c: c.name)
def test_parity_degenerate_and_extreme_layers(cfg):
    _check_layer(cfg, n_sample=10 ** 9)


def test_parity_relu2_tiny_f32_all_tokens():
    _check_layer(configs.TINY_RELU2_F32, n_sample=10 ** 9)


def test_parity_relu2_95b_shape():
    """Squared-ReLU experts at the article's 95B running-example layer shape."""
    _check_layer(configs.RELU2_95B, n_sample=96)


@pytest.mark.parametrize("cfg,T", [(configs.TINY_F32, 1), (configs.TINY_F32, 5),
                                   (configs.TINY_F32, 63), (configs.README_ACC, 1),
                                   (configs.README_ACC, 5), (configs.README_ACC, 129),
                                   (configs.README_ACC, 333)],
                         ids=["f32-1", "f32-5", "f32-63", "bf16-1", "bf16-5", "bf16-129",
                              "bf16-333"])
def test_ragged_token_counts(cfg, T):
    """Token counts that are not a multiple of any tile, in a larger workspace."""
    assert T <= cfg.T
    inp = _inputs(cfg)
    x = inp["x"][:T].contiguous()
    layer, y, ids, gates, offsets, perm = _run(cfg, inp, x=x, max_tokens=cfg.T)
    L = pu.oracle_layer(inp, cfg.k_active)
    x_np = synth.to_numpy(x)
    s_ref = oracle.router_logits(L, x_np)
    ids_g = ids.cpu().numpy()
    _, flipped = pu.check_routing(ids_g, gates.cpu().numpy(), s_ref, cfg.k_active)
    pu.check_dispatch(ids_g, offsets.cpu().numpy(), perm.cpu().numpy(), cfg.n_routed)
    tok = np.arange(T) if T <= 64 else pu.sample_tokens(T, 48)
    y_ref = pu.reference_y(L, x_np, tok, ids_g, flipped)
    tol = pu.TOL_F32 if cfg.dtype == "f32" else pu.TOL_BF16
    assert pu.rel_err(pu.y_to_numpy(y)[tok], y_ref) <= tol
    layer.close()


@pytest.mark.parametrize("T", [1023, 1024, 1025])
def test_permuted_rows_on_both_copy_paths(T):
    """Below 1024 tokens the scatter itself copies z into dispatch order; from 1024 on, a
    positions-only scatter and a row-copy launch do.  Either way the permuted rows are
    zp[r] = z[perm[r] // K'] bit for bit, and y matches the oracle."""
    cfg = configs.README_ACC
    inp = _inputs(cfg)
    x = inp["x"][:T].contiguous()
    layer, y, ids, gates, offsets, perm = _run(cfg, inp, x=x, max_tokens=cfg.T)
    K, l = cfg.k_active, cfg.l
    z = layer.debug_tensor(1, torch.bfloat16, (T, l)).view(torch.int16)
    zp = layer.debug_tensor(2, torch.bfloat16, (T * K, l)).view(torch.int16)
    src = perm.long() // K
    assert torch.equal(zp, z[src])
    L = pu.oracle_layer(inp, K)
    x_np = synth.to_numpy(x)
    s_ref = oracle.router_logits(L, x_np)
    ids_g = ids.cpu().numpy()
    _, flipped = pu.check_routing(ids_g, gates.cpu().numpy(), s_ref, K)
    pu.check_dispatch(ids_g, offsets.cpu().numpy(), perm.cpu().numpy(), cfg.n_routed)
    tok = pu.sample_tokens(T, 48)
    y_ref = pu.reference_y(L, x_np, tok, ids_g, flipped)
    assert pu.rel_err(pu.y_to_numpy(y)[tok], y_ref) <= pu.TOL_BF16
    layer.close()


@pytest.mark.parametrize("cfg", [configs.TINY_F32, configs.README_ACC], ids=["f32", "bf16"])
def test_zero_tokens(cfg):
    lm = _lmoe()
    inp = _inputs(cfg)
    layer = lm.LatentMoELayer(cfg, inp)
    y = torch.full((1, cfg.d), 7.0, device="cuda", dtype=inp["x"].dtype)
    lm.lmoe_forward(layer.handle, inp["x"], y, 0)
    offsets = torch.full((cfg.n_routed + 1,), -1, dtype=torch.int32, device="cuda")
    lm.lmoe_route(layer.handle, inp["x"], 0, None, None, offsets, None)
    torch.cuda.synchronize()
    assert (y == 7.0).all()
    assert (offsets == 0).all()
    layer.close()


def test_hot_expert_and_starved_experts():
    """A router bias that sends every token to expert 3 (one expert gets all
    T tokens, several get none): dispatch and output still match."""
    cfg = configs.README_ACC
    inp = dict(_inputs(cfg))
    T = 512
    bias = torch.zeros(cfg.n_routed, device="cuda")
    bias[3] = 50.0
    bias[100:140] = -50.0
    inp["b_router"] = bias
    from dataclasses import replace
    cfgb = replace(cfg, router_bias_std=1.0)
    x = inp["x"][:T].contiguous()
    layer, y, ids, gates, offsets, perm = _run(cfgb, inp, x=x, max_tokens=T)
    off = offsets.cpu().numpy()
    assert off[4] - off[3] == T
    assert (np.diff(off)[100:140] == 0).all()
    L = pu.oracle_layer(inp, cfg.k_active)
    x_np = synth.to_numpy(x)
    s_ref = oracle.router_logits(L, x_np)
    ids_g = ids.cpu().numpy()
    _, flipped = pu.check_routing(ids_g, gates.cpu().numpy(), s_ref, cfg.k_active)
    pu.check_dispatch(ids_g, off, perm.cpu().numpy(), cfg.n_routed)
    tok = pu.sample_tokens(T, 40)
    y_ref = pu.reference_y(L, x_np, tok, ids_g, flipped)
    assert pu.rel_err(pu.y_to_numpy(y)[tok], y_ref) <= pu.TOL_BF16
    layer.close()


@pytest.mark.parametrize("pattern", ["four_levels", "thirty_equal"])
def test_exact_ties_route_to_lower_index(pattern):
    """Exactly equal router scores (zero router weights, a bias with repeated
    values): the selection takes the lower expert index among equal scores and
    the gates are equal.  "four_levels" (bias e % 4: 64 experts share the top
    score) leaves too many candidates for the short list; "thirty_equal"
    (thirty experts on distinct lanes share the top score) fills it with ties."""
    from dataclasses import replace
    cfg = configs.README_ACC
    N, K, T = cfg.n_routed, cfg.k_active, 256
    inp = dict(_inputs(cfg))
    inp["w_router"] = torch.zeros_like(inp["w_router"])
    bias = torch.zeros(N, device="cuda")
    if pattern == "four_levels":
        bias += (torch.arange(N, device="cuda") % 4).float()
        top = [e for e in range(N) if e % 4 == 3]
    else:
        chosen = sorted(5 + 7 * k for k in range(30))
        bias[chosen] = 1.0
        top = chosen
    inp["b_router"] = bias
    layer = _lmoe().LatentMoELayer(replace(cfg, router_bias_std=1.0), inp, max_tokens=T)
    ids, gates, offsets, perm = layer.route(inp["x"][:T].contiguous())
    torch.cuda.synchronize()
    want = np.array(top[:K], dtype=np.int32)
    assert (ids.cpu().numpy() == want[None, :]).all()
    g = gates.cpu().numpy()
    assert (g == g[0, 0]).all() and abs(float(g[0, 0]) - 1.0 / K) < 1e-7
    pu.check_dispatch(ids.cpu().numpy(), offsets.cpu().numpy(), perm.cpu().numpy(), N)
    layer.close()


@pytest.mark.parametrize("cfg", [configs.TINY_F32, configs.README_ACC], ids=["f32", "bf16"])
def test_deterministic(cfg):
    inp = _inputs(cfg)
    lm = _lmoe()
    layer = lm.LatentMoELayer(cfg, inp)
    y1 = layer.forward(inp["x"]).clone()
    y2 = layer.forward(inp["x"]).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    layer.close()


def test_forward_host_matches_device_path():
    cfg = configs.README_ACC
    inp = _inputs(cfg)
    lm = _lmoe()
    layer = lm.LatentMoELayer(cfg, inp)
    y_dev = layer.forward(inp["x"])
    x_h = inp["x"].cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    lm.lmoe_forward_host(layer.handle, x_h, y_h, cfg.T)
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_dev.cpu())
    layer.close()


@pytest.mark.parametrize("cfg,n,T", [(configs.README_ACC, 1, 1536), (configs.README_ACC, 2, 1536),
                                     (configs.README_ACC, 5, 1536), (configs.TINY_F32, 3, 40)],
                         ids=["bf16-1", "bf16-2", "bf16-5", "f32-3"])
def test_forward_host_batches_match_device_path(cfg, n, T):
    """Each batch of a stream (two staging sets, copies overlapping the neighbours'
    forwards) gives lmoe_forward's y for that batch, bit for bit; batches differ."""
    inp = _inputs(cfg)
    lm = _lmoe()
    layer = lm.LatentMoELayer(cfg, inp)
    step = max(1, (cfg.T - T) // 5)
    xs_dev = [inp["x"][(i * step) % (cfg.T - T + 1):][:T].contiguous() for i in range(n)]
    xs_dev = [x * (1.0 + 0.25 * i) for i, x in enumerate(xs_dev)]
    y_ref = [layer.forward(x).cpu() for x in xs_dev]
    x_h = [x.cpu().pin_memory() for x in xs_dev]
    y_h = [torch.full_like(x, float("nan")).pin_memory() for x in x_h]
    lm.lmoe_forward_host_batches(layer.handle, x_h, y_h, T)
    for i in range(n):
        assert torch.equal(y_h[i], y_ref[i]), i
    assert lm.lmoe_device_status(layer.handle) == 0
    # no batches, no tokens, and NULL entries
    lm.lmoe_forward_host_batches(layer.handle, [], [], T)
    lm.lmoe_forward_host_batches(layer.handle, x_h, y_h, 0)
    with pytest.raises(RuntimeError):
        lm.lmoe_forward_host_batches(layer.handle, [x_h[0], None], [y_h[0], y_h[0]], T)
    layer.close()


def test_call_errors_on_device_handle():
    cfg = configs.TINY_F32
    lm = _lmoe()
    h = lm.lmoe_create(lm.config_from(cfg))
    inp = _inputs(cfg)
    y = torch.empty_like(inp["x"])
    with pytest.raises(lm.LmoeError) as e:
        lm.lmoe_forward(h, inp["x"], y, cfg.T)
    assert e.value.code == -3     # not loaded
    lm.lmoe_load_weights(h, inp)
    with pytest.raises(lm.LmoeError) as e:
        lm.lmoe_forward(h, inp["x"], y, cfg.T + 1)
    assert e.value.code == -4     # too many tokens
    with pytest.raises(lm.LmoeError) as e:
        lm.lmoe_forward(h, inp["x"], None, cfg.T)
    assert e.value.code == -2
    lm.lmoe_destroy(h)


def test_misaligned_device_arrays_are_refused_before_any_launch():
    """x or y a few bytes off a 16-byte boundary (2 bytes for bf16, 4 for
    fp32): route and forward return LMOE_ERR_MISALIGNED without launching
    anything, and the same handle then runs a normal forward."""
    lm = _lmoe()
    for cfg in (configs.TINY_F32, MID_PAIR):
        inp = _inputs(cfg)
        x = inp["x"]
        T, d = x.shape
        layer = lm.LatentMoELayer(cfg, inp)
        buf = torch.empty(2 * T * d + 16, dtype=x.dtype, device=x.device)
        x_bad = buf[1:1 + T * d].view(T, d)
        y_bad = buf[T * d + 9:2 * T * d + 9].view(T, d)
        assert x_bad.data_ptr() % 16 != 0 and y_bad.data_ptr() % 16 != 0
        x_bad.copy_(x)
        y = torch.empty_like(x)
        for xx, yy in ((x_bad, y), (x, y_bad)):
            with pytest.raises(lm.LmoeError) as e:
                lm.lmoe_forward(layer.handle, xx, yy, T)
            assert e.value.code == -9
        with pytest.raises(lm.LmoeError) as e:
            lm.lmoe_route(layer.handle, x_bad, T)
        assert e.value.code == -9
        y_ok = layer.forward(x)
        torch.cuda.synchronize()
        assert lm.lmoe_device_status(layer.handle) == 0
        assert torch.isfinite(y_ok.float()).all()
        layer.close()


def test_bounded_wait_reports_timeout_and_context_survives():
    """Failure detection without a GPU fault: a wait that nothing completes
    runs out after 1 ms, the status word reports it, and the next forward on
    the same context is still correct."""
    cfg = configs.TINY_F32
    lm = _lmoe()
    inp = _inputs(cfg)
    layer = lm.LatentMoELayer(cfg, inp)
    assert lm.lmoe_device_status(layer.handle) == 0
    lm.lmoe_selftest_wait_timeout(layer.handle, 1_000_000)
    assert lm.lmoe_device_status(layer.handle) == -6      # LMOE_ERR_DEVICE_TIMEOUT
    assert lm.lmoe_device_status(layer.handle) == 0       # read clears it
    y = layer.forward(inp["x"])
    torch.cuda.synchronize()
    assert lm.lmoe_device_status(layer.handle) == 0
    L = pu.oracle_layer(inp, cfg.k_active)
    x_np = synth.to_numpy(inp["x"])
    y_ref, _, _ = oracle.forward(L, x_np, tokens=np.arange(8))
    assert pu.rel_err(pu.y_to_numpy(y)[:8], y_ref) <= pu.TOL_F32
    with pytest.raises(lm.LmoeError):
        lm.lmoe_selftest_wait_timeout(layer.handle, 0)
    layer.close()
