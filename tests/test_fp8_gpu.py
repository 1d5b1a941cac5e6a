"""GPU checks of the E4M3 routed experts (LMOE_WEIGHTS_FP8): both operands
of the expert GEMMs in E4M3 with power-of-two row scales.

1. The library's weight codes and row scales, decoded on the host from the
   E4M3 definition, equal the oracle's quantisation of the same bf16 weights
   bit for bit (both round W / s to nearest-even with saturation, s a power
   of two, so there is one right answer).
2. The same holds for the activation rows the library quantises on the fly
   (each expert input row z, each hidden row h), taken from the library's
   own bf16 z and H: the quantiser sees the same values on both sides.
3. The layer output matches the fp64 oracle run with the dequantised expert
   weights, every other weight widened from bf16, and act_fp8 with act_bf16
   (z and h rounded to bf16, as the library holds them, then quantised per
   row); tolerance 2e-2, the bf16 mode's.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from latent_mixture_experts_top_b200 import configs, synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

MID_FP8 = configs.LayerConfig("mid_fp8_T300_d512_l256_m256_N32_K8", T=300, d=512, m=256,
                              n_experts=16, top_k=4, alpha=2, n_shared=1, m_shared=256,
                              variant="acc", weights="fp8")
MID_RELU2_FP8 = replace(MID_FP8, name="mid_relu2_fp8_T300_d512_l256_m384_N32_K8", m=384,
                        m_shared=384, activation="relu2")


def _e4m3_table():
    t = np.empty(256)
    for code in range(256):
        sgn = -1.0 if code & 0x80 else 1.0
        e, m = (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            t[code] = np.nan
        elif e == 0:
            t[code] = sgn * m / 8 * 2.0 ** -6
        else:
            t[code] = sgn * 2.0 ** (e - 7) * (1 + m / 8)
    return t


def _detile(codes, groups, rows, cols):
    nt, kbc = (rows + 255) // 256, cols // 128
    a = codes.reshape(groups, nt, kbc, 256, 128).transpose(0, 1, 3, 2, 4)
    return a.reshape(groups, nt * 256, cols)[:, :rows]


def _widen(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _lmoe():
    from latent_mixture_experts_top_b200 import lmoe
    return lmoe


@pytest.mark.parametrize("cfg", [MID_FP8, MID_RELU2_FP8], ids=lambda c: c.name)
def test_codes_and_scales_equal_the_oracle_quantisation(cfg):
    lm = _lmoe()
    inp = synth.make_inputs(cfg, 0, "cuda")
    layer = lm.LatentMoELayer(cfg, inp)
    N, l, m = cfg.n_routed, cfg.l, cfg.m
    relu2 = cfg.activation == "relu2"
    gu_rows = m if relu2 else 2 * m
    n12 = lm.lmoe_debug_buffer(layer.handle, 12)[1]
    n14 = lm.lmoe_debug_buffer(layer.handle, 14)[1]
    c_gu = layer.debug_tensor(12, torch.uint8, (n12,)).cpu().numpy()
    s_gu = layer.debug_tensor(13, torch.float32, (N, gu_rows)).cpu().numpy().astype(np.float64)
    c_o = layer.debug_tensor(14, torch.uint8, (n14,)).cpu().numpy()
    s_o = layer.debug_tensor(15, torch.float32, (N, l)).cpu().numpy().astype(np.float64)
    table = _e4m3_table()
    w_gu = table[_detile(c_gu, N, gu_rows, l)] * s_gu[:, :, None]
    w_o = table[_detile(c_o, N, l, m)] * s_o[:, :, None]
    n = {k: synth.to_numpy(v) for k, v in inp.items() if v is not None}
    wu_q, wu_s = oracle.fp8_rows(n["w_upx"])
    wo_q, wo_s = oracle.fp8_rows(n["w_out"])
    np.testing.assert_array_equal(w_o, wo_q)
    np.testing.assert_array_equal(s_o.reshape(-1), wo_s)
    if relu2:
        np.testing.assert_array_equal(w_gu, wu_q)
    else:
        wg_q, _ = oracle.fp8_rows(n["w_gate"])
        r = np.arange(gu_rows)
        blk, i = r // 256, r % 256
        unit = 128 * blk + (i % 128)
        expect = np.where((i < 128)[None, :, None], wg_q[:, unit, :], wu_q[:, unit, :])
        np.testing.assert_array_equal(w_gu, expect)
    layer.close()


def _fp8_layer_case(cfg, n_sample):
    lm = _lmoe()
    inp = synth.make_inputs(cfg, 0, "cuda")
    layer = lm.LatentMoELayer(cfg, inp)
    x = inp["x"]
    y = layer.forward(x)
    ids, gates, offsets, perm = layer.route(x)
    torch.cuda.synchronize()
    assert lm.lmoe_device_status(layer.handle) == 0
    n = {k: (None if v is None else synth.to_numpy(v)) for k, v in inp.items()}
    wide = {k: (None if v is None else _widen(v)) for k, v in n.items() if k != "b_router"}
    for k in ("w_gate", "w_upx", "w_out"):
        if n[k] is not None:
            wide[k] = oracle.fp8_rows(n[k])[0]
    bias = None if n["b_router"] is None else n["b_router"].astype(np.float64)
    L = oracle.Layer(w_router=wide["w_router"], b_router=bias, w_down=wide["w_down"],
                     w_up=wide["w_up"], w_gate=wide["w_gate"], w_upx=wide["w_upx"],
                     w_out=wide["w_out"], s_gate=wide["s_gate"], s_up=wide["s_up"],
                     s_out=wide["s_out"], k_active=cfg.k_active, activation=cfg.activation,
                     act_fp8=True, act_bf16=True)
    x64 = wide["x"]
    ids_g = ids.cpu().numpy()
    s_ref = oracle.router_logits(L, x64)
    near, flipped = pu.check_routing(ids_g, gates.cpu().numpy(), s_ref, cfg.k_active)
    tok = pu.sample_tokens(cfg.T, n_sample) if n_sample < cfg.T else np.arange(cfg.T)
    y_ref = pu.reference_y(L, x64, tok, ids_g, flipped)
    err = pu.rel_err(pu.y_to_numpy(y)[tok], y_ref)
    print(f"{cfg.name}: rel err {err:.3e} (tol {pu.TOL_BF16}), near-tie {near.sum()}, "
          f"flipped {flipped.sum()}")
    layer.close()
    assert err <= pu.TOL_BF16


@pytest.mark.parametrize("cfg", [MID_FP8, MID_RELU2_FP8], ids=lambda c: c.name)
def test_activation_codes_equal_the_oracle_quantisation(cfg):
    """The E4M3 rows the expert GEMMs read, from the library's own z (in
    dispatch order) and hidden H: codes and row scales bit for bit."""
    lm = _lmoe()
    inp = synth.make_inputs(cfg, 0, "cuda")
    layer = lm.LatentMoELayer(cfg, inp)
    layer.forward(inp["x"])
    torch.cuda.synchronize()
    T, K, l, m = cfg.T, cfg.k_active, cfg.l, cfg.m
    TK = T * K
    table = _e4m3_table()
    z = layer.debug_tensor(1, torch.bfloat16, (T, l)).view(torch.int16).cpu().numpy().view(np.uint16)
    perm = layer.debug_tensor(9, torch.int32, (TK,)).cpu().numpy()
    H = layer.debug_tensor(3, torch.bfloat16, (TK, m)).view(torch.int16).cpu().numpy().view(np.uint16)
    zq = table[layer.debug_tensor(16, torch.uint8, (TK, l)).cpu().numpy()]
    zs = layer.debug_tensor(17, torch.float32, (TK,)).cpu().numpy().astype(np.float64)
    hq = table[layer.debug_tensor(18, torch.uint8, (TK, m)).cpu().numpy()]
    hs = layer.debug_tensor(19, torch.float32, (TK,)).cpu().numpy().astype(np.float64)
    zref, zref_s = oracle.fp8_rows(z[perm // K])
    np.testing.assert_array_equal(zq * zs[:, None], zref)
    np.testing.assert_array_equal(zs, zref_s)
    href, href_s = oracle.fp8_rows(H)
    np.testing.assert_array_equal(hq * hs[:, None], href)
    np.testing.assert_array_equal(hs, href_s)
    layer.close()


def test_fp8_mid_swiglu_all_tokens():
    _fp8_layer_case(MID_FP8, 10 ** 9)


def test_fp8_mid_relu2_all_tokens():
    _fp8_layer_case(MID_RELU2_FP8, 10 ** 9)


def test_fp8_decode_workload():
    _fp8_layer_case(configs.DECODE_FP8, 10 ** 9)


def test_fp8_relu2_95b_shape():
    _fp8_layer_case(configs.RELU2_95B_FP8, 48)


def test_fp8_with_training_is_refused():
    lm = _lmoe()
    cfg = MID_FP8
    with pytest.raises(lm.LmoeError) as e:
        lm.lmoe_create(lm.config_from(cfg, training=True))
    assert e.value.code == -7
