"""GPU checks of the NVFP4 routed experts (LMOE_WEIGHTS_NVFP4): both operands
of the expert GEMMs as E2M1 codes with an E4M3 scale per 16 elements and a
power-of-two scale per row; the GEMMs run tcgen05 kind::mxf4nvf4.

1. The library's packed weight codes, block scales and row scales, decoded
   on the host from the two formats' definitions, equal the oracle's NVFP4
   quantisation of the same bf16 weights bit for bit (the rule leaves one
   right answer: the division, reciprocal and product are IEEE single
   precision, both roundings to nearest even).
2. The same for the activation rows the library quantises on the fly (each
   expert input row z in dispatch order, each hidden row h), taken from the
   library's own bf16 z and H: the quantiser sees the same values on both
   sides; the block scales sit in the per-tile layout the MMA reads.
3. The layer output matches the fp64 oracle run with the dequantised expert
   weights, every other weight widened from bf16, and act_fp4 with act_bf16
   (z and h rounded to bf16, then quantised per row, as the library holds
   them).  Tolerance 2e-2, the bf16 mode's.  The mid-size cases have
   m = 384, a ragged last 256-element K-block for the down GEMM.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle
from latent_mixture_experts_top_b200 import configs, synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

MID_NVFP4 = configs.LayerConfig("mid_nvfp4_T300_d512_l256_m384_N32_K8", T=300, d=512, m=384,
                                n_experts=16, top_k=4, alpha=2, n_shared=1, m_shared=256,
                                variant="acc", weights="nvfp4")
MID_RELU2_NVFP4 = replace(MID_NVFP4, name="mid_relu2_nvfp4_T300_d512_l256_m384_N32_K8",
                          activation="relu2")
ATOM = 512


def _e2m1_table():
    """The 16 E2M1 codes: sign bit 3, exponent bits 2..1 (bias 1), mantissa
    bit 0; exponent 0 is subnormal (0 or 0.5)."""
    t = np.empty(16)
    for c in range(16):
        sgn = -1.0 if c & 8 else 1.0
        e, m = (c >> 1) & 3, c & 1
        t[c] = sgn * (m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2))
    return t


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


E2M1, E4M3 = _e2m1_table(), _e4m3_table()


def _unpack(codes):
    """bytes [..., n] -> E2M1 values [..., 2n] (element 2i in the low nibble)."""
    lo, hi = codes & 15, codes >> 4
    return E2M1[np.stack([lo, hi], axis=-1).reshape(*codes.shape[:-1], 2 * codes.shape[-1])]


def _weights_decoded(codes, sf, groups, rows, cols):
    """Tiled codes [g][nt][nkb][256][128] and scales [g][nt][nkb][2][4][512]
    -> values [g][rows][cols] and block scales [g][rows][cols / 16]."""
    nt, nkb = (rows + 255) // 256, (cols + 255) // 256
    c = codes.reshape(groups, nt, nkb, 256, 128)
    v = _unpack(c).transpose(0, 1, 3, 2, 4).reshape(groups, nt * 256, nkb * 256)
    s = sf.reshape(groups, nt, nkb, 2, 4, 32, 4, 4)        # [.., rb, k, r0, r1, q]
    # row rr = 128 rb + 32 r1 + r0, block = 16 kb + 4 k + q
    s = s.transpose(0, 1, 3, 6, 5, 2, 4, 7).reshape(groups, nt * 256, nkb * 16)
    return v[:, :rows, :cols], E4M3[s[:, :rows, :cols // 16]]


def _tile_rows(offsets, n_routed):
    """(m-tile, row within the tile) of every dispatch row, from the offsets:
    each expert's rows split into 128-row tiles, in expert order."""
    TK = int(offsets[n_routed])
    mt_of, i_of = np.empty(TK, np.int64), np.empty(TK, np.int64)
    mt = 0
    for e in range(n_routed):
        a, b = int(offsets[e]), int(offsets[e + 1])
        for r0 in range(a, b, 128):
            r1 = min(b, r0 + 128)
            mt_of[r0:r1] = mt
            i_of[r0:r1] = np.arange(r1 - r0)
            mt += 1
    return mt_of, i_of


def _act_block_scales(sf, mt_of, i_of, cols):
    nkb, nblk = (cols + 255) // 256, cols // 16
    blk = np.arange(nblk)
    kb, k, q = blk // 16, (blk % 16) // 4, blk % 4
    idx = (mt_of[:, None] * nkb * 4 * ATOM + (kb * 4 + k)[None, :] * ATOM
           + 16 * (i_of[:, None] % 32) + 4 * (i_of[:, None] // 32) + q[None, :])
    return E4M3[sf[idx]]


def _widen(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _lmoe():
    from latent_mixture_experts_top_b200 import lmoe
    return lmoe


@pytest.mark.parametrize("cfg", [MID_NVFP4, MID_RELU2_NVFP4], ids=lambda c: c.name)
def test_weight_codes_and_scales_equal_the_oracle_quantisation(cfg):
    lm = _lmoe()
    inp = synth.make_inputs(cfg, 0, "cuda")
    layer = lm.LatentMoELayer(cfg, inp)
    N, l, m = cfg.n_routed, cfg.l, cfg.m
    relu2 = cfg.activation == "relu2"
    gu_rows = m if relu2 else 2 * m
    grab = lambda which: layer.debug_tensor(which, torch.uint8,
                                            (lm.lmoe_debug_buffer(layer.handle, which)[1],))
    c_gu, c_o = grab(12).cpu().numpy(), grab(14).cpu().numpy()
    f_gu, f_o = grab(20).cpu().numpy(), grab(21).cpu().numpy()
    s_gu = layer.debug_tensor(13, torch.float32, (N, gu_rows)).cpu().numpy().astype(np.float64)
    s_o = layer.debug_tensor(15, torch.float32, (N, l)).cpu().numpy().astype(np.float64)
    v_gu, b_gu = _weights_decoded(c_gu, f_gu, N, gu_rows, l)
    v_o, b_o = _weights_decoded(c_o, f_o, N, l, m)
    n = {k: synth.to_numpy(v) for k, v in inp.items() if v is not None}
    wo_q, wo_s, wo_b = oracle.nvfp4_rows(n["w_out"])
    np.testing.assert_array_equal(v_o * np.repeat(b_o, 16, axis=2) * s_o[:, :, None], wo_q)
    np.testing.assert_array_equal(b_o, wo_b)
    np.testing.assert_array_equal(s_o.reshape(-1), wo_s)
    wu_q, wu_s, wu_b = oracle.nvfp4_rows(n["w_upx"])
    got = v_gu * np.repeat(b_gu, 16, axis=2) * s_gu[:, :, None]
    if relu2:
        np.testing.assert_array_equal(got, wu_q)
        np.testing.assert_array_equal(b_gu, wu_b)
    else:
        wg_q, _, wg_b = oracle.nvfp4_rows(n["w_gate"])
        r = np.arange(gu_rows)
        blk, i = r // 256, r % 256
        unit = 128 * blk + (i % 128)
        gate = (i < 128)[None, :, None]
        np.testing.assert_array_equal(got, np.where(gate, wg_q[:, unit, :], wu_q[:, unit, :]))
        np.testing.assert_array_equal(b_gu, np.where(gate, wg_b[:, unit, :], wu_b[:, unit, :]))
    layer.close()


@pytest.mark.parametrize("cfg", [MID_NVFP4, MID_RELU2_NVFP4], ids=lambda c: c.name)
def test_activation_codes_equal_the_oracle_quantisation(cfg):
    """The NVFP4 rows the expert GEMMs read, from the library's own z (in
    dispatch order) and hidden H: codes, block scales (in the per-tile
    layout) and row scales bit for bit."""
    lm = _lmoe()
    inp = synth.make_inputs(cfg, 0, "cuda")
    layer = lm.LatentMoELayer(cfg, inp)
    layer.forward(inp["x"])
    torch.cuda.synchronize()
    T, K, l, m, N = cfg.T, cfg.k_active, cfg.l, cfg.m, cfg.n_routed
    TK = T * K
    u16 = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    z = u16(layer.debug_tensor(1, torch.bfloat16, (T, l)))
    perm = layer.debug_tensor(9, torch.int32, (TK,)).cpu().numpy()
    offsets = layer.debug_tensor(8, torch.int32, (N + 1,)).cpu().numpy()
    H = u16(layer.debug_tensor(3, torch.bfloat16, (TK, m)))
    mt_of, i_of = _tile_rows(offsets, N)
    grab = lambda which: layer.debug_tensor(which, torch.uint8,
                                            (lm.lmoe_debug_buffer(layer.handle, which)[1],))
    for rows, cols, cw, sw, fw in ((z[perm // K], l, 16, 17, 22), (H, m, 18, 19, 23)):
        vals = _unpack(grab(cw).cpu().numpy()[:TK * cols // 2].reshape(TK, cols // 2))
        rs = layer.debug_tensor(sw, torch.float32, (TK,)).cpu().numpy().astype(np.float64)
        bs = _act_block_scales(grab(fw).cpu().numpy(), mt_of, i_of, cols)
        ref_q, ref_s, ref_b = oracle.nvfp4_rows(rows)
        np.testing.assert_array_equal(bs, ref_b)
        np.testing.assert_array_equal(rs, ref_s)
        np.testing.assert_array_equal(vals * np.repeat(bs, 16, axis=1) * rs[:, None], ref_q)
    layer.close()


def _nvfp4_layer_case(cfg, n_sample):
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
            wide[k] = oracle.nvfp4_rows(n[k])[0]
    bias = None if n["b_router"] is None else n["b_router"].astype(np.float64)
    L = oracle.Layer(w_router=wide["w_router"], b_router=bias, w_down=wide["w_down"],
                     w_up=wide["w_up"], w_gate=wide["w_gate"], w_upx=wide["w_upx"],
                     w_out=wide["w_out"], s_gate=wide["s_gate"], s_up=wide["s_up"],
                     s_out=wide["s_out"], k_active=cfg.k_active, activation=cfg.activation,
                     act_fp4=True, act_bf16=True)
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


def test_nvfp4_mid_swiglu_all_tokens():
    _nvfp4_layer_case(MID_NVFP4, 10 ** 9)


def test_nvfp4_mid_relu2_all_tokens():
    _nvfp4_layer_case(MID_RELU2_NVFP4, 10 ** 9)


def test_nvfp4_decode_workload():
    _nvfp4_layer_case(configs.DECODE_NVFP4, 10 ** 9)


def test_nvfp4_relu2_95b_shape():
    _nvfp4_layer_case(configs.RELU2_95B_NVFP4, 48)


def test_nvfp4_with_training_or_expert_parallelism_is_refused():
    lm = _lmoe()
    with pytest.raises(lm.LmoeError) as e:
        lm.lmoe_create(lm.config_from(MID_NVFP4, training=True))
    assert e.value.code == -7
