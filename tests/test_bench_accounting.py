"""CPU checks of the work accounting behind bench.py's roofline fractions.

The roofline numerators are algorithmic FLOPs and bytes of the layer as the
pages define it ("LatentMoE Explained", Figures 3, 6, 8, 9: router and W_down
at width d, K' latent experts l -> m -> l, W_up, shared experts at width d).
Here they are held to the oracle's independent per-token count
(oracle.costs.layer_flops_per_token) and to closed forms, so that a dropped
term or a wrong factor in bench.py shows up without a GPU.
"""
from dataclasses import replace

import pytest

import bench
from latent_mixture_experts_top_b200 import configs
from oracle import costs

SWIGLU = [configs.README_ACC, configs.README_EFF, configs.PREFILL, configs.DECODE]
ALL = SWIGLU + [configs.RELU2_95B, configs.DECODE_FP8, configs.RELU2_95B_FP8,
               configs.DECODE_NVFP4, configs.RELU2_95B_NVFP4]


def _shared_gate_up_flops(cfg):
    # the shared experts' gate/up GEMM runs on a side stream, not as a stage
    gu = bench.n_mats(cfg) - 1
    return 2.0 * cfg.T * cfg.d * gu * cfg.n_shared * cfg.m_shared


@pytest.mark.parametrize("cfg", SWIGLU, ids=lambda c: c.name)
def test_layer_flops_match_the_oracle_count(cfg):
    per_token = costs.layer_flops_per_token(cfg.d, cfg.l, cfg.m, cfg.n_routed, cfg.k_active,
                                            cfg.n_shared, cfg.m_shared)
    assert bench.layer_flops(cfg) == cfg.T * per_token


def test_squared_relu_layer_flops_drop_one_matrix_per_expert():
    cfg = configs.RELU2_95B
    swiglu = replace(cfg, activation="swiglu")
    per_token_3 = costs.layer_flops_per_token(cfg.d, cfg.l, cfg.m, cfg.n_routed, cfg.k_active,
                                              cfg.n_shared, cfg.m_shared)
    one_matrix = 2.0 * (cfg.k_active * cfg.l * cfg.m + cfg.n_shared * cfg.d * cfg.m_shared)
    assert bench.layer_flops(swiglu) == cfg.T * per_token_3
    assert bench.layer_flops(cfg) == cfg.T * (per_token_3 - one_matrix)


@pytest.mark.parametrize("cfg", ALL, ids=lambda c: c.name)
def test_stage_flops_add_up_to_the_layer(cfg):
    work = bench.stage_work(cfg)
    staged = sum(w[0] for w in work.values())
    assert bench.shared_gate_up_work(cfg)[0] == _shared_gate_up_flops(cfg)
    assert staged + _shared_gate_up_flops(cfg) == pytest.approx(bench.layer_flops(cfg), rel=1e-12)
    for stage in (1, 2, 3, 6):   # routing, dispatch, permute, combine: intermediates only
        assert work[stage][0] == 0.0 and work[stage][1] == 0.0 and work[stage][2] > 0.0


@pytest.mark.parametrize("cfg", ALL, ids=lambda c: c.name)
def test_stage_bytes_add_up_to_the_layer(cfg):
    """Algorithmic bytes are touched weights + x + y only: summed over the
    stages and the side-stream shared GEMM they give layer_bytes exactly."""
    for touched in (None, 37):
        work = bench.stage_work(cfg, touched=touched)
        staged = sum(w[1] for w in work.values()) + bench.shared_gate_up_work(cfg)[1]
        ids = None if touched is None else __import__("numpy").arange(touched)
        assert staged == pytest.approx(bench.layer_bytes(cfg, ids), rel=1e-12)


def test_readme_acc_figures_quoted_in_the_design_notes():
    cfg = configs.README_ACC
    work = bench.stage_work(cfg)
    assert round(bench.layer_flops(cfg) / 1e9, 1) == 588.4
    assert round(work[4][0] / 1e9, 1) == 283.5      # expert gate/up GEMM
    assert round(work[5][0] / 1e9, 1) == 141.7      # expert down GEMM
    # gate/up: algorithmic bytes are the 256 experts' gate/up weights; the
    # permuted z in and H out are intermediates
    TK = cfg.T * cfg.k_active
    assert work[4][1] == 2 * 256 * 2 * cfg.m * cfg.l
    assert round(work[4][1] / 1e6, 1) == 738.2
    assert work[4][2] == 2 * TK * cfg.l + 2 * TK * cfg.m
    # so the stage is tensor-bound at the measured peaks
    peaks = {"bf16_tflops": 1640.9, "hbm_gbs": 6441.9}
    assert bench.stage_bound(work[4][0], work[4][1], peaks) == "tensor"


def test_touched_experts_scale_only_the_weight_bytes():
    cfg = configs.DECODE
    full, part = bench.stage_work(cfg), bench.stage_work(cfg, touched=100)
    per_expert_gu = 2.0 * 2 * cfg.m * cfg.l
    assert full[4][0] == part[4][0]
    assert full[4][1] - part[4][1] == pytest.approx((cfg.n_routed - 100) * per_expert_gu)


def test_e4m3_experts_halve_the_routed_weight_bytes():
    bf, f8 = configs.DECODE, configs.DECODE_FP8
    wb, w8 = bench.stage_work(bf), bench.stage_work(f8)
    per_expert_bf16 = 2.0 * 2 * bf.m * bf.l
    assert wb[4][1] - w8[4][1] == pytest.approx(bf.n_routed * per_expert_bf16 / 2)
    assert bench.layer_bytes(bf) - bench.layer_bytes(f8) == pytest.approx(
        bf.n_routed * 3 * bf.l * bf.m * 1.0)


def test_stage_bound_picks_the_slower_roof():
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 1000.0}
    assert bench.stage_bound(2e12, 1e9, peaks) == "tensor"    # 2 ms of math, 1 ms of bytes
    assert bench.stage_bound(1e12, 2e9, peaks) == "hbm"
    assert bench.stage_bound(0.0, 0.0, peaks) == "hbm"     # a memory-only helper


def test_nvfp4_experts_take_half_a_byte_and_a_sixteenth_per_weight():
    """E2M1 codes (4 bits) plus one E4M3 block scale per 16 weights."""
    bf, f4 = configs.DECODE, configs.DECODE_NVFP4
    per_weight = 0.5 + 1.0 / 16
    assert bench.layer_bytes(bf) - bench.layer_bytes(f4) == pytest.approx(
        bf.n_routed * 3 * bf.l * bf.m * (2.0 - per_weight))
    w4 = bench.stage_work(f4)
    assert w4[4][1] == pytest.approx(f4.n_routed * 2 * f4.m * f4.l * per_weight)
