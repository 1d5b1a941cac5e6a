"""Pins of the oracle's cost counts by the figures the pages print.

"LatentMoE Explained" (95B running example: d=4096, l=1024, m=2688, N=128,
K=6, two shared experts, squared-ReLU experts with two matrices, router not
counted): Figure 1, Figure 9, Figure 11, Figure 13 and the paragraphs after the
LatentMoE code module and the combinatorics paragraph.  "Shaping Latent MoE":
Tables 1, 4 and 6 (SwiGLU experts, three matrices).
"""
import pytest

from oracle import costs

BASE = costs.LayerShape(d=4096, m=2688, n_experts=128, top_k=6, n_shared=2, m_shared=2688)
ACC = costs.LayerShape(d=4096, m=2688, n_experts=512, top_k=24, n_shared=2,
                       m_shared=2688, l=1024)
EFF = costs.LayerShape(d=4096, m=2688, n_experts=512, top_k=6, n_shared=2,
                       m_shared=2688, l=1024)
SUPER = costs.LayerShape(d=4096, m=2688, n_experts=512, top_k=22, n_shared=2,
                         m_shared=2688, l=1024)


def M(x):
    return round(x / 1e6, 1)


def test_expert_sizes():
    assert M(costs.expert_params(4096, 2688, 2)) == 22.0      # Figure 1
    assert M(costs.expert_params(1024, 2688, 2)) == 5.5       # Figure 9
    assert round(costs.expert_params(1024, 2688, 1) / 1e6, 2) == 2.75


def test_layer_totals_and_active():
    b, a, e = costs.layer_counts(BASE), costs.layer_counts(ACC), costs.layer_counts(EFF)
    assert M(b["total_params"]) == 2862.6
    assert M(a["total_params"]) == 2871.0
    assert M(a["total_params"] - b["total_params"]) == 8.4
    assert a["projection_params"] == 2 * 4096 * 1024
    assert round(100 * a["projection_params"] / a["routed_params"], 1) == 0.3
    assert round(b["routed_params"] / 1e9, 2) == 2.82 == round(a["routed_params"] / 1e9, 2)
    assert M(b["active_params"]) == 176.2
    assert M(a["active_params"]) == 184.5
    assert M(e["active_params"]) == 85.5
    assert M(b["active_routed_params"]) == 132.1
    assert round(4096 * 512 / 1e6, 1) == 2.1                 # router, "2.1 million"


def test_bytes_per_token():
    mb = lambda s: round(costs.expert_bytes_per_token(s, 1.0) / 1e6)
    assert mb(BASE) == 132 and mb(ACC) == 132 and mb(SUPER) == 121 and mb(EFF) == 33
    t = costs.expert_bytes_per_token(BASE, 1.0) / 8e12
    assert round(t * 1e6, 1) == 16.5                           # microseconds at 8 TB/s
    assert round(32 * costs.expert_bytes_per_token(EFF, 1.0) / 1e9, 1) == 1.1
    assert round(32 * costs.expert_bytes_per_token(BASE, 1.0) / 1e9, 1) == 4.2
    assert round(32 * costs.expert_bytes_per_token(EFF, 1.0) / 8e12 * 1e3, 2) == 0.13
    assert round(32 * costs.expert_bytes_per_token(BASE, 1.0) / 8e12 * 1e3, 2) == 0.53
    kb = lambda s: costs.all_to_all_bytes_per_token(s) / 1024
    assert kb(BASE) == 60 and kb(ACC) == 60 and kb(SUPER) == 55 and kb(EFF) == 15
    assert 4096 * 0.5 / 1024 == 2 and 4096 * 2 / 1024 == 8    # Figure 12: 2 KB out, 8 KB back


def test_combinations():
    assert round(costs.log10_combinations(128, 6), 1) == 9.7
    assert round(10 ** costs.log10_combinations(128, 6) / 1e9, 1) == 5.4
    assert round(costs.log10_combinations(512, 24)) == 41
    assert round(4 * costs.log10_combinations(128, 6), 1) == 38.9


@pytest.mark.parametrize("shallow,deep,d", [((352, 448, 640, 20, 490), (512, 440, 448, 14, 448), 1024)])
def test_shaping_table1_iso_parameter(shallow, deep, d):
    def shape(c):
        l, m, N, K, ms = c
        return costs.LayerShape(d=d, m=m, n_experts=N, top_k=K, n_shared=1, m_shared=ms,
                                l=l, n_mats=3)
    a = costs.layer_counts(shape(shallow), include_router=True)
    b = costs.layer_counts(shape(deep), include_router=True)
    assert a["routed_params"] == b["routed_params"] == 302_776_320
    assert a["active_routed_params"] == b["active_routed_params"] == 9_461_760
    assert abs(a["total_params"] - b["total_params"]) == 2048


def test_shaping_table4_and_table6():
    # Table 4: N' l = N d and K' l = K d for the uniform LatentMoE models
    for d, N, K, rows in [(1280, 256, 8, [(320, 1024, 32), (640, 512, 16)]),
                          (1024, 256, 8, [(256, 1024, 32)])]:
        for l, Np, Kp in rows:
            assert Np * l == N * d and Kp * l == K * d
    # Table 6: per-expert size l*m is held fixed within each sweep (two exceptions)
    s8 = [(320, 2048), (512, 1280), (640, 1024), (1024, 640)]
    s3 = [(256, 1536), (512, 768), (768, 512), (1024, 384)]
    assert {l * m for l, m in s8} == {655_360}
    assert {l * m for l, m in s3} == {393_216}
    assert 816 * 800 != 655_360 and 640 * 616 != 393_216
