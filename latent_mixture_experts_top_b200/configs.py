"""The five synthetic LatentMoE layer workloads and the layer-shape record.

The record mirrors ``LatentMoEConfig(d, m, n_experts, top_k, alpha, n_shared,
variant)`` of the Latent-MoE README ("Usage"), plus the fields the five
workloads need beyond it: the shared-expert width, explicit N'/K' overrides
(the shipped Nemotron-3-Super-like shape uses K'=22, which is not alpha*K --
"LatentMoE Explained", the paragraph naming Nemotron 3 Super), a router bias
switch, the element type and the token count.

Derived sizes follow the README's two variants: l = d / alpha, N' = alpha*N,
K' = alpha*K for "acc" and K' = K for "eff".
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int                    # tokens in one forward call
    d: int                    # model width
    m: int                    # routed expert intermediate width
    n_experts: int            # base N
    top_k: int                # base K
    alpha: int                # compression factor, l = d / alpha
    n_shared: int             # shared SwiGLU experts at width d
    m_shared: int             # their intermediate width
    variant: str = "acc"      # "acc" | "eff"
    dtype: str = "bf16"       # "bf16" | "f32"
    n_routed_override: int = 0
    top_k_override: int = 0
    router_bias_std: float = 0.0   # > 0: per-expert router bias ~ N(0, std)
    activation: str = "swiglu"     # "swiglu" (3 matrices) | "relu2" (2 matrices)
    weights: str = "bf16"          # routed experts: "bf16" | "fp8" (E4M3, row scales) | "nvfp4"
    x_std: float = 1.0
    w_std: float = 0.02

    @property
    def l(self) -> int:
        return self.d // self.alpha

    @property
    def n_routed(self) -> int:
        return self.n_routed_override or self.alpha * self.n_experts

    @property
    def k_active(self) -> int:
        if self.top_k_override:
            return self.top_k_override
        return self.alpha * self.top_k if self.variant == "acc" else self.top_k

    @property
    def has_router_bias(self) -> bool:
        return self.router_bias_std > 0.0

    def with_tokens(self, T: int) -> "LayerConfig":
        return replace(self, T=T)


TINY_F32 = LayerConfig("tiny_f32_T64_d256_l128_N16_K4", T=64, d=256, m=256,
                       n_experts=8, top_k=2, alpha=2, n_shared=1, m_shared=256,
                       variant="acc", dtype="f32")
README_ACC = LayerConfig("readme_acc_T4096_d2048_l512_m1408_N256_K24", T=4096, d=2048,
                         m=1408, n_experts=64, top_k=6, alpha=4, n_shared=2,
                         m_shared=1408, variant="acc")
README_EFF = replace(README_ACC, name="readme_eff_T4096_d2048_l512_m1408_N256_K6",
                     variant="eff")
PREFILL = LayerConfig("prefill_T16384_d4096_l1024_m2048_N512_K22_bias", T=16384,
                      d=4096, m=2048, n_experts=128, top_k=6, alpha=4, n_shared=1,
                      m_shared=4096, variant="acc", n_routed_override=512,
                      top_k_override=22, router_bias_std=0.5)
DECODE = replace(PREFILL, name="decode_T64_d4096_l1024_m2048_N512_K22", T=64,
                 router_bias_std=0.0)

# Squared-ReLU experts ("LatentMoE Explained", the Expert class and the 95B
# running example: d=4096, l=1024, m=2688, N=128 -> N'=512, K=6 -> K'=24, two
# shared experts of width m).
TINY_RELU2_F32 = replace(TINY_F32, name="tiny_relu2_f32_T64_d256_l128_N16_K4",
                         activation="relu2")
RELU2_95B = LayerConfig("relu2_95b_T1024_d4096_l1024_m2688_N512_K24", T=1024, d=4096,
                        m=2688, n_experts=128, top_k=6, alpha=4, n_shared=2, m_shared=2688,
                        variant="acc", activation="relu2")

# The decode workload with E4M3 routed-expert weights ("LatentMoE Explained":
# an expert is about 22 MB in FP8), and the 95B squared-ReLU shape likewise.
DECODE_FP8 = replace(DECODE, name="decode_fp8_T64_d4096_l1024_m2048_N512_K22", weights="fp8")
RELU2_95B_FP8 = replace(RELU2_95B, name="relu2_95b_fp8_T1024_d4096_l1024_m2688_N512_K24",
                        weights="fp8")
# The same two with NVFP4 routed experts ("LatentMoE Explained": the shipped
# models were pretrained in NVFP4): E2M1 codes, an E4M3 scale per 16 elements
# and a power-of-two scale per row, on weights and activations alike.
DECODE_NVFP4 = replace(DECODE, name="decode_nvfp4_T64_d4096_l1024_m2048_N512_K22",
                       weights="nvfp4")
RELU2_95B_NVFP4 = replace(RELU2_95B, name="relu2_95b_nvfp4_T1024_d4096_l1024_m2688_N512_K24",
                          weights="nvfp4")

CONFIGS = [TINY_F32, README_ACC, README_EFF, PREFILL, DECODE]
EXTRA_CONFIGS = [TINY_RELU2_F32, RELU2_95B, DECODE_FP8, RELU2_95B_FP8, DECODE_NVFP4,
                 RELU2_95B_NVFP4]
BY_NAME = {c.name: c for c in CONFIGS + EXTRA_CONFIGS}
