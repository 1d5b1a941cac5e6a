"""Parameter, byte and routing-combination counts of standard and latent MoE layers.

TEST INFRASTRUCTURE ONLY (part of the oracle).  Plain integer arithmetic from
the layer's definition; it plays the part of the Latent-MoE README's
``cost_summary()`` (README, "Usage": asymptotic cost quantities).  The paper's
Table 1 itself is not on the pages, so the counts are rebuilt from the layer's
shapes and pinned by the figures the pages print:

* "LatentMoE Explained", Figure 1 (22.0M per d-expert), Figure 9 (5.5M per
  latent expert), Figure 11 (132 MB per token in FP8), Figure 12 (an FP4
  value out and a BF16 value back per coordinate), Figure 13 (60 / 55 / 15 KB
  all-to-all, 121 / 33 MB), and the paragraphs after the LatentMoE code module
  (2,862.6M vs 2,871.0M per layer; 176.2M / 184.5M / 85.5M active);
* "Shaping Latent MoE", Tables 1, 4 and 6 (iso-parameter shapes).

``n_mats`` is 2 for the squared-ReLU expert the article's code uses and 3 for
a SwiGLU expert.  The router is counted only where ``include_router`` is set.
"""
from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass(frozen=True)
class LayerShape:
    d: int                 # model width
    m: int                 # expert intermediate width
    n_experts: int         # routed experts in the layer (N, or N' for latent)
    top_k: int             # active routed experts per token
    n_shared: int          # always-on shared experts
    m_shared: int          # shared-expert intermediate width
    l: int | None = None   # latent width; None = standard (d-space) MoE
    n_mats: int = 2


def expert_params(width: int, m: int, n_mats: int) -> int:
    return n_mats * width * m


def layer_counts(s: LayerShape, include_router: bool = False) -> dict:
    width = s.d if s.l is None else s.l
    per_expert = expert_params(width, s.m, s.n_mats)
    per_shared = expert_params(s.d, s.m_shared, s.n_mats)
    proj = 0 if s.l is None else 2 * s.d * s.l
    router = s.d * s.n_experts if include_router else 0
    routed = s.n_experts * per_expert
    shared = s.n_shared * per_shared
    return {
        "params_per_expert": per_expert,
        "routed_params": routed,
        "shared_params": shared,
        "projection_params": proj,
        "router_params": router,
        "total_params": routed + shared + proj + router,
        "active_routed_params": s.top_k * per_expert,
        "active_params": s.top_k * per_expert + shared + proj + router,
    }


def expert_bytes_per_token(s: LayerShape, bytes_per_weight: float) -> float:
    """Routed expert weight bytes one token streams in one layer."""
    width = s.d if s.l is None else s.l
    return s.top_k * expert_params(width, s.m, s.n_mats) * bytes_per_weight


def all_to_all_bytes_per_token(s: LayerShape, out_bytes: float = 0.5,
                               back_bytes: float = 2.0) -> float:
    """One round trip per selected expert at the routed width (FP4 out, BF16 back)."""
    width = s.d if s.l is None else s.l
    return s.top_k * width * (out_bytes + back_bytes)


def log10_combinations(n: int, k: int) -> float:
    return math.log10(math.comb(n, k))


def layer_flops_per_token(d: int, l: int, m: int, n_routed: int, k_active: int,
                          n_shared: int, m_shared: int) -> int:
    """Algorithmic multiply-add flops (2 per MAC) of one token through the
    SwiGLU LatentMoE layer: router, W_down, K' experts (3 matrices), W_up,
    shared experts (3 matrices)."""
    return 2 * (d * n_routed + 2 * d * l + 3 * k_active * l * m
                + 3 * n_shared * d * m_shared)
