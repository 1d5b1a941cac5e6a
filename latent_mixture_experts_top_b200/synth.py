"""Seeded synthetic inputs for the LatentMoE layer.

This module only draws random numbers; it holds none of the layer's
arithmetic.  Both the fp64 oracle (tests, bench baseline) and the CUDA library
take their inputs from here.

Recipe (one torch Philox/MT generator seeded with ``seed``, fixed draw order):
  x ~ N(0, x_std) [T][d]; W_r [N'][d]; b_r [N'] ~ N(0, bias_std) (only when the
  workload has a router bias); W_down [l][d]; W_up [d][l]; W_g, W_u [N'][m][l];
  W_o [N'][l][m]; S_g, S_u [n_s][m_s][d]; S_o [n_s][d][m_s]; every weight
  ~ N(0, w_std).  Squared-ReLU workloads draw no W_g / S_g (two-matrix
  experts), so their later draws come earlier in the stream.  Values are
  drawn in float32 and, for bf16 workloads, rounded to bf16 (round to nearest
  even, torch's cast).  Large tensors are drawn in slices along their first
  axis so that the float32 staging stays small; the slicing is part of the
  recipe (same seed + device -> same values).
The router bias is always float32 (the library takes it in float32).
"""
from __future__ import annotations

import torch

from .configs import LayerConfig

ORDER = ("x", "w_router", "b_router", "w_down", "w_up", "w_gate", "w_upx", "w_out",
         "s_gate", "s_up", "s_out")


def _normal(gen, shape, std, dtype, device, slice_elems=1 << 26):
    out = torch.empty(shape, dtype=dtype, device=device)
    if len(shape) == 0 or out.numel() == 0:
        return out
    rows = shape[0]
    per_row = out.numel() // rows
    step = max(1, slice_elems // max(per_row, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        chunk = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                            dtype=torch.float32, device=device)
        if std != 1.0:
            chunk.mul_(std)
        out[r0:r1] = chunk.to(dtype)
    return out


def make_inputs(cfg: LayerConfig, seed: int = 0, device: str | torch.device = "cpu",
                T: int | None = None) -> dict:
    """Draw x and every weight of ``cfg`` on ``device``; see module docstring."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    T = cfg.T if T is None else T
    d, l, m, N = cfg.d, cfg.l, cfg.m, cfg.n_routed
    ns, ms = cfg.n_shared, cfg.m_shared
    w = cfg.w_std
    out = {}
    out["x"] = _normal(gen, (T, d), cfg.x_std, dt, device)
    out["w_router"] = _normal(gen, (N, d), w, dt, device)
    out["b_router"] = (_normal(gen, (N,), cfg.router_bias_std, torch.float32, device)
                       if cfg.has_router_bias else None)
    out["w_down"] = _normal(gen, (l, d), w, dt, device)
    out["w_up"] = _normal(gen, (d, l), w, dt, device)
    relu2 = cfg.activation == "relu2"   # two-matrix experts: no gate weights drawn
    out["w_gate"] = None if relu2 else _normal(gen, (N, m, l), w, dt, device)
    out["w_upx"] = _normal(gen, (N, m, l), w, dt, device)
    out["w_out"] = _normal(gen, (N, l, m), w, dt, device)
    out["s_gate"] = None if relu2 else _normal(gen, (ns, ms, d), w, dt, device)
    out["s_up"] = _normal(gen, (ns, ms, d), w, dt, device)
    out["s_out"] = _normal(gen, (ns, d, ms), w, dt, device)
    return out


def make_cotangent(cfg: LayerConfig, seed: int = 0, device: str | torch.device = "cpu",
                   T: int | None = None) -> torch.Tensor:
    """dy [T][d] ~ N(0, 1) in the layer's element type, from its own generator
    (seed + 1000003), so that x and the weights keep their draws."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 1000003)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    T = cfg.T if T is None else T
    return _normal(gen, (T, cfg.d), 1.0, dt, device)


def to_numpy(t: torch.Tensor):
    """Host numpy copy; bf16 becomes its raw uint16 bit pattern (exact)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()
