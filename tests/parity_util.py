"""Shared helpers of the GPU parity tests: run the CUDA library and the fp64
oracle on the same seeded inputs and compare.

Comparison rules (tolerances stated where they are used):
* routing: the oracle's fp64 logits decide.  A token whose K'-th and
  (K'+1)-th largest logits are within NEAR_TIE of each other is "near-tie":
  several selections are correct up to rounding, so there the GPU's set must
  be a correct top-K' of the fp64 logits (up to ORDER_TOL) with every
  differing expert inside the tie band.  Everywhere else the selected set must be identical, and the slot
  order identical wherever consecutive selected logits differ by more than
  ORDER_TOL; within ORDER_TOL the GPU order must still be non-increasing in
  the oracle's logits up to ORDER_TOL.
* dispatch: offsets / perm must equal the oracle's dispatch of the GPU's own
  ids exactly (integer work, unique result).
* y: max|y - y_ref| / max|y_ref| over the compared tokens, where y_ref uses
  the oracle's routing for tokens whose selection matches and the GPU's ids
  (oracle forward_given_ids) for near-tie tokens that flipped.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from latent_mixture_experts_top_b200 import synth

NEAR_TIE = 1e-3      # K'-th / (K'+1)-th logit gap below which selection is not unique
ORDER_TOL = 1e-4     # fp32-accumulated logits differ from fp64 by ~1e-6; 100x margin
TOL_F32 = 1e-5
TOL_BF16 = 2e-2


def oracle_layer(inputs: dict, k_active: int, activation: str = "swiglu") -> oracle.Layer:
    n = {k: (None if v is None else synth.to_numpy(v)) for k, v in inputs.items()}
    bias = None if n["b_router"] is None else n["b_router"].astype(np.float64)
    return oracle.Layer(w_router=n["w_router"], b_router=bias, w_down=n["w_down"],
                        w_up=n["w_up"], w_gate=n["w_gate"], w_upx=n["w_upx"],
                        w_out=n["w_out"], s_gate=n["s_gate"], s_up=n["s_up"],
                        s_out=n["s_out"], k_active=k_active, activation=activation)


def boundary_gap(s_ref: np.ndarray, K: int) -> np.ndarray:
    N = s_ref.shape[1]
    if K >= N:
        return np.full(s_ref.shape[0], np.inf)
    part = -np.sort(-s_ref, axis=1)
    return part[:, K - 1] - part[:, K]


def check_routing(ids_gpu: np.ndarray, gates_gpu: np.ndarray, s_ref: np.ndarray, K: int):
    """Returns (near mask, flipped mask) after asserting the rules above.

    Where the GPU's set differs from the oracle's (possible only on near-tie
    tokens), the GPU's set must itself be a correct top-K' of the fp64
    logits: its smallest selected logit is not below the largest unselected
    one (up to ORDER_TOL, the fp32-vs-fp64 logit error), and every expert
    that is in one set but not the other lies within NEAR_TIE of the K'-th
    largest logit.  Gates are checked on every token against the oracle's
    gates for the GPU's own ids."""
    T, N = s_ref.shape
    ids_ref, g_ref = oracle.select(s_ref, K)
    near = boundary_gap(s_ref, K) <= NEAR_TIE
    # every GPU selection is well formed: in range, K' distinct experts
    assert ((ids_gpu >= 0) & (ids_gpu < N)).all()
    assert all(len(set(r)) == K for r in ids_gpu.tolist())
    same_set = np.array([set(a) == set(b) for a, b in zip(ids_gpu.tolist(), ids_ref.tolist())])
    bad = ~same_set & ~near
    assert not bad.any(), f"selection differs on {bad.sum()} tokens with a clear gap, e.g. {np.nonzero(bad)[0][:5]}"
    # the GPU's set is a top-K' of the fp64 logits on every token
    if K < N:
        chosen = np.zeros((T, N), dtype=bool)
        chosen[np.arange(T)[:, None], ids_gpu.astype(np.int64)] = True
        sel_min = np.where(chosen, s_ref, np.inf).min(axis=1)
        unsel_max = np.where(chosen, -np.inf, s_ref).max(axis=1)
        worst = np.nonzero(sel_min < unsel_max - ORDER_TOL)[0]
        assert worst.size == 0, f"not a top-K' selection on tokens {worst[:5]}"
        # flipped experts sit in the near-tie band around the K'-th logit
        kth = -np.sort(-s_ref, axis=1)[:, K - 1]
        for t in np.nonzero(~same_set)[0]:
            diff = set(ids_gpu[t].tolist()) ^ set(ids_ref[t].tolist())
            for e in diff:
                assert abs(s_ref[t, e] - kth[t]) <= NEAR_TIE, (t, e, s_ref[t, e] - kth[t])
    # order: non-increasing in the oracle's logits (up to ORDER_TOL); identical
    # where the oracle's consecutive gaps are clear
    s_sel = np.take_along_axis(s_ref, ids_gpu.astype(np.int64), 1)
    assert (np.diff(s_sel, axis=1) <= ORDER_TOL).all(), "slot order not by logit"
    s_ref_sel = np.take_along_axis(s_ref, ids_ref.astype(np.int64), 1)
    clear = (np.abs(np.diff(s_ref_sel, axis=1)) > ORDER_TOL).all(axis=1) & same_set
    np.testing.assert_array_equal(ids_gpu[clear], ids_ref[clear])
    # gates: renormalised softmax at the GPU's own ids (fp32 vs fp64), on every
    # token; where the ids are the oracle's own, also its own gates
    g_for_gpu_ids = oracle.gates_for_ids(s_ref, ids_gpu)
    np.testing.assert_allclose(gates_gpu, g_for_gpu_ids, rtol=0, atol=1e-4)
    ids_match = (ids_gpu == ids_ref).all(axis=1)
    np.testing.assert_allclose(gates_gpu[ids_match], g_ref[ids_match], rtol=0, atol=1e-4)
    np.testing.assert_allclose(gates_gpu.sum(1), 1.0, rtol=0, atol=1e-5)
    flipped = ~same_set
    return near, flipped


def check_dispatch(ids_gpu: np.ndarray, offsets: np.ndarray, perm: np.ndarray, N: int):
    off_ref, perm_ref, _ = oracle.dispatch(ids_gpu, N)
    np.testing.assert_array_equal(offsets, off_ref)
    np.testing.assert_array_equal(perm, perm_ref)


def check_dispatch_against_oracle_ids(ids_ref: np.ndarray, ids_gpu: np.ndarray,
                                      offsets: np.ndarray, perm: np.ndarray, N: int):
    """Dispatch vs the oracle's own routing, when both select the same sets.

    perm stores t*K' + k.  Where two selected logits are equal to within
    rounding, the slot order k may legitimately differ, so the unique part --
    the token sequence of every expert -- is compared, and the slot part only
    where the two slot orders agree."""
    K = ids_ref.shape[1]
    off_ref, perm_ref, _ = oracle.dispatch(ids_ref, N)
    np.testing.assert_array_equal(offsets, off_ref)
    np.testing.assert_array_equal(perm // K, perm_ref // K)
    same_order = (ids_ref == ids_gpu).all(axis=1)
    agree = same_order[perm_ref // K]
    np.testing.assert_array_equal(perm[agree], perm_ref[agree])


def rel_err(y: np.ndarray, y_ref: np.ndarray) -> float:
    return float(np.abs(y - y_ref).max() / max(np.abs(y_ref).max(), 1e-30))


def reference_y(L: oracle.Layer, x_np, tokens: np.ndarray, ids_gpu: np.ndarray,
                flipped: np.ndarray):
    """y_ref for `tokens`: oracle routing, except GPU ids where the selection flipped."""
    y = np.empty((len(tokens), L.d))
    own = ~flipped[tokens]
    if own.any():
        y[own], _, _ = oracle.forward(L, x_np, tokens=tokens[own])
    if (~own).any():
        y[~own], _, _ = oracle.forward(L, x_np, tokens=tokens[~own], ids=ids_gpu)
    return y


def y_to_numpy(y: torch.Tensor) -> np.ndarray:
    return y.detach().float().cpu().numpy().astype(np.float64)


def tile_cover_tokens(offsets: np.ndarray, perm: np.ndarray, K: int,
                      tile_rows=(128, 256)) -> np.ndarray:
    """Tokens that put at least one compared row into every expert's first
    and last M-tile, for each grouped-GEMM tile height: per expert, the first
    row of its range, the first row of its last tile and its last row (the
    ragged tail)."""
    rows = set()
    for e in range(len(offsets) - 1):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 <= r0:
            continue
        rows.update((r0, r1 - 1))
        for tm in tile_rows:
            rows.add(r0 + (r1 - 1 - r0) // tm * tm)
    rows = np.array(sorted(rows), dtype=np.int64)
    return np.unique(perm[rows] // K).astype(np.int64)


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    """First and last few tokens, tile boundaries, and a random spread."""
    rng = np.random.default_rng(seed)
    fixed = {0, 1, 127, 128, T - 1, T - 2, T // 2}
    fixed = {t for t in fixed if 0 <= t < T}
    rest = rng.choice(T, size=min(T, max(0, n - len(fixed))), replace=False)
    return np.array(sorted(fixed | set(rest.tolist())), dtype=np.int64)
