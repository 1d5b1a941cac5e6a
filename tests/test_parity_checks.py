"""The parity checks themselves (tests/parity_util.py), on the CPU: a correct
near-tie flip passes; a selection that is not a top-K' of the fp64 logits, a
flip outside the tie band, or wrong gates fail.  The GPU parity tests rely on
these checks to accept a flipped near-tie token."""
import numpy as np
import pytest

import oracle
from tests import parity_util as pu


def _logits(T=6, N=12, seed=3):
    rng = np.random.default_rng(seed)
    s = rng.normal(0.0, 1.0, size=(T, N))
    # token 0: the K'-th and (K'+1)-th logits 2e-5 apart (a near tie closer than
    # the checks' logit tolerance, so either selection passes)
    order = np.argsort(-s[0], kind="stable")
    s[0, order[4]] = s[0, order[3]] - 2e-5
    return s


def _gpu_like(s, K):
    ids, g = oracle.select(s, K)
    return ids.copy(), g.astype(np.float32)


def test_oracle_selection_passes():
    s = _logits()
    ids, g = _gpu_like(s, 4)
    near, flipped = pu.check_routing(ids, g, s, 4)
    assert near[0] and not flipped.any()


def test_valid_near_tie_flip_passes_and_is_reported():
    s = _logits()
    K = 4
    ids, _ = _gpu_like(s, K)
    order = np.argsort(-s[0], kind="stable")
    ids[0, K - 1] = order[K]          # the (K'+1)-th instead of the K'-th: both correct
    g = oracle.gates_for_ids(s, ids).astype(np.float32)
    near, flipped = pu.check_routing(ids, g, s, K)
    assert flipped[0] and flipped.sum() == 1


def test_selection_that_is_not_top_k_fails():
    s = _logits()
    K = 4
    ids, _ = _gpu_like(s, K)
    order = np.argsort(-s[0], kind="stable")
    ids[0, K - 1] = order[K + 2]      # the (K'+3)-th on a near-tie token
    g = oracle.gates_for_ids(s, ids).astype(np.float32)
    with pytest.raises(AssertionError):
        pu.check_routing(ids, g, s, K)


def test_flip_on_a_clear_gap_fails():
    s = _logits()
    K = 4
    ids, _ = _gpu_like(s, K)
    order = np.argsort(-s[1], kind="stable")
    ids[1, K - 1] = order[K]
    g = oracle.gates_for_ids(s, ids).astype(np.float32)
    with pytest.raises(AssertionError):
        pu.check_routing(ids, g, s, K)


def test_wrong_gates_fail_on_a_flipped_token():
    s = _logits()
    K = 4
    ids, _ = _gpu_like(s, K)
    order = np.argsort(-s[0], kind="stable")
    ids[0, K - 1] = order[K]
    g = oracle.gates_for_ids(s, ids).astype(np.float32)
    g[0, 0] += 1e-3
    g[0, 1] -= 1e-3                    # still sums to one
    with pytest.raises(AssertionError):
        pu.check_routing(ids, g, s, K)


def test_gates_for_ids_matches_select_on_its_own_ids():
    s = _logits(T=40, N=16, seed=7)
    ids, g = oracle.select(s, 5)
    np.testing.assert_array_equal(oracle.gates_for_ids(s, ids), g)
    # order-independent: a permutation of the slots permutes the gates
    perm = np.array([4, 2, 0, 3, 1])
    np.testing.assert_allclose(oracle.gates_for_ids(s, ids[:, perm]), g[:, perm], rtol=0,
                               atol=1e-15)


def test_tile_cover_reaches_every_first_and_last_tile():
    rng = np.random.default_rng(0)
    T, K, N = 500, 6, 20
    ids = np.stack([rng.choice(N, size=K, replace=False) for _ in range(T)]).astype(np.int32)
    offsets, perm, _ = oracle.dispatch(ids, N)
    tok = set(pu.tile_cover_tokens(offsets, perm, K, tile_rows=(16, 32)).tolist())
    for e in range(N):
        r0, r1 = offsets[e], offsets[e + 1]
        rows_tok = perm[r0:r1] // K
        for tm in (16, 32):
            first = rows_tok[:tm]
            last = rows_tok[(r1 - 1 - r0) // tm * tm:]
            assert tok & set(first.tolist()) and tok & set(last.tolist())
