"""Pins of the oracle's indexer and pooled importance against things other than
itself: a library cosine routine, a library sigmoid, brute-force loops over a
materialised score matrix, and structural properties.

Source: "IndexMem" technical summary, §2.A Learnable indexer (Architecture,
Function, Training bullets).
"""
import math

import numpy as np
import pytest
from scipy.spatial.distance import cdist
from scipy.special import expit

from oracle import indexmem_oracle as om


def _rand_case(rng, b=2, L=13, H=6, Hq=3, d=5, dI=4):
    X = rng.standard_normal((b, L, H))
    Q = rng.standard_normal((b, L, Hq, d))
    W_iq = rng.standard_normal((Hq, d, dI)) / math.sqrt(d)
    W_ik = rng.standard_normal((H, dI)) / math.sqrt(H)
    w_ig = rng.standard_normal((H, Hq)) / math.sqrt(H)
    return X, Q, W_iq, W_ik, w_ig


def test_qk_norm_is_unit_rms_and_positively_proportional():
    rng = np.random.default_rng(1)
    X, Q, W_iq, W_ik, w_ig = _rand_case(rng)
    qhat, khat, gate = om.indexer_features(X, Q, W_iq, W_ik, w_ig)
    ms = np.mean(qhat ** 2, axis=-1)
    assert np.allclose(ms, 1.0, atol=1e-4)
    assert np.allclose(np.mean(khat ** 2, axis=-1), 1.0, atol=1e-4)
    # direction is the raw projection's direction (positive multiple)
    raw = np.einsum("bld,dj->blj", X, W_ik)
    cos = np.sum(raw * khat, -1) / (np.linalg.norm(raw, axis=-1) * np.linalg.norm(khat, axis=-1))
    assert np.allclose(cos, 1.0, atol=1e-12)
    assert np.all((gate > 0) & (gate < 1))


def test_single_head_score_is_scaled_cosine_library_pin():
    """One head, zero gate weights (gate = 1/2), permutation projections whose
    effect is written as array shifts: A[s,t] = 0.5 * sqrt(dI) * cos(qI_s, kI_t),
    with the cosine taken from scipy's cdist -- pins the RMS normalisation, the
    1/sqrt(dI) scale, the gate, and the orientation (query rows, key columns)."""
    rng = np.random.default_rng(2)
    b, L, H, dI = 1, 11, 9, 6
    d = dI
    X = rng.standard_normal((b, L, H))
    Q = rng.standard_normal((b, L, 1, d))
    # W_iq[0][i, j] = 1 iff j == (i + 1) % d  ->  (q @ W)[j] = q[j - 1]  (roll by +1)
    W_iq = np.zeros((1, d, dI))
    for i in range(d):
        W_iq[0, i, (i + 1) % d] = 1.0
    # W_ik[i, j] = 1 iff i == j + 2  ->  (x @ W)[j] = x[j + 2]
    W_ik = np.zeros((H, dI))
    for j in range(dI):
        W_ik[j + 2, j] = 1.0
    w_ig = np.zeros((H, 1))
    qhat, khat, gate = om.indexer_features(X, Q, W_iq, W_ik, w_ig)
    A = om.score_block(qhat[0], gate[0], khat[0], dI)
    qI = np.roll(Q[0, :, 0, :], 1, axis=-1)
    kI = X[0, :, 2:2 + dI]
    cos = 1.0 - cdist(qI, kI, metric="cosine")
    expect = 0.5 * math.sqrt(dI) * cos
    assert np.allclose(A, expect, rtol=1e-5, atol=1e-6)
    # pooled: causal column max, diagonal included
    I = om.pooled_importance(qhat, khat, gate)[0]
    for t in range(L):
        assert I[t] == pytest.approx(max(expect[s, t] for s in range(t, L)), rel=1e-5, abs=1e-6)


def test_multi_head_gate_library_pin():
    """Gated head sum with the gate from scipy's expit and per-head cosines from
    cdist: A[s,t] = sum_h expit(x_s . w_ig[:,h]) sqrt(dI) cos(qI_{s,h}, kI_t)."""
    rng = np.random.default_rng(3)
    X, Q, W_iq, W_ik, w_ig = _rand_case(rng, b=1, L=10, H=7, Hq=4, d=6, dI=5)
    qhat, khat, gate = om.indexer_features(X, Q, W_iq, W_ik, w_ig)
    A = om.score_block(qhat[0], gate[0], khat[0], 5)
    kI = X[0] @ W_ik
    expect = np.zeros((10, 10))
    for h in range(4):
        qI = Q[0, :, h, :] @ W_iq[h]
        g = expit(X[0] @ w_ig[:, h])
        expect += g[:, None] * math.sqrt(5) * (1.0 - cdist(qI, kI, metric="cosine"))
    assert np.allclose(A, expect, rtol=1e-5, atol=1e-6)


def _brute_force_I(qhat, khat, gate, q_ranges):
    """Materialise A with plain loops (math.fsum), then take running column maxima
    over the query ranges in order."""
    b, L, Hq, dI = qhat.shape
    out = np.full((b, L), -np.inf)
    for bi in range(b):
        A = [[math.fsum(gate[bi, s, h] * math.fsum(qhat[bi, s, h, j] * khat[bi, t, j]
                                                   for j in range(dI))
                        for h in range(Hq)) / math.sqrt(dI)
              for t in range(L)] for s in range(L)]
        for (q0, q1) in q_ranges:
            for t in range(L):
                if t >= q1:
                    continue
                if t >= q0:
                    out[bi, t] = -np.inf
                for s in range(max(t, q0), q1):
                    out[bi, t] = max(out[bi, t], A[s][t])
    return out


@pytest.mark.parametrize("ranges", [[(0, 13)], [(0, 4), (4, 9), (9, 13)], [(0, 1), (1, 13)]])
def test_streaming_max_equals_materialised_max(ranges):
    rng = np.random.default_rng(4)
    X, Q, W_iq, W_ik, w_ig = _rand_case(rng)
    qhat, khat, gate = om.indexer_features(X, Q, W_iq, W_ik, w_ig)
    I = None
    for q0, q1 in ranges:
        I = om.pooled_importance(qhat, khat, gate, q_begin=q0, q_end=q1, prev=I, key_block=4)
    ref = _brute_force_I(qhat, khat, gate, ranges)
    assert np.allclose(I, ref, rtol=1e-12, atol=1e-12)


def test_partial_range_leaves_unseen_keys_at_minus_inf():
    rng = np.random.default_rng(5)
    X, Q, W_iq, W_ik, w_ig = _rand_case(rng)
    qhat, khat, gate = om.indexer_features(X, Q, W_iq, W_ik, w_ig)
    I = om.pooled_importance(qhat, khat, gate, q_begin=0, q_end=6)
    assert np.all(np.isneginf(I[:, 6:]))
    assert np.all(np.isfinite(I[:, :6]))
    ref = _brute_force_I(qhat, khat, gate, [(0, 6)])
    assert np.allclose(I[:, :6], ref[:, :6], rtol=1e-12)


def test_key_subset_and_blocking_invariance():
    rng = np.random.default_rng(6)
    X, Q, W_iq, W_ik, w_ig = _rand_case(rng, L=29)
    qhat, khat, gate = om.indexer_features(X, Q, W_iq, W_ik, w_ig)
    full = om.pooled_importance(qhat, khat, gate, key_block=128)
    small = om.pooled_importance(qhat, khat, gate, key_block=3)
    keys = np.array([28, 0, 17, 5])
    sub = om.pooled_importance(qhat, khat, gate, keys=keys, key_block=2)
    assert np.array_equal(full, small) or np.allclose(full, small, rtol=1e-14)
    assert np.allclose(sub, full[:, keys], rtol=1e-14)


def test_collapsed_query_identity():
    """A[s,t] = qtilde_s . khat_t with qtilde_s = sum_h gate[s,h] qhat[s,h] / sqrt(dI):
    exact algebra of the gated head sum (no activation between product and sum)."""
    rng = np.random.default_rng(7)
    X, Q, W_iq, W_ik, w_ig = _rand_case(rng, b=1, L=17)
    qhat, khat, gate = om.indexer_features(X, Q, W_iq, W_ik, w_ig)
    A = om.score_block(qhat[0], gate[0], khat[0], 4)
    qt = np.einsum("sh,shj->sj", gate[0], qhat[0]) / 2.0
    assert np.allclose(A, qt @ khat[0].T, rtol=1e-12, atol=1e-14)


def test_last_key_has_only_its_own_query():
    rng = np.random.default_rng(8)
    X, Q, W_iq, W_ik, w_ig = _rand_case(rng, b=1, L=9)
    qhat, khat, gate = om.indexer_features(X, Q, W_iq, W_ik, w_ig)
    I = om.pooled_importance(qhat, khat, gate)[0]
    A = om.score_block(qhat[0], gate[0], khat[0], 4)
    assert I[-1] == A[-1, -1]
    assert I[0] == A[:, 0].max()
