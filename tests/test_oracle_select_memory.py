"""Pins of the oracle's top-B selection, compaction and latent-memory update.

Sources: "IndexMem" technical summary §1 (token eviction) and §2.B Latent
memory (Mechanism: decayed outer-product accumulation into M and stabiliser b);
"MOMENTKV" technical summary, Method §1 (running sums s_k and S = sum v k^T over
the evicted set), which the memory reduces to when the decay is 1 and the
feature map is the identity.
"""
import math

import numpy as np
import pytest

from oracle import indexmem_oracle as om


# ----------------------------------------------------------------- selection

def _python_sorted_topb(I, B):
    L = len(I)
    order = sorted(range(L), key=lambda t: (-(float(I[t]) + 0.0), t))
    return sorted(order[:B]), sorted(order[B:])


@pytest.mark.parametrize("B", [0, 1, 5, 16, 31, 32])
def test_select_equals_python_sort_with_ties(B):
    rng = np.random.default_rng(10)
    I = rng.integers(-3, 4, size=(3, 32)).astype(np.float32)   # many ties
    I[0, 5] = -0.0
    I[0, 6] = 0.0
    I[1, :] = 0.0
    I[1, ::3] = -0.0                                           # -0 and +0 mixed
    R, E = om.select_budget(I, B)
    for bi in range(3):
        r, e = _python_sorted_topb(I[bi], B)
        assert list(R[bi]) == r and list(E[bi]) == e


def test_select_invariants_random():
    rng = np.random.default_rng(11)
    I = rng.standard_normal((4, 257)).astype(np.float32)
    I[:, 100:110] = I[:, 50:60]    # exact duplicates
    B = 40
    R, E = om.select_budget(I, B)
    for bi in range(4):
        assert np.all(np.diff(R[bi]) > 0) and np.all(np.diff(E[bi]) > 0)
        assert sorted(set(R[bi]) | set(E[bi])) == list(range(257))
        assert len(set(R[bi]) & set(E[bi])) == 0
        assert I[bi, R[bi]].min() >= I[bi, E[bi]].max()
        # at the threshold, a kept tie is never after an evicted tie
        thr = I[bi, R[bi]].min()
        kept_eq = R[bi][I[bi, R[bi]] == thr]
        ev_eq = E[bi][I[bi, E[bi]] == thr]
        if len(kept_eq) and len(ev_eq):
            assert kept_eq.max() < ev_eq.min()


def test_select_full_budget_and_compact_identity():
    rng = np.random.default_rng(12)
    K = rng.standard_normal((2, 9, 3, 4)).astype(np.float32)
    V = rng.standard_normal((2, 9, 3, 4)).astype(np.float32)
    I = rng.standard_normal((2, 9))
    R, E = om.select_budget(I, 9)
    assert E.shape == (2, 0)
    KR, VR = om.compact(K, V, R)
    assert np.array_equal(KR, K) and np.array_equal(VR, V)
    KR2, _ = om.compact(K, V, R, cap=12)
    assert KR2.shape == (2, 12, 3, 4) and np.all(KR2[:, 9:] == 0)


def test_compact_gathers_rows_in_position_order():
    K = np.arange(2 * 6 * 1 * 2, dtype=np.float32).reshape(2, 6, 1, 2)
    R = np.array([[1, 4], [0, 5]])
    KR, _ = om.compact(K, K, R)
    assert np.array_equal(KR[0, :, 0], [[2, 3], [8, 9]])
    assert np.array_equal(KR[1, :, 0], [[12, 13], [22, 23]])


# -------------------------------------------------------------------- memory

def test_memory_hand_worked_example():
    """lam = 1/2, d = r = 2, W_phi = [[1,0],[1,1]] (phi(k) = (k0, k0+k1)).
    Evicted positions 1 and 3 of a 4-token context:
      k1 = (1,2), v1 = (3,-1) -> phi1 = (1,3);  k3 = (0,1), v3 = (2,2) -> phi3 = (0,1).
    After pos 1: M = phi1 v1^T = [[3,-1],[9,-3]], b = (1,3).
    After pos 3: M = 1/2 M + phi3 v3^T = [[1.5,-0.5],[6.5,0.5]], b = (0.5,2.5).
    With a prior state M0 = all ones, b0 = (2,2): lam^2 M0 is added, giving
    [[1.75,-0.25],[6.75,0.75]] and b = (1.0,3.0)."""
    K = np.zeros((1, 4, 1, 2))
    V = np.zeros((1, 4, 1, 2))
    K[0, 1, 0] = [1, 2]; V[0, 1, 0] = [3, -1]
    K[0, 3, 0] = [0, 1]; V[0, 3, 0] = [2, 2]
    K[0, 0, 0] = [5, 5]; V[0, 0, 0] = [7, 7]      # retained, must not enter
    W = np.array([[1.0, 0.0], [1.0, 1.0]])
    E = np.array([[1, 3]])
    M, b = om.memory_update(K, V, E, W, 0.5)
    assert np.array_equal(M[0, 0], [[1.5, -0.5], [6.5, 0.5]])
    assert np.array_equal(b[0, 0], [0.5, 2.5])
    M, b = om.memory_update(K, V, E, W, 0.5, M0=np.ones((1, 1, 2, 2)), b0=np.full((1, 1, 2), 2.0))
    assert np.array_equal(M[0, 0], [[1.75, -0.25], [6.75, 0.75]])
    assert np.array_equal(b[0, 0], [1.0, 3.0])


def test_memory_identity_features_no_decay_equals_moment_sums():
    """lam = 1, W_phi = I: M = sum_i k_i v_i^T and b = sum_i k_i over the evicted
    set, i.e. MomentKV's S = sum v k^T transposed and its key sum s_k."""
    rng = np.random.default_rng(13)
    b_, L, Hkv, d = 2, 40, 3, 5
    K = rng.standard_normal((b_, L, Hkv, d))
    V = rng.standard_normal((b_, L, Hkv, d))
    I = rng.standard_normal((b_, L))
    _, E = om.select_budget(I, 12)
    M, bs = om.memory_update(K, V, E, np.eye(d), 1.0)
    for bi in range(b_):
        for h in range(Hkv):
            Ke, Ve = K[bi, E[bi], h], V[bi, E[bi], h]
            S = sum(np.outer(Ve[i], Ke[i]) for i in range(len(E[bi])))   # MomentKV S
            assert np.allclose(M[bi, h], S.T, rtol=1e-12, atol=1e-12)
            assert np.allclose(bs[bi, h], Ke.sum(0), rtol=1e-12, atol=1e-12)


def test_memory_decay_closed_form():
    """M = lam^n M0 + W_phi K_E^T diag(lam^(n-1-i)) V_E (one weighted matrix
    product per head) equals the sequential update."""
    rng = np.random.default_rng(14)
    b_, L, Hkv, d, r, lam = 1, 300, 2, 6, 4, 0.97
    K = rng.standard_normal((b_, L, Hkv, d))
    V = rng.standard_normal((b_, L, Hkv, d))
    W = rng.standard_normal((r, d))
    E = np.sort(rng.choice(L, size=250, replace=False))[None]
    M0 = rng.standard_normal((b_, Hkv, r, d))
    b0 = rng.standard_normal((b_, Hkv, r))
    M, bs = om.memory_update(K, V, E, W, lam, M0, b0)
    n = E.shape[1]
    w = lam ** (n - 1 - np.arange(n))
    for h in range(Hkv):
        Ke, Ve = K[0, E[0], h], V[0, E[0], h]
        Mc = lam ** n * M0[0, h] + W @ (Ke.T * w) @ Ve
        bc = lam ** n * b0[0, h] + W @ (Ke.T @ w)
        assert np.allclose(M[0, h], Mc, rtol=1e-10, atol=1e-10)
        assert np.allclose(bs[0, h], bc, rtol=1e-10, atol=1e-10)


def test_memory_chunked_equals_sequential_and_empty_is_identity():
    rng = np.random.default_rng(15)
    K = rng.standard_normal((2, 64, 2, 4))
    V = rng.standard_normal((2, 64, 2, 4))
    W = rng.standard_normal((3, 4))
    _, E = om.select_budget(rng.standard_normal((2, 64)), 10)
    M, b = om.memory_update(K, V, E, W, 0.9)
    M1, b1 = om.memory_update(K, V, E[:, :20], W, 0.9)
    M2, b2 = om.memory_update(K, V, E[:, 20:], W, 0.9, M1, b1)
    assert np.allclose(M, M2, rtol=1e-12) and np.allclose(b, b2, rtol=1e-12)
    M0 = rng.standard_normal(M.shape)
    b0 = rng.standard_normal(b.shape)
    Me, be = om.memory_update(K, V, E[:, :0], W, 0.9, M0, b0)
    assert np.array_equal(Me, M0) and np.array_equal(be, b0)


def test_memory_underflow_of_long_decay_is_zero_weight():
    """0.995^n underflows in float32 for very long evictions; in float64 the
    oldest token's weight is tiny but exact (lam^(n-1))."""
    K = np.zeros((1, 3, 1, 1)); V = np.zeros((1, 3, 1, 1))
    K[0, 0, 0, 0] = 1.0; V[0, 0, 0, 0] = 1.0
    M, _ = om.memory_update(K, V, np.array([[0, 1, 2]]), np.eye(1), 0.5)
    assert M[0, 0, 0, 0] == 0.25
