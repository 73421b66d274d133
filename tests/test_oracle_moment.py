"""Pins of the MomentKV oracle ("MomentKV" technical summary, Method §1, §2,
§4) against facts other than itself: the library attention routine, the
library covariance, the exact evicted partition function and the error order
of a first-order expansion."""
import math

import numpy as np
import pytest
import torch

from oracle import indexmem_oracle as om
from oracle import momentkv_oracle as mk


def _sdpa(q, K, V):
    """Textbook softmax attention of one query over rows K, V (float64)."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q[None]), t(K), t(V)).numpy()[0, 0, 0]


def _case(rng, b=2, Hkv=2, group=2, d=16, n_R=5, n_E=7, same_keys=False):
    L = n_R + n_E
    K = rng.standard_normal((b, L, Hkv, d))
    V = rng.standard_normal((b, L, Hkv, d))
    perm = np.stack([rng.permutation(L) for _ in range(b)])
    R = np.sort(perm[:, :n_R], axis=1)
    E = np.sort(perm[:, n_R:], axis=1)
    if same_keys:
        k0 = rng.standard_normal((b, Hkv, d))
        for bi in range(b):
            K[bi, E[bi]] = k0[bi]
    q = rng.standard_normal((b, Hkv * group, d))
    kn = rng.standard_normal((b, Hkv, d))
    vn = rng.standard_normal((b, Hkv, d))
    return K, V, R, E, q, kn, vn


def _retained(K, V, R, cap):
    b, _, Hkv, d = K.shape
    KR = np.zeros((b, cap, Hkv, d))
    VR = np.zeros_like(KR)
    for bi in range(b):
        KR[bi, :R.shape[1]] = K[bi, R[bi]]
        VR[bi, :R.shape[1]] = V[bi, R[bi]]
    return KR, VR


def test_identical_evicted_keys_recover_full_attention():
    # With every evicted key equal, the expansion of §2 is exact (f_E = v_bar)
    # and Jensen's bound of §4 holds with equality, so the mix is full softmax
    # attention over retained + new + evicted rows.
    rng = np.random.default_rng(11)
    K, V, R, E, q, kn, vn = _case(rng, same_keys=True)
    b, Hq, d = q.shape
    Hkv = kn.shape[1]
    n_R = R.shape[1]
    KR, VR = _retained(K, V, R, n_R + 1)
    stats = mk.moment_stats(K, V, E)
    o, new_len, _, _, w_R = mk.moment_decode_step(q, kn, vn, KR, VR, np.full(b, n_R), *stats)
    assert np.all(new_len == n_R + 1)
    assert np.all((w_R > 0) & (w_R < 1))
    for bi in range(b):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            Kall = np.concatenate([K[bi, R[bi], kv], kn[bi, kv][None], K[bi, E[bi], kv]])
            Vall = np.concatenate([V[bi, R[bi], kv], vn[bi, kv][None], V[bi, E[bi], kv]])
            ref = _sdpa(q[bi, h], Kall, Vall)
            np.testing.assert_allclose(o[bi, h], ref, rtol=1e-11, atol=1e-12)


def test_estimate_error_is_second_order_in_key_spread():
    # §2 is a first-order expansion about the mean key: halving the spread of
    # the evicted keys must divide the error of v_bar + S~q/(n sqrt d) by ~4,
    # and the error of v_bar alone (no correction) by ~2.
    rng = np.random.default_rng(5)
    d, n = 32, 50
    kbar = rng.standard_normal(d)
    delta = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    q = rng.standard_normal(d)
    errs, errs0 = [], []
    for eps in (0.2, 0.1, 0.05):
        Kc = kbar + eps * delta
        exact = _sdpa(q, Kc, V)
        s_k, s_v, S = Kc.sum(0), V.sum(0), V.T @ Kc
        f_hat, _ = mk.evicted_estimate(q, float(n), s_k, s_v, S)
        errs.append(np.linalg.norm(f_hat - exact))
        errs0.append(np.linalg.norm(V.mean(0) - exact))
    for a, c in zip(errs, errs[1:]):
        assert 3.4 < a / c < 4.6, errs
    for a, c in zip(errs0, errs0[1:]):
        assert 1.7 < a / c < 2.3, errs0


def test_covariance_matches_library_two_pass():
    # S~ = S - s_v s_k^T / n_e must be n_e times the (biased) cross-covariance
    # of values and keys; checked through f_E^ - v_bar = S~ q / (n_e sqrt d).
    rng = np.random.default_rng(3)
    d, n = 24, 40
    Kc = rng.standard_normal((n, d)) + 3.0
    V = rng.standard_normal((n, d)) - 1.0
    q = rng.standard_normal(d)
    f_hat, _ = mk.evicted_estimate(q, float(n), Kc.sum(0), V.sum(0), V.T @ Kc)
    cov = np.cov(V.T, Kc.T, bias=True)[:d, d:]        # library two-pass covariance
    ref = V.mean(0) + n * cov @ q / (n * math.sqrt(d))
    np.testing.assert_allclose(f_hat, ref, rtol=1e-11, atol=1e-12)


def test_jensen_bound_below_exact_partition_function():
    rng = np.random.default_rng(9)
    d, n = 16, 30
    for _ in range(20):
        Kc = rng.standard_normal((n, d)) * rng.uniform(0.1, 2.0)
        q = rng.standard_normal(d)
        _, log_ze = mk.evicted_estimate(q, float(n), Kc.sum(0), np.zeros(d), np.zeros((d, d)))
        exact = math.log(np.exp(Kc @ q / math.sqrt(d)).sum())
        assert log_ze <= exact + 1e-12


def test_no_evicted_tokens_is_retained_attention():
    rng = np.random.default_rng(2)
    K, V, R, E, q, kn, vn = _case(rng)
    b, Hq, d = q.shape
    Hkv = kn.shape[1]
    n_R = R.shape[1]
    KR, VR = _retained(K, V, R, n_R + 3)
    zeros = (np.zeros(b), np.zeros((b, Hkv, d)), np.zeros((b, Hkv, d)), np.zeros((b, Hkv, d, d)))
    o, _, o_R, _, w_R = mk.moment_decode_step(q, kn, vn, KR, VR, np.full(b, n_R), *zeros)
    assert np.all(w_R == 1.0)
    for bi in range(b):
        for h in range(Hq):
            kv = h // (Hq // Hkv)
            Kall = np.concatenate([K[bi, R[bi], kv], kn[bi, kv][None]])
            Vall = np.concatenate([V[bi, R[bi], kv], vn[bi, kv][None]])
            np.testing.assert_allclose(o[bi, h], _sdpa(q[bi, h], Kall, Vall), rtol=1e-12,
                                       atol=1e-13)


def test_statistics_are_additive_and_order_free():
    rng = np.random.default_rng(4)
    K, V, R, E, *_ = _case(rng, n_E=9)
    E1, E2 = E[:, :4], E[:, 4:]
    part = mk.moment_stats(K, V, E1)
    both = mk.moment_stats(K, V, E2, stats0=part)
    once = mk.moment_stats(K, V, E[:, ::-1])
    for x, y in zip(both, once):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=1e-12)


def test_moment_sums_equal_indexmem_memory_at_identity_map():
    # With lambda = 1 and W_phi = I the IndexMem memory is sum k v^T and sum k:
    # S^T and s_k of the moment statistics.
    rng = np.random.default_rng(8)
    K, V, R, E, *_ = _case(rng, n_E=6)
    d = K.shape[-1]
    M, bs = om.memory_update(K, V, E, np.eye(d), 1.0)
    n_e, s_k, s_v, S = mk.moment_stats(K, V, E)
    np.testing.assert_allclose(M, np.swapaxes(S, -1, -2), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(bs, s_k, rtol=1e-12, atol=1e-12)
    assert np.all(n_e == E.shape[1])
