"""CPU oracle for the MomentKV readout variant -- TEST INFRASTRUCTURE ONLY.

Plain float64 NumPy restatement of the moment-statistics compensation, used by
the test-suite to check the CUDA path's moment mode. Only the tests may import
it; the product path never does and shares no code with it.

Source, cited by page title and section:

* [MK-sum]  "MomentKV" technical summary (gist.science), Method:
            §1 compact moment statistics -- four running sums per head over
               the evicted set: the count n_e, the key sum s_k, the value sum
               s_v and the outer-product sum S = sum v k^T;
            §2 first-order approximation of the evicted output -- logits
               re-centred on the mean key, first-order Taylor expansion of the
               softmax: f_E(q) ~ v_bar + S~ q / (n_e sqrt(d));
            §4 normalisation-corrected inference -- the output is a convex mix
               w_R f_R(q) + (1 - w_R) f_E(q), with w_R from a lower bound on
               the evicted partition function obtained through Jensen's
               inequality.

Readings (the page gives the formulas' shape, not every step):

* S~, the value-key covariance, is sum_i (v_i - v_bar)(k_i - k_bar)^T
  = S - s_v s_k^T / n_e. This is what the expansion in §2 produces: with
  weights proportional to 1 + q.(k_i - k_bar)/sqrt(d) (whose sum is n_e) the
  weighted value mean is v_bar + sum_i v_i (k_i - k_bar)^T q / (n_e sqrt(d)).
* The Jensen bound of §4: Z_E = sum_i exp(q.k_i/sqrt(d)) >= n_e exp(q.k_bar/
  sqrt(d)) =: Z_E^; w_R = Z_R / (Z_R + Z_E^) with Z_R the retained partition
  function (the retained set includes the decode tokens appended to it).
* The sums carry no decay. With grouped-query attention the statistics are
  kept per KV head (the evicted keys and values are per KV head) and read by
  the query heads of its group. With n_e = 0 the output is the retained
  attention.

Parity status: pinned by tests/test_oracle_moment.py -- exact recovery of
full attention when the evicted keys coincide (library attention routine),
the second-order error of the estimate (ratio of errors under halved key
spread), the covariance against the library's two-pass covariance, the
Jensen bound against the exact evicted partition function, additivity of the
statistics and n_e = 0.
"""

from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().float().numpy()
    return np.asarray(a, dtype=np.float64)


def moment_stats(K, V, E, stats0: Optional[Tuple] = None):
    """[MK-sum] §1: running sums over the evicted positions.

    K, V [b, L, Hkv, d]; E [b, n] positions (the sums do not depend on the
    order). stats0 = (n_e, s_k, s_v, S) to continue from, else zeros.
    Returns n_e [b], s_k [b,Hkv,d], s_v [b,Hkv,d], S [b,Hkv,d,d] with
    S[h] = sum_i v_i k_i^T (row = value dimension, column = key dimension).
    """
    K, V = _f64(K), _f64(V)
    E = np.asarray(E, dtype=np.int64)
    b, _, Hkv, d = K.shape
    if stats0 is None:
        n_e = np.zeros(b)
        s_k = np.zeros((b, Hkv, d))
        s_v = np.zeros((b, Hkv, d))
        S = np.zeros((b, Hkv, d, d))
    else:
        n_e, s_k, s_v, S = (np.array(_f64(x)) for x in stats0)
    for bi in range(b):
        for p in E[bi]:
            n_e[bi] += 1.0
            for h in range(Hkv):
                k, v = K[bi, p, h], V[bi, p, h]
                s_k[bi, h] += k
                s_v[bi, h] += v
                S[bi, h] += np.outer(v, k)
    return n_e, s_k, s_v, S


def evicted_estimate(q, n_e: float, s_k, s_v, S):
    """[MK-sum] §2 and §4 for one query and one head's statistics.

    Returns (f_E^ [d], log Z_E^) with
      k_bar = s_k / n_e, v_bar = s_v / n_e, S~ = S - s_v s_k^T / n_e,
      f_E^ = v_bar + S~ q / (n_e sqrt(d)),  log Z_E^ = log n_e + q.k_bar / sqrt(d).
    n_e must be positive.
    """
    q, s_k, s_v, S = _f64(q), _f64(s_k), _f64(s_v), _f64(S)
    d = q.shape[0]
    k_bar = s_k / n_e
    v_bar = s_v / n_e
    S_tilde = S - np.outer(s_v, s_k) / n_e
    f_hat = v_bar + (S_tilde @ q) / (n_e * math.sqrt(d))
    log_z = math.log(n_e) + float(q @ k_bar) / math.sqrt(d)
    return f_hat, log_z


def moment_decode_step(q, k_new, v_new, K_R, V_R, cache_len, n_e, s_k, s_v, S):
    """One decode step with the MomentKV readout, every sequence.

    q [b,Hq,d]; k_new, v_new [b,Hkv,d] appended at row cache_len[b] of the
    retained cache K_R/V_R [b,cap,Hkv,d] (not written back); n_e [b];
    s_k, s_v [b,Hkv,d]; S [b,Hkv,d,d]. Query head h reads KV head h//(Hq/Hkv).
    Returns (o [b,Hq,d], new cache_len, o_R, f_E^, w_R [b,Hq]):
      o_R = softmax(q K^T / sqrt(d)) V over the cache incl. the new row,
      log Z_R = the log-sum-exp of those logits,
      w_R = 1 / (1 + exp(log Z_E^ - log Z_R)),  o = w_R o_R + (1 - w_R) f_E^
    (o = o_R and w_R = 1 when n_e = 0).
    """
    q, k_new, v_new = _f64(q), _f64(k_new), _f64(v_new)
    KR, VR = _f64(K_R), _f64(V_R)
    n_e, s_k, s_v, S = _f64(n_e), _f64(s_k), _f64(s_v), _f64(S)
    cache_len = np.asarray(cache_len).astype(np.int64)
    b, Hq, d = q.shape
    Hkv = k_new.shape[1]
    group = Hq // Hkv
    o = np.zeros((b, Hq, d))
    o_R = np.zeros((b, Hq, d))
    f_E = np.zeros((b, Hq, d))
    w_R = np.ones((b, Hq))
    for bi in range(b):
        n = int(cache_len[bi])
        Kc = np.concatenate([KR[bi, :n], k_new[bi][None]], axis=0)
        Vc = np.concatenate([VR[bi, :n], v_new[bi][None]], axis=0)
        for h in range(Hq):
            kv = h // group
            s = Kc[:, kv] @ q[bi, h] / math.sqrt(d)
            mx = s.max()
            p = np.exp(s - mx)
            o_R[bi, h] = (p @ Vc[:, kv]) / p.sum()
            if n_e[bi] > 0:
                log_zr = mx + math.log(p.sum())
                f_E[bi, h], log_ze = evicted_estimate(q[bi, h], n_e[bi], s_k[bi, kv],
                                                      s_v[bi, kv], S[bi, kv])
                w_R[bi, h] = 1.0 / (1.0 + math.exp(log_ze - log_zr))
                o[bi, h] = w_R[bi, h] * o_R[bi, h] + (1.0 - w_R[bi, h]) * f_E[bi, h]
            else:
                o[bi, h] = o_R[bi, h]
    return o, cache_len + 1, o_R, f_E, w_R
