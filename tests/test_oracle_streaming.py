"""The streamed evaluation of the pooled importance at a few keys equals the
full pooled importance (same definition, queries taken in blocks)."""
import numpy as np

from oracle import indexmem_oracle as om


def test_importance_at_keys_equals_full_pooling():
    rng = np.random.default_rng(30)
    L, H, Hq, d, dI = 37, 8, 3, 6, 4
    X = rng.standard_normal((L, H))
    Q = rng.standard_normal((L, Hq, d))
    W_iq = rng.standard_normal((Hq, d, dI))
    W_ik = rng.standard_normal((H, dI))
    w_ig = rng.standard_normal((H, Hq))
    qhat, khat, gate = om.indexer_features(X[None], Q[None], W_iq, W_ik, w_ig)
    full = om.pooled_importance(qhat, khat, gate)[0]
    keys = np.array([0, 5, 36, 17])
    part = om.importance_at_keys(X, Q, W_iq, W_ik, w_ig, keys, s_block=5)
    assert np.allclose(part, full[keys], rtol=1e-12, atol=1e-12)
    part2 = om.importance_at_keys(X, Q, W_iq, W_ik, w_ig, keys, q_end=30, s_block=7)
    full2 = om.pooled_importance(qhat, khat, gate, q_end=30)[0]
    ok = keys < 30
    assert np.allclose(part2[ok], full2[keys[ok]], rtol=1e-12)
    assert np.all(np.isneginf(part2[~ok]))
