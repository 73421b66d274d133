"""Pins of the pre-eviction oracle (chunked prefill that evicts after every
query range; "IndexMem" technical summary §2.A, pre-eviction before the full
prefill) against a brute-force simulation on a materialised score matrix, the
one-shot prefill, and exact special cases."""
import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import synth
from oracle import indexmem_oracle as om


def _inputs(L, batch=1, seed=3):
    wl = synth.WORKLOADS["c0"]
    w = synth.make_weights(wl.shape, seed)
    inp = synth.make_layer_inputs(wl, w, seed, L=L, batch=batch)
    return wl, w, inp


def _ranges(L, chunk):
    return [(q, min(L, q + chunk)) for q in range(0, L, chunk)]


def _run(inp, w, lam, B, ranges):
    return om.prefill_streaming(inp["X"], inp["Q"], inp["K"], inp["V"], w["W_iq"], w["W_ik"],
                                w["w_ig"], w["W_phi"], lam, B, ranges)


def test_single_range_equals_one_shot_prefill():
    L, B = 96, 20
    wl, w, inp = _inputs(L, batch=2)
    st = _run(inp, w, wl.shape.lam, B, [(0, L)])
    one = om.prefill_layer(inp["X"], inp["Q"], inp["K"], inp["V"], w["W_iq"], w["W_ik"],
                           w["w_ig"], w["W_phi"], wl.shape.lam, B)
    assert np.array_equal(st["R"], one["R"])
    assert np.array_equal(st["chunks"][0]["E"], one["E"])
    np.testing.assert_allclose(st["M"], one["M"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st["b"], one["b"], rtol=1e-12, atol=1e-12)


def test_budget_covering_the_context_evicts_nothing():
    L = 50
    wl, w, inp = _inputs(L)
    st = _run(inp, w, wl.shape.lam, L, _ranges(L, 16))
    assert np.array_equal(st["R"][0], np.arange(L))
    assert all(c["E"].shape[1] == 0 for c in st["chunks"])
    assert np.all(st["M"] == 0) and np.all(st["b"] == 0)


def test_matches_brute_force_simulation():
    # the full score matrix A[s,t] (score_block over all pairs), then the
    # streaming rule simulated with Python lists and sorted()
    L, B, chunk = 41, 7, 9
    wl, w, inp = _inputs(L, batch=2, seed=5)
    lam = wl.shape.lam
    st = _run(inp, w, lam, B, _ranges(L, chunk))
    qhat, khat, gate = om.indexer_features(inp["X"], inp["Q"], w["W_iq"], w["W_ik"], w["w_ig"])
    dI = khat.shape[-1]
    for bi in range(2):
        A = om.score_block(qhat[bi], gate[bi], khat[bi], dI)      # [L, L]
        R, IR, evicted = [], {}, []
        for ci, (q0, q1) in enumerate(_ranges(L, chunk)):
            cand = R + list(range(q0, q1))
            I = {}
            for t in cand:
                col = max(A[s, t] for s in range(max(t, q0), q1))
                I[t] = max(IR[t], col) if t in IR else col
            keep = sorted(cand, key=lambda t: (-I[t], t))[:B]
            E = sorted(set(cand) - set(keep))
            R = sorted(keep)
            IR = {t: I[t] for t in R}
            evicted += E
            rec = st["chunks"][ci]
            assert list(rec["cand"][bi]) == cand
            np.testing.assert_allclose(rec["I"][bi], [I[t] for t in cand], rtol=1e-12, atol=1e-12)
            assert list(rec["R"][bi]) == R
            assert list(rec["E"][bi]) == E
        assert list(st["R"][bi]) == R
        # the memory is the sequential update over the evictions in their order
        M, bs = om.memory_update(inp["K"][bi:bi + 1], inp["V"][bi:bi + 1],
                                 np.array(evicted)[None], w["W_phi"], lam)
        np.testing.assert_allclose(st["M"][bi:bi + 1], M, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(st["b"][bi:bi + 1], bs, rtol=1e-12, atol=1e-12)


def test_all_ties_keep_the_first_positions_and_match_one_shot_memory():
    # zero context: q^ = k^ = 0, so every score is exactly 0 and every choice
    # is a tie; the first B positions stay, the rest leave in ascending order
    # (range by range), so the memory equals the one-shot prefill's
    L, B = 60, 12
    wl, w, inp = _inputs(L)
    inp = dict(inp)
    inp["X"] = torch.zeros_like(inp["X"])
    inp["Q"] = torch.zeros_like(inp["Q"])
    st = _run(inp, w, wl.shape.lam, B, _ranges(L, 13))
    one = om.prefill_layer(inp["X"], inp["Q"], inp["K"], inp["V"], w["W_iq"], w["W_ik"],
                           w["w_ig"], w["W_phi"], wl.shape.lam, B)
    assert np.array_equal(st["R"][0], np.arange(B))
    assert np.array_equal(np.concatenate([c["E"][0] for c in st["chunks"]]), np.arange(B, L))
    np.testing.assert_allclose(st["M"], one["M"], rtol=1e-12, atol=1e-12)


def test_invariants_on_random_context():
    L, B, chunk = 200, 30, 48
    wl, w, inp = _inputs(L, batch=2, seed=9)
    st = _run(inp, w, wl.shape.lam, B, _ranges(L, chunk))
    for bi in range(2):
        seen = set()
        for (q0, q1), rec in zip(_ranges(L, chunk), st["chunks"]):
            R, E = list(rec["R"][bi]), list(rec["E"][bi])
            assert len(R) == min(B, q1)
            assert R == sorted(R) and E == sorted(E)
            assert not (set(E) & seen)
            seen |= set(E)
            assert set(R) | seen == set(range(q1)) and not (set(R) & seen)
