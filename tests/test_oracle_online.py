"""Pins of the online-eviction decode oracle ("IndexMem" technical summary
§2.B, memory updated online during inference; §2.A, the indexer's pooled
importance): a decode step with online eviction is pre-eviction with a
one-token query range, so a run of steps must reproduce the (brute-force
pinned) pre-eviction oracle over the same tokens; and exact special cases."""
import numpy as np
import torch

from learned_kv_cache_indexmem_b200 import synth
from oracle import indexmem_oracle as om


def _setup(L, batch, seed):
    wl = synth.WORKLOADS["c0"]
    w = synth.make_weights(wl.shape, seed)
    inp = synth.make_layer_inputs(wl, w, seed, L=L, batch=batch)
    return wl, w, inp


def _online_state(inp, w, st, B):
    """Cache state (slots in position order) after a pre-eviction prefill."""
    R = st["R"]
    last = st["chunks"][-1]
    b = R.shape[0]
    _, khat, _ = om.indexer_features(inp["X"], inp["Q"], w["W_iq"], w["W_ik"], w["w_ig"])
    K, V = om.f64(inp["K"]), om.f64(inp["V"])
    Hkv, d = K.shape[2:]
    KR = np.zeros((b, B + 1, Hkv, d)); VR = np.zeros_like(KR)
    khR = np.zeros((b, B + 1, khat.shape[-1])); IR = np.zeros((b, B + 1))
    posR = np.zeros((b, B + 1), dtype=np.int64)
    for bi in range(b):
        idx = np.searchsorted(last["cand"][bi], R[bi])
        KR[bi, :B], VR[bi, :B] = K[bi, R[bi]], V[bi, R[bi]]
        khR[bi, :B] = khat[bi, R[bi]]
        IR[bi, :B] = last["I"][bi, idx]
        posR[bi, :B] = R[bi]
    return KR, VR, khR, IR, posR


def test_online_steps_equal_pre_eviction_with_one_token_ranges():
    L0, L, B, C, batch = 48, 60, 10, 16, 2
    wl, w, inp = _setup(L, batch, seed=7)
    lam = wl.shape.lam
    pre = [(q, min(L0, q + C)) for q in range(0, L0, C)]
    ref = om.prefill_streaming(inp["X"], inp["Q"], inp["K"], inp["V"], w["W_iq"], w["W_ik"],
                               w["w_ig"], w["W_phi"], lam, B, pre + [(t, t + 1) for t in range(L0, L)])
    head = {k: v[:, :L0] for k, v in inp.items()}
    st = om.prefill_streaming(head["X"], head["Q"], head["K"], head["V"], w["W_iq"], w["W_ik"],
                              w["w_ig"], w["W_phi"], lam, B, pre)
    KR, VR, khR, IR, posR = _online_state(head, w, st, B)
    M, bs = st["M"], st["b"]
    for i, t in enumerate(range(L0, L)):
        o, ev, new = om.decode_step_online(
            om.f64(inp["X"][:, t]), om.f64(inp["Q"][:, t]), om.f64(inp["K"][:, t]),
            om.f64(inp["V"][:, t]), KR, VR, khR, IR, posR, np.full(batch, t), M, bs,
            w["W_iq"], w["W_ik"], w["w_ig"], w["W_phi"], w["w_gate"], lam)
        rec = ref["chunks"][len(pre) + i]
        assert np.array_equal(ev, rec["E"][:, 0]), "step %d" % i
        KR, VR, khR, IR, posR = new["K_R"], new["V_R"], new["khat_R"], new["I_R"], new["pos_R"]
        M, bs = new["M"], new["b"]
        for bi in range(batch):
            assert np.array_equal(np.sort(posR[bi, :B]), rec["R"][bi])
            # importances carried for the retained tokens match the reference's
            idx = np.searchsorted(rec["cand"][bi], posR[bi, :B])
            np.testing.assert_allclose(IR[bi, :B], rec["I"][bi, idx], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(M, ref["M"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(bs, ref["b"], rtol=1e-12, atol=1e-12)


def test_all_ties_evict_the_newest_token():
    # zero hidden states and queries: every indexer score is exactly 0, so the
    # newest token (highest position) leaves at every step and the cache is
    # unchanged; the memory takes the decoded tokens in order
    L0, steps, B = 20, 6, 8
    wl, w, inp = _setup(L0 + steps, 1, seed=2)
    lam = wl.shape.lam
    inp = dict(inp)
    inp["X"] = torch.zeros_like(inp["X"])
    inp["Q"] = torch.zeros_like(inp["Q"])
    head = {k: v[:, :L0] for k, v in inp.items()}
    st = om.prefill_streaming(head["X"], head["Q"], head["K"], head["V"], w["W_iq"], w["W_ik"],
                              w["w_ig"], w["W_phi"], lam, B, [(0, L0)])
    KR, VR, khR, IR, posR = _online_state(head, w, st, B)
    M, bs = st["M"], st["b"]
    for t in range(L0, L0 + steps):
        _, ev, new = om.decode_step_online(
            np.zeros((1, wl.shape.hidden)), np.zeros((1,) + tuple(inp["Q"].shape[2:])),
            om.f64(inp["K"][:, t]), om.f64(inp["V"][:, t]), KR, VR, khR, IR, posR,
            np.array([t]), M, bs, w["W_iq"], w["W_ik"], w["w_ig"], w["W_phi"], w["w_gate"], lam)
        assert ev[0] == t
        assert np.array_equal(new["pos_R"][0, :B], np.arange(B))
        KR, VR, khR, IR, posR = new["K_R"], new["V_R"], new["khat_R"], new["I_R"], new["pos_R"]
        M, bs = new["M"], new["b"]
    E = np.concatenate([np.arange(B, L0), np.arange(L0, L0 + steps)])[None]
    M_ref, b_ref = om.memory_update(inp["K"], inp["V"], E, w["W_phi"], lam)
    np.testing.assert_allclose(M, M_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(bs, b_ref, rtol=1e-12, atol=1e-12)
