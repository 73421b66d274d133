"""GPU parity at the workloads' full sizes, in the launch configurations the
benchmark uses, on outputs the oracle can compute one by one:

* c2 (batch 4, L 16384, budgets 128, 256, 512 and 1024): pooled importance at
  sampled keys of one sequence, the whole selection, the whole compaction, the
  memory state of one sequence, two decode steps of one sequence;
* c3 (one 131072-token sequence, 8192-token chunked prefill, planted needles,
  budget 13107): importance at sampled keys and at every needle position,
  selection, compaction, memory state, two decode steps;
* c4 decode shape (batch 64, 2048 retained rows): two decode steps checked on
  sampled sequences;
* the full-cache decode the benchmark sets beside the evicted cache (c2, budget
  B = L = 16384, batch 4, memory empty): three steps on two sequences.
Decode steps are compared with the oracle's decode over the GPU's own memory
state, which is itself checked against the oracle's at the memory tolerance.
Sources: "IndexMem" technical summary §2.A (indexer, streaming pooled max,
pre-eviction), §1/§4 (top-B eviction, decoding time against the full cache),
§2.B (memory, readout).
"""
import math

import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import synth
from learned_kv_cache_indexmem_b200.layer import IndexMemLayer
from oracle import indexmem_oracle as om

from .parity import check_decode, check_memory, ill_conditioned, to_np, SCORE_TOL

pytestmark = pytest.mark.gpu


def _check_sampled_scores(I_gpu_row, I_ref, what):
    scale = max(np.abs(I_ref).max(), math.sqrt(np.mean(I_ref ** 2)))
    err = np.abs(I_gpu_row - I_ref).max()
    assert err <= SCORE_TOL * scale, "%s: score err %.3e > %.3e" % (what, err, SCORE_TOL * scale)


def _run_full(wl, B, dev, n_dec=2, ranges=None, needles=0, seq=0, n_keys=192):
    s = wl.shape
    w = synth.make_weights(s, wl.seed, dev)
    inp = synth.make_layer_inputs(wl, w, wl.seed, dev)
    dec = synth.make_decode_inputs(wl, w, max(n_dec, 8), wl.seed, dev)
    pos = None
    if needles:
        pos, _ = synth.plant_needles(wl, inp["K"], dec["q"], needles, wl.seed)
    b, L = wl.batch, wl.L
    cap = B + n_dec
    lay = IndexMemLayer.from_shape(s, w)
    st = lay.new_state(b, L, B, cap, dev)
    lay.score_and_evict(inp["X"], inp["Q"], inp["K"], inp["V"], st, B, q_ranges=ranges)
    lay.update_memory(inp["K"], inp["V"], st, B, chunk=wl.mem_chunk)
    outs = [lay.decode(dec["q"][i], dec["k_new"][i], dec["v_new"][i], st).clone() for i in range(n_dec)]
    lay.sync()

    # pooled importance at sampled keys of one sequence (+ edges, + needle keys)
    rng = np.random.default_rng(wl.seed)
    planted = [] if pos is None else pos.cpu().numpy().tolist()
    keys = np.unique(np.concatenate([rng.choice(L, n_keys, replace=False), [0, L - 2, L - 1],
                                     np.asarray(planted, dtype=np.int64)])).astype(np.int64)
    assert all(p in keys for p in planted)
    Xc, Qc = inp["X"][seq].cpu(), inp["Q"][seq].cpu()
    wc = {k: v.cpu() for k, v in w.items()}
    I_ref = om.importance_at_keys(Xc, Qc, wc["W_iq"], wc["W_ik"], wc["w_ig"], keys)
    I_gpu = to_np(st.running_max)
    _check_sampled_scores(I_gpu[seq, keys], I_ref, "%s keys" % wl.name)
    # selection over everything: the oracle's top-B of the GPU's scores
    R, E = om.select_budget(I_gpu, B)
    assert np.array_equal(st.idx_retained.cpu().numpy(), R)
    if B < L:
        assert np.array_equal(st.idx_evicted.cpu().numpy()[:, :L - B], E)
    # compaction, every sequence
    Rt = torch.from_numpy(R).to(dev)
    for bi in range(b):
        assert torch.equal(st.K_ret[bi, :B], inp["K"][bi, Rt[bi]])
        assert torch.equal(st.V_ret[bi, :B], inp["V"][bi, Rt[bi]])
    # memory state of one sequence (all KV heads)
    Kc, Vc = inp["K"][seq:seq + 1].cpu(), inp["V"][seq:seq + 1].cpu()
    M_ref, b_ref = om.memory_update(Kc, Vc, E[seq:seq + 1], wc["W_phi"], s.lam)
    M_gpu, b_gpu = to_np(st.M[seq:seq + 1]), to_np(st.bstab[seq:seq + 1])
    check_memory(M_gpu, b_gpu, M_ref, b_ref, wl.name)
    # decode steps of that sequence, over the memory state the GPU left
    W_phi = to_np(wc["W_phi"]); w_gate = to_np(wc["w_gate"])
    group = s.n_q_heads // s.n_kv_heads
    KR, VR = om.compact(to_np(Kc), to_np(Vc), R[seq:seq + 1], cap)
    clen = np.array([B])
    for i in range(n_dec):
        qc = to_np(dec["q"][i][seq:seq + 1]); kn = to_np(dec["k_new"][i][seq:seq + 1])
        vn = to_np(dec["v_new"][i][seq:seq + 1])
        o_ref, new_len, _, _, _ = om.decode_step(qc, kn, vn, KR, VR, clen, M_gpu, b_gpu, W_phi,
                                                 w_gate)
        KR[0, clen[0]] = kn[0]; VR[0, clen[0]] = vn[0]
        clen = new_len
        check_decode(to_np(outs[i][seq:seq + 1]), o_ref, ill_conditioned(b_gpu, qc, W_phi, group),
                     "%s decode %d" % (wl.name, i))
    assert st.cache_len.cpu().tolist() == [B + n_dec] * b
    lay.close()
    return pos, I_gpu


@pytest.mark.parametrize("B", [128, 256, 512, 1024])
def test_c2_full_size(cuda_device, B):
    _run_full(synth.WORKLOADS["c2"], B, cuda_device, seq=1)


def test_c3_full_size_chunked_with_needles(cuda_device):
    wl = synth.WORKLOADS["c3"]
    ranges = [(i, min(wl.L, i + wl.prefill_chunk)) for i in range(0, wl.L, wl.prefill_chunk)]
    pos, I_gpu = _run_full(wl, wl.budget, cuda_device, ranges=ranges, needles=wl.needles,
                           n_keys=96)
    assert pos is not None and len(pos) == wl.needles


def test_c4_decode_shape(cuda_device):
    wl = synth.WORKLOADS["c4"]
    s = wl.shape
    dev = cuda_device
    b, B, n_dec = wl.batch, wl.budget, 2
    w = synth.make_weights(s, wl.seed, dev)
    inp = synth.make_layer_inputs(wl, w, wl.seed, dev, L=B)     # the retained rows
    dec = synth.make_decode_inputs(wl, w, n_dec, wl.seed, dev)
    M0, b0 = synth.make_memory_state(s, b, wl.seed, dev)
    lay = IndexMemLayer.from_shape(s, w)
    st = lay.new_state(b, B + 1, B, B + n_dec, dev)
    st.K_ret[:, :B] = inp["K"]; st.V_ret[:, :B] = inp["V"]
    st.M.copy_(M0); st.bstab.copy_(b0)
    lay.workspace(b, B + 1, B, dev)
    outs = [lay.decode(dec["q"][i], dec["k_new"][i], dec["v_new"][i], st).clone() for i in range(n_dec)]
    lay.sync()
    W_phi = to_np(w["W_phi"]); w_gate = to_np(w["w_gate"])
    group = s.n_q_heads // s.n_kv_heads
    for seq in (0, 31, 63):
        KR = np.zeros((1, B + n_dec) + tuple(inp["K"].shape[2:])); VR = np.zeros_like(KR)
        KR[0, :B] = to_np(inp["K"][seq]); VR[0, :B] = to_np(inp["V"][seq])
        Mr, br = to_np(M0[seq:seq + 1]), to_np(b0[seq:seq + 1])
        clen = np.array([B])
        for i in range(n_dec):
            qc = to_np(dec["q"][i][seq:seq + 1]); kn = to_np(dec["k_new"][i][seq:seq + 1])
            vn = to_np(dec["v_new"][i][seq:seq + 1])
            o_ref, new_len, _, _, _ = om.decode_step(qc, kn, vn, KR, VR, clen, Mr, br, W_phi, w_gate)
            KR[0, clen[0]] = kn[0]; VR[0, clen[0]] = vn[0]
            clen = new_len
            check_decode(to_np(outs[i][seq:seq + 1]), o_ref, ill_conditioned(br, qc, W_phi, group),
                         "c4 seq %d step %d" % (seq, i))
    assert st.cache_len.cpu().tolist() == [B + n_dec] * b
    lay.close()


def test_c2_full_cache_decode(cuda_device):
    """Budget B = L: the whole 16384-token context of every sequence in the
    cache, memory empty (m = 0), three decode steps; sequences 0 and 3 are
    compared with the oracle's full softmax attention, the rest checked for
    their appended rows and lengths."""
    wl = synth.WORKLOADS["c2"]
    s = wl.shape
    dev = cuda_device
    b, L, n_dec = wl.batch, wl.L, 3
    w = synth.make_weights(s, wl.seed, dev)
    inp = synth.make_layer_inputs(wl, w, wl.seed, dev)
    dec = synth.make_decode_inputs(wl, w, n_dec, wl.seed, dev)
    lay = IndexMemLayer.from_shape(s, w)
    st = lay.new_state(b, L, L, L + n_dec, dev)        # M, b zero
    st.K_ret[:, :L] = inp["K"]; st.V_ret[:, :L] = inp["V"]
    st.cache_len.fill_(L)
    lay.workspace(b, L, L, dev)
    outs = [lay.decode(dec["q"][i], dec["k_new"][i], dec["v_new"][i], st).clone()
            for i in range(n_dec)]
    lay.sync()
    assert st.cache_len.cpu().tolist() == [L + n_dec] * b
    for i in range(n_dec):
        assert torch.equal(st.K_ret[:, L + i], dec["k_new"][i])
        assert torch.equal(st.V_ret[:, L + i], dec["v_new"][i])
    W_phi = to_np(w["W_phi"]); w_gate = to_np(w["w_gate"])
    M0 = np.zeros((1, s.n_kv_heads, s.mem_r, s.head_dim)); b0 = np.zeros((1, s.n_kv_heads, s.mem_r))
    for seq in (0, 3):
        KR = np.zeros((1, L + n_dec, s.n_kv_heads, s.head_dim)); VR = np.zeros_like(KR)
        KR[0, :L] = to_np(inp["K"][seq]); VR[0, :L] = to_np(inp["V"][seq])
        clen = np.array([L])
        for i in range(n_dec):
            qc = to_np(dec["q"][i][seq:seq + 1]); kn = to_np(dec["k_new"][i][seq:seq + 1])
            vn = to_np(dec["v_new"][i][seq:seq + 1])
            o_ref, new_len, o_attn, _, _ = om.decode_step(qc, kn, vn, KR, VR, clen, M0, b0, W_phi,
                                                          w_gate)
            assert np.array_equal(o_ref, o_attn)        # empty memory: plain attention
            KR[0, clen[0]] = kn[0]; VR[0, clen[0]] = vn[0]
            clen = new_len
            check_decode(to_np(outs[i][seq:seq + 1]), o_ref, None,
                         "full cache seq %d step %d" % (seq, i))
    lay.close()
