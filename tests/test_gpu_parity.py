"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle
on the same seeded inputs, stage by stage and end to end.

Stages and sources ("IndexMem" technical summary): §2.A indexer scores pooled
per key by a running max; §1/§4 top-B eviction; §2.B memory update and the
residual readout o = o_attn + g(q) m(q).
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import binding, synth
from oracle import indexmem_oracle as om

from .parity import (Case, check_decode, check_memory, check_scores, ill_conditioned, to_np,
                     SCORE_TOL)

pytestmark = pytest.mark.gpu

W = synth.WORKLOADS


def _prefill_gpu(case, B, cap=None, ranges=None):
    lay = case.layer()
    dev = case.device
    cap = B + 4 if cap is None else cap
    st = lay.new_state(case.batch, case.L, B, cap, dev)
    d = case.in_dev
    lay.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st, B, q_ranges=ranges)
    lay.sync()
    return lay, st


def _check_selection(st, I_gpu, I_ref, B, L):
    R_g = st.idx_retained.cpu().numpy()
    E_g = st.idx_evicted.cpu().numpy()[:, :L - B]
    # bit-exact: the oracle's top-B of the GPU's scores
    R_o, E_o = om.select_budget(I_gpu, B)
    assert np.array_equal(R_g, R_o), "retained set differs from the oracle's selection"
    assert np.array_equal(E_g, E_o), "evicted set differs from the oracle's selection"
    # and against the oracle's own scores: only near-ties at the threshold may flip
    R_r, _ = om.select_budget(I_ref, B)
    for bi in range(I_ref.shape[0]):
        diff = set(R_g[bi]) ^ set(R_r[bi])
        if diff:
            ref = I_ref[bi]
            scale = max(np.abs(ref).max(), math.sqrt(np.mean(ref ** 2)))
            thr = np.sort(ref)[::-1][B - 1]
            for t in diff:
                assert abs(ref[t] - thr) <= 2 * SCORE_TOL * scale, (bi, t, ref[t], thr)


@pytest.mark.parametrize("name,L,batch,B", [
    ("c0", None, None, 128),
    ("c0", 777, 2, 100),        # ragged L, batch 2
    ("c1", None, None, 410),
    ("c1", 1000, 1, 1),         # budget 1
    ("c1", 300, 3, 300),        # budget = L: nothing evicted
])
def test_prefill_parity(cuda_device, name, L, batch, B):
    case = Case(W[name], cuda_device, L=L, batch=batch, n_decode=1)
    lay, st = _prefill_gpu(case, B)
    qhat, khat, gate = case.oracle_features()
    I_ref = om.pooled_importance(qhat, khat, gate)
    I_gpu = to_np(st.running_max)
    check_scores(I_gpu, I_ref, name)
    _check_selection(st, I_gpu, I_ref, B, case.L)
    R = st.idx_retained.long().cpu()
    for bi in range(case.batch):
        assert torch.equal(st.K_ret[bi, :B].cpu(), case.in_cpu["K"][bi, R[bi]])
        assert torch.equal(st.V_ret[bi, :B].cpu(), case.in_cpu["V"][bi, R[bi]])
    lay.close()


def test_chunked_prefill_equals_one_shot(cuda_device):
    case = Case(W["c1"], cuda_device, L=2500, batch=2, n_decode=1)
    B = 250
    _, st1 = _prefill_gpu(case, B)
    ranges = [(0, 1024), (1024, 2048), (2048, 2500)]
    _, st2 = _prefill_gpu(case, B, ranges=ranges)
    assert torch.equal(st1.running_max, st2.running_max)
    assert torch.equal(st1.idx_retained, st2.idx_retained)
    qhat, khat, gate = case.oracle_features()
    I_ref = None
    for q0, q1 in ranges:
        I_ref = om.pooled_importance(qhat, khat, gate, q_begin=q0, q_end=q1, prev=I_ref)
    check_scores(to_np(st2.running_max), I_ref, "chunked")


def test_split_calls_equal_score_and_evict(cuda_device):
    """imem_indexer_features + imem_indexer_score per query range, then
    imem_select_compact, give bitwise the outputs of imem_score_and_evict."""
    case = Case(W["c1"], cuda_device, L=2500, batch=2, n_decode=1)
    B = 250
    ranges = [(0, 1024), (1024, 2048), (2048, 2500)]
    _, st1 = _prefill_gpu(case, B, ranges=ranges)
    lay = case.layer()
    st2 = lay.new_state(case.batch, case.L, B, B + 4, cuda_device)
    ws = lay.workspace(case.batch, case.L, B, cuda_device)
    d = case.in_dev
    for q0, q1 in ranges:
        binding.indexer_features(lay.ctx, case.batch, case.L, d["X"], d["Q"], st2.running_max,
                                 q0, q1, ws)
        binding.indexer_score(lay.ctx, case.batch, case.L, st2.running_max, q0, q1, ws)
    binding.select_compact(lay.ctx, case.batch, case.L, B, st2.running_max, d["K"], d["V"],
                           st2.idx_retained, st2.idx_evicted, st2.K_ret, st2.V_ret, B + 4, ws)
    lay.sync()
    assert torch.equal(st1.running_max, st2.running_max)
    assert torch.equal(st1.idx_retained, st2.idx_retained)
    assert torch.equal(st1.idx_evicted, st2.idx_evicted)
    assert torch.equal(st1.K_ret[:, :B], st2.K_ret[:, :B])
    assert torch.equal(st1.V_ret[:, :B], st2.V_ret[:, :B])
    lay.close()


def test_constant_context_ties_go_to_lower_positions(cuda_device):
    """Identical tokens give identical scores for every key; the retained set is
    then the first B positions."""
    case = Case(W["c1"], cuda_device, L=640, batch=1, n_decode=1)
    for k in ("X", "Q", "K", "V"):
        case.in_dev[k][:] = case.in_dev[k][:, :1]
    B = 100
    _, st = _prefill_gpu(case, B)
    I = st.running_max.cpu()
    assert torch.all(I == I[0, 0])
    assert torch.equal(st.idx_retained.cpu()[0], torch.arange(B, dtype=torch.int32))
    assert torch.equal(st.idx_evicted.cpu()[0, :640 - B], torch.arange(B, 640, dtype=torch.int32))


def _workload(name):
    """A workload by name; "c0-bf16" is the tiny c0 layer in bf16 (head dim 64
    on the bf16 tensor-core memory path)."""
    if name == "c0-bf16":
        wl = W["c0"]
        return dataclasses.replace(wl, shape=dataclasses.replace(wl.shape, dtype="bf16"))
    return W[name]


@pytest.mark.parametrize("name,L,batch,n_e,chunk", [
    ("c0", None, None, 896, 64),
    ("c0-bf16", None, 2, 896, 64),
    ("c0-bf16", 700, 1, 699, 64),
    ("c1", None, None, 3686, 512),
    ("c1", 1500, 3, 1499, 128),
    ("c1", 600, 2, 0, 64),
])
def test_memory_update_parity(cuda_device, name, L, batch, n_e, chunk):
    case = Case(_workload(name), cuda_device, L=L, batch=batch, n_decode=1)
    E = synth.make_index_subset(case.batch, case.L, n_e, case.seed)
    M0, b0 = synth.make_memory_state(case.shape, case.batch, case.seed)
    lay = case.layer()
    lay.workspace(case.batch, case.L, max(1, case.L - n_e), cuda_device)
    M = M0.to(cuda_device).clone()
    b = b0.to(cuda_device).clone()
    Ed = E.to(cuda_device) if n_e else None
    binding.update_memory(lay.ctx, case.batch, case.L, case.in_dev["K"], case.in_dev["V"], Ed,
                          n_e, chunk, M, b, lay._ws)
    lay.sync()
    M_ref, b_ref = om.memory_update(case.in_cpu["K"], case.in_cpu["V"], E.numpy(),
                                    case.w_cpu["W_phi"], case.shape.lam, M0, b0)
    check_memory(to_np(M), to_np(b), M_ref, b_ref, name)
    if n_e == 0:
        assert torch.equal(M.cpu(), M0) and torch.equal(b.cpu(), b0)
    lay.close()


def _decode_case(case, cap, lens, gate_override=None):
    """Retained cache = the first len rows of the layer's K/V; memory state drawn
    by the generator. Returns (layer, state, cpu copies)."""
    lay = case.layer(gate_override=gate_override)
    dev = case.device
    b_ = case.batch
    st = lay.new_state(b_, case.L, 1, cap, dev)
    for bi in range(b_):
        n = lens[bi]
        st.K_ret[bi, :n] = case.in_dev["K"][bi, :n]
        st.V_ret[bi, :n] = case.in_dev["V"][bi, :n]
    st.cache_len[:] = torch.tensor(lens, dtype=torch.int32, device=dev)
    M0, b0 = synth.make_memory_state(case.shape, b_, case.seed)
    st.M.copy_(M0)
    st.bstab.copy_(b0)
    lay.workspace(b_, case.L, 1, dev)
    return lay, st, M0.numpy().astype(np.float64), b0.numpy().astype(np.float64)


@pytest.mark.parametrize("name,batch,lens,cap,steps", [
    ("c0", 1, [128], 144, 16),
    ("c1", 1, [410], 410 + 256, 256),
    ("c1", 3, [410, 37, 1], 420, 8),        # ragged cache lengths
    ("c1", 2, [2000, 1500], 2100, 4),       # several splits
    ("c1", 4, [128, 100, 60, 1], 640, 8),   # short ragged caches, 4 splits
    # blocks one stage longer than the ring (6 splits of up to 256 rows) and,
    # for the shorter caches, blocks that fit it
    ("c1", 4, [1500, 1200, 1100, 700], 1536, 4),
    # blocks several stages longer than the ring (15 splits of up to 288 rows)
    ("c1", 1, [4000], 4100, 3),
])
def test_decode_parity(cuda_device, name, batch, lens, cap, steps):
    L = max(max(lens), 64)
    case = Case(W[name], cuda_device, L=L, batch=batch, n_decode=steps)
    group = case.shape.n_q_heads // case.shape.n_kv_heads
    W_phi = case.w_cpu["W_phi"].numpy().astype(np.float64)
    w_gate = case.w_cpu["w_gate"].numpy().astype(np.float64)
    for gate_override in (None, 0.0):
        lay, st, M0, b0 = _decode_case(case, cap, lens, gate_override)
        KR = np.zeros((batch, cap) + case.in_cpu["K"].shape[2:])
        VR = np.zeros_like(KR)
        for bi in range(batch):
            KR[bi, :lens[bi]] = to_np(case.in_cpu["K"][bi, :lens[bi]])
            VR[bi, :lens[bi]] = to_np(case.in_cpu["V"][bi, :lens[bi]])
        clen = np.array(lens)
        for s in range(steps):
            q, kn, vn = (case.dec_dev[k][s] for k in ("q", "k_new", "v_new"))
            out = lay.decode(q, kn, vn, st)
            lay.sync()
            qc, knc, vnc = (to_np(case.dec_cpu[k][s]) for k in ("q", "k_new", "v_new"))
            o_ref, new_len, _, _, _ = om.decode_step(qc, knc, vnc, KR, VR, clen, M0, b0, W_phi,
                                                     w_gate, gate_override=gate_override)
            for bi in range(batch):
                KR[bi, clen[bi]] = knc[bi]
                VR[bi, clen[bi]] = vnc[bi]
            clen = new_len
            mask = None if gate_override is not None else ill_conditioned(b0, qc, W_phi, group)
            check_decode(to_np(out), o_ref, mask, "%s step %d gate %s" % (name, s, gate_override))
        assert np.array_equal(st.cache_len.cpu().numpy(), clen)
        # the appended rows are in the cache
        for bi in range(batch):
            n = clen[bi]
            assert np.array_equal(to_np(st.K_ret[bi, :n]), KR[bi, :n])
        lay.close()


def test_decode_into_full_cache_reports_and_skips(cuda_device):
    case = Case(W["c1"], cuda_device, L=64, batch=2, n_decode=1)
    lay, st, _, _ = _decode_case(case, 40, [40, 10])
    before = st.K_ret.clone()
    out = torch.full_like(case.dec_dev["q"][0], 7.0)
    lay.decode(case.dec_dev["q"][0], case.dec_dev["k_new"][0], case.dec_dev["v_new"][0], st, out=out)
    with pytest.raises(binding.IndexMemError) as ei:
        lay.sync()
    assert ei.value.name == "IMEM_ERR_SHAPE"
    assert st.cache_len.cpu().tolist() == [40, 11]
    assert torch.all(out[0] == 7.0)          # full sequence: output row untouched
    assert torch.equal(st.K_ret[0], before[0])
    lay.sync()                                # error was cleared
    lay.close()


@pytest.mark.parametrize("name,B,steps", [("c0", 128, 16), ("c1", 410, 32)])
def test_end_to_end_parity(cuda_device, name, B, steps):
    """Whole path: prefill (score, select, compact), memory update, decode steps.
    The retained set is the one integer decision taken from floating point: it is
    checked bit-exactly as the oracle's selection on the GPU's scores, and the
    oracle's downstream stages continue from that selection; likewise the
    memory state is checked against the oracle's at its tolerance and the
    oracle's decode steps read the GPU's state."""
    case = Case(W[name], cuda_device, n_decode=steps)
    cap = B + steps
    lay, st = _prefill_gpu(case, B, cap=cap)
    lay.update_memory(case.in_dev["K"], case.in_dev["V"], st, B, chunk=512)
    outs = []
    for s in range(steps):
        outs.append(to_np(lay.decode(case.dec_dev["q"][s], case.dec_dev["k_new"][s],
                                     case.dec_dev["v_new"][s], st)))
    lay.sync()
    qhat, khat, gate = case.oracle_features()
    I_ref = om.pooled_importance(qhat, khat, gate)
    I_gpu = to_np(st.running_max)
    check_scores(I_gpu, I_ref, name)
    _check_selection(st, I_gpu, I_ref, B, case.L)
    R, E = om.select_budget(I_gpu, B)
    KR, VR = om.compact(to_np(case.in_cpu["K"]), to_np(case.in_cpu["V"]), R, cap)
    M_ref, b_ref = om.memory_update(case.in_cpu["K"], case.in_cpu["V"], E, case.w_cpu["W_phi"],
                                    case.shape.lam)
    M_gpu, b_gpu = to_np(st.M), to_np(st.bstab)
    check_memory(M_gpu, b_gpu, M_ref, b_ref, name)
    W_phi = case.w_cpu["W_phi"].numpy().astype(np.float64)
    w_gate = case.w_cpu["w_gate"].numpy().astype(np.float64)
    group = case.shape.n_q_heads // case.shape.n_kv_heads
    clen = np.full(case.batch, B)
    for s in range(steps):
        qc, knc, vnc = (to_np(case.dec_cpu[k][s]) for k in ("q", "k_new", "v_new"))
        # decode reads the memory state the GPU left (checked above against the
        # oracle's at its own tolerance), as selection is checked on the GPU's scores
        o_ref, new_len, _, _, _ = om.decode_step(qc, knc, vnc, KR, VR, clen, M_gpu, b_gpu, W_phi,
                                                 w_gate)
        for bi in range(case.batch):
            KR[bi, clen[bi]] = knc[bi]
            VR[bi, clen[bi]] = vnc[bi]
        clen = new_len
        check_decode(outs[s], o_ref, ill_conditioned(b_gpu, qc, W_phi, group),
                     "%s step %d" % (name, s))
    lay.close()
