"""Pre-eviction during chunked prefill ("IndexMem" technical summary §2.A,
eviction before the full prefill) through the C ABI against the oracle, range
by range: the candidates' pooled importances within the score tolerance, the
selection bit-exact on the GPU's own importances, the evicted positions and
their order, the memory against the sequential update in eviction order, and
the final compaction."""
import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import binding, synth
from oracle import indexmem_oracle as om

from .parity import Case, check_memory, check_scores, to_np

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.mark.parametrize("name,L,B,chunk,batch", [
    ("c0", 1024, 128, 256, 1),
    ("c1", 1000, 100, 300, 2),     # ragged last range, B not a multiple of anything
    ("c1", 640, 64, 64, 1),        # ranges as long as the budget
    ("c1", 700, 900, 256, 1),      # budget above the context: nothing leaves
    ("c1", 2100, 410, 1024, 1),    # c1-like budget, several score tiles per range
])
def test_pre_eviction_parity(cuda_device, name, L, B, chunk, batch):
    case = Case(W[name], cuda_device, L=L, batch=batch, n_decode=1)
    lay = case.layer()
    nB = min(B, L)
    st = lay.new_state(batch, L, B, nB + 4, cuda_device)
    d = case.in_dev
    recs = lay.prefill_evict(d["X"], d["Q"], d["K"], d["V"], st, B, chunk, mem_chunk=64,
                             record=True)
    lay.sync()
    qhat, khat, gate = case.oracle_features()
    R_prev = [np.zeros(0, dtype=np.int64) for _ in range(batch)]
    I_prev = [np.zeros(0) for _ in range(batch)]
    evicted = [[] for _ in range(batch)]
    for rec in recs:
        q0, q1 = rec["range"]
        I_gpu = to_np(rec["I"])
        ret_gpu = to_np(rec["retained"]).astype(np.int64)
        ev_gpu = to_np(rec["evicted"]).astype(np.int64)
        for bi in range(batch):
            cand = np.concatenate([R_prev[bi], np.arange(q0, q1)])
            assert I_gpu.shape[1] == len(cand)
            prev = np.full((1, L), -np.inf)
            prev[0, R_prev[bi]] = I_prev[bi]      # what the GPU carried
            I_ref = om.pooled_importance(qhat[bi:bi + 1], khat[bi:bi + 1], gate[bi:bi + 1],
                                         q_begin=q0, q_end=q1, prev=prev, keys=cand)
            check_scores(I_gpu[bi:bi + 1], I_ref, "%s range %d-%d" % (name, q0, q1))
            if len(cand) > B:
                ri, ei = om.select_budget(I_gpu[bi:bi + 1], B)
                R_exp, E_exp, I_prev[bi] = cand[ri[0]], cand[ei[0]], I_gpu[bi, ri[0]]
            else:
                R_exp, E_exp, I_prev[bi] = cand, np.zeros(0, dtype=np.int64), I_gpu[bi]
            assert np.array_equal(ret_gpu[bi], R_exp), "%s range %d-%d retained" % (name, q0, q1)
            assert np.array_equal(ev_gpu[bi], E_exp), "%s range %d-%d evicted" % (name, q0, q1)
            R_prev[bi] = R_exp
            evicted[bi] += list(E_exp)
    # the memory: the sequential update over each sequence's evictions in order
    M_ref, b_ref = om.memory_update(case.in_cpu["K"], case.in_cpu["V"], np.array(evicted),
                                    case.w_cpu["W_phi"], case.shape.lam)
    check_memory(to_np(st.M), to_np(st.bstab), M_ref, b_ref, name)
    # the final compaction
    final = to_np(st.idx_retained[:, :nB]).astype(np.int64)
    for bi in range(batch):
        assert np.array_equal(final[bi], R_prev[bi])
        assert np.array_equal(to_np(st.K_ret[bi, :nB]), to_np(case.in_cpu["K"][bi, final[bi]]))
        assert np.array_equal(to_np(st.V_ret[bi, :nB]), to_np(case.in_cpu["V"][bi, final[bi]]))
    assert np.all(to_np(st.cache_len) == nB)
    lay.close()


def test_single_range_equals_one_shot_prefill(cuda_device):
    # one range over the whole context: the candidates are all tokens, so the
    # selection, the evicted set and the memory are the one-shot prefill's
    L, B, batch = 900, 90, 2
    case = Case(W["c1"], cuda_device, L=L, batch=batch, n_decode=1)
    d = case.in_dev
    a = case.layer()
    st_a = a.new_state(batch, L, B, B, cuda_device)
    a.prefill_evict(d["X"], d["Q"], d["K"], d["V"], st_a, B, L, mem_chunk=64)
    b_ = case.layer()
    st_b = b_.new_state(batch, L, B, B, cuda_device)
    b_.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st_b, B)
    b_.update_memory(d["K"], d["V"], st_b, B, chunk=64)
    a.sync()
    b_.sync()
    assert np.array_equal(to_np(st_a.idx_retained), to_np(st_b.idx_retained))
    assert np.array_equal(to_np(st_a.K_ret), to_np(st_b.K_ret))
    np.testing.assert_array_equal(to_np(st_a.M), to_np(st_b.M))
    np.testing.assert_array_equal(to_np(st_a.bstab), to_np(st_b.bstab))
    a.close()
    b_.close()


def test_memory_between_ranges_after_join(cuda_device):
    # each range's memory update runs on the context's second stream beside the
    # next range's prologue and scoring; after imem_join the caller's stream
    # sees M and bstab with every eviction so far, range by range
    L, B, chunk, batch = 2100, 410, 512, 2
    case = Case(W["c1"], cuda_device, L=L, batch=batch, n_decode=1)
    lay = case.layer()
    st = lay.new_state(batch, L, B, B + 4, cuda_device)
    d = case.in_dev
    ws = lay.workspace_evict(batch, L, B, chunk, cuda_device)
    ev = torch.empty(batch * chunk, dtype=torch.int32, device=cuda_device)
    evicted = [[] for _ in range(batch)]
    checked = 0
    for q0 in range(0, L, chunk):
        q1 = min(L, q0 + chunk)
        n_ev = max(0, min(B, q0) + (q1 - q0) - B)
        binding.prefill_evict_chunk(lay.ctx, batch, L, B, chunk, d["X"], d["Q"], d["K"], d["V"],
                                    q0, q1, st.idx_retained, ev, None, st.M, st.bstab, 64,
                                    q1 == L, st.K_ret, st.V_ret, st.K_ret.shape[1], ws)
        binding.join(lay.ctx)
        e = to_np(ev[:batch * n_ev].view(batch, n_ev)).astype(np.int64)
        for bi in range(batch):
            evicted[bi] += list(e[bi])
        if n_ev:
            M_ref, b_ref = om.memory_update(case.in_cpu["K"], case.in_cpu["V"], np.array(evicted),
                                            case.w_cpu["W_phi"], case.shape.lam)
            check_memory(to_np(st.M), to_np(st.bstab), M_ref, b_ref,
                         "after range %d-%d" % (q0, q1))
            checked += 1
    assert checked >= 3
    lay.sync()
    lay.close()
