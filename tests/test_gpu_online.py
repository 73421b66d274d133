"""Decode-time online eviction ("IndexMem" technical summary §2.B, memory
updated online during inference; §2.A, pooled importance) through the C ABI
against the oracle, step by step from the GPU's own state before each step:
the output; the B + 1 candidates' importances the GPU used (slot B keeps the
token that left) against the oracle's within the score tolerance; the evicted
token bit-exactly as the least important of those importances (ties: the
higher position leaves); the memory updated with it; and the cache rows after
the move."""
import math

import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import synth
from oracle import indexmem_oracle as om

from .parity import SCORE_TOL, Case, check_decode, check_memory, ill_conditioned, to_np

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.mark.parametrize("name,L,B,steps,batch", [
    ("c0", 512, 64, 12, 1),
    ("c1", 1024, 128, 20, 2),
    ("c1", 600, 300, 8, 1),      # several score CTAs per sequence
])
def test_online_eviction_parity(cuda_device, name, L, B, steps, batch):
    case = Case(W[name], cuda_device, L=L + steps, batch=batch, n_decode=1)
    s = case.shape
    lay = case.layer()
    cap = B + 1
    st = lay.new_state(batch, L, B, cap, cuda_device)
    d = {k: v[:, :L].contiguous() for k, v in case.in_dev.items()}
    lay.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st, B)
    lay.update_memory(d["K"], d["V"], st, B, chunk=64)
    on = lay.online_init(st, B, L)
    lay.sync()
    assert np.array_equal(to_np(on.pos_ret[:, :B]), to_np(st.idx_retained))
    assert np.all(to_np(on.next_pos) == L)
    w = case.w_cpu
    W_phi = w["W_phi"].numpy().astype(np.float64)
    group = s.n_q_heads // s.n_kv_heads
    K_all, V_all = to_np(case.in_cpu["K"]), to_np(case.in_cpu["V"])
    for i in range(steps):
        t = L + i
        pre = {"K": to_np(st.K_ret), "V": to_np(st.V_ret), "kh": to_np(on.khat_ret),
               "I": to_np(on.I_ret), "pos": to_np(on.pos_ret).astype(np.int64),
               "M": to_np(st.M), "b": to_np(st.bstab)}
        x, q, kn, vn = (case.in_dev[k][:, t].contiguous() for k in ("X", "Q", "K", "V"))
        out = lay.decode_online(x, q, kn, vn, st, on, B)
        lay.sync()
        xc, qc, knc, vnc = (to_np(case.in_cpu[k][:, t]) for k in ("X", "Q", "K", "V"))
        o_ref, ev_ref, new = om.decode_step_online(
            xc, qc, knc, vnc, pre["K"], pre["V"], pre["kh"][..., :s.idx_dim], pre["I"],
            pre["pos"], np.full(batch, t), pre["M"], pre["b"], w["W_iq"], w["W_ik"], w["w_ig"],
            W_phi, w["w_gate"], s.lam)
        what = "%s step %d" % (name, i)
        check_decode(to_np(out), o_ref, ill_conditioned(pre["b"], qc, W_phi, group), what)
        ev = to_np(on.evicted).astype(np.int64)
        pos_after = on.pos_ret.cpu().numpy().astype(np.int64)
        I_after = on.I_ret.cpu().numpy()                 # float32, as the GPU compared them
        # the oracle's importances of the B + 1 candidates from the GPU's state
        qh, kh_new, g = om.indexer_features(xc[:, None], qc[:, None], w["W_iq"], w["W_ik"],
                                            w["w_ig"])
        qt = np.einsum("bh,bhd->bd", g[:, 0], qh[:, 0]) / math.sqrt(s.idx_dim)
        for bi in range(batch):
            cand_pos = list(pre["pos"][bi, :B]) + [t]
            I_cand = np.concatenate([
                np.maximum(pre["I"][bi, :B], pre["kh"][bi, :B, :s.idx_dim] @ qt[bi]),
                [kh_new[bi, 0] @ qt[bi]]])
            scale = max(np.abs(I_cand).max(), math.sqrt(np.mean(I_cand ** 2)))
            # slots [0, B] after the step are the step's B + 1 candidates, slot B
            # the one that left
            assert sorted(pos_after[bi, :B + 1]) == sorted(cand_pos), what
            assert pos_after[bi, B] == ev[bi], what
            for j in range(B + 1):
                p = pos_after[bi, j]
                assert abs(float(I_after[bi, j]) - I_cand[cand_pos.index(p)]) <= \
                    SCORE_TOL * scale, "%s: importance of %d" % (what, p)
            # the eviction, bit-exact on the GPU's importances: the least
            # important leaves, ties to the higher position (-0 == +0)
            Ig = I_after[bi, :B + 1].astype(np.float32) + np.float32(0.0)
            low = np.flatnonzero(Ig == Ig.min())
            assert ev[bi] == pos_after[bi, low].max(), "%s: eviction" % what
            # the cache after the move: rows by position, slot B the evicted row
            for j in range(B + 1):
                p = pos_after[bi, j]
                assert np.array_equal(to_np(st.K_ret[bi, j]), K_all[bi, p]), what
                assert np.array_equal(to_np(st.V_ret[bi, j]), V_all[bi, p]), what
        # the memory: the state before the step updated with the GPU's choice
        E = np.array([[ev[bi]] for bi in range(batch)])
        M_ref, b_ref = om.memory_update(case.in_cpu["K"], case.in_cpu["V"], E, W_phi, s.lam,
                                        M0=pre["M"], b0=pre["b"])
        check_memory(to_np(st.M), to_np(st.bstab), M_ref, b_ref, what)
        assert np.all(to_np(st.cache_len) == B)
        assert np.all(to_np(on.next_pos) == t + 1)
    lay.close()


def test_online_steps_back_to_back_equal_synchronised_steps(cuda_device):
    """The same online steps from the same state, (a) with a host
    synchronisation after every step, (b) enqueued back to back, (c) replayed
    as one CUDA graph: the kernels are deterministic, so outputs, evicted
    positions, cache rows, importances and memory must agree bitwise. A missed
    ordering between the steps (the features on the second stream, the next
    attention step's early loads after the eviction) would show here."""
    B, L, steps, batch = 128, 1024, 12, 2
    case = Case(W["c1"], cuda_device, L=L + steps, batch=batch, n_decode=1)
    lay = case.layer()
    cap = B + 1
    st = lay.new_state(batch, L, B, cap, cuda_device)
    d = {k: v[:, :L].contiguous() for k, v in case.in_dev.items()}
    lay.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st, B)
    lay.update_memory(d["K"], d["V"], st, B, chunk=64)
    on = lay.online_init(st, B, L)
    lay.sync()
    names = ("K_ret", "V_ret", "M", "bstab", "cache_len")
    onames = ("khat_ret", "I_ret", "pos_ret", "next_pos", "evicted")
    init = ({k: getattr(st, k).clone() for k in names}, {k: getattr(on, k).clone() for k in onames})

    def restore():
        for k in names:
            getattr(st, k).copy_(init[0][k])
        for k in onames:
            getattr(on, k).copy_(init[1][k])
        lay.invalidate_decode(batch)

    toks = [tuple(case.in_dev[k][:, L + i].contiguous() for k in ("X", "Q", "K", "V"))
            for i in range(steps)]
    outs = [torch.empty_like(toks[0][1]) for _ in range(steps)]
    evs = [torch.empty_like(on.evicted) for _ in range(steps)]

    def run(sync):
        for i, (x, q, kn, vn) in enumerate(toks):
            lay.decode_online(x, q, kn, vn, st, on, B, out=outs[i])
            evs[i].copy_(on.evicted)
            if sync:
                lay.sync()

    def snapshot():
        torch.cuda.synchronize()
        return ([o.clone() for o in outs], [e.clone() for e in evs],
                {k: getattr(st, k).clone() for k in names},
                {k: getattr(on, k).clone() for k in onames})

    restore(); run(True); ref = snapshot()
    restore(); run(False); lay.sync(); b2b = snapshot()
    s = torch.cuda.Stream(cuda_device)
    restore(); torch.cuda.synchronize()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i, (x, q, kn, vn) in enumerate(toks):
                lay.decode_online(x, q, kn, vn, st, on, B, out=outs[i], stream=s)
                evs[i].copy_(on.evicted)
    torch.cuda.synchronize()
    restore(); torch.cuda.synchronize()
    g.replay(); torch.cuda.synchronize(); lay.sync()
    gr = snapshot()
    for what, got in (("back to back", b2b), ("graph", gr)):
        for i in range(steps):
            assert torch.equal(got[0][i], ref[0][i]), "%s: output of step %d" % (what, i)
            assert torch.equal(got[1][i], ref[1][i]), "%s: eviction of step %d" % (what, i)
        for k in names:
            assert torch.equal(got[2][k], ref[2][k]), "%s: %s" % (what, k)
        for k in onames:
            assert torch.equal(got[3][k], ref[3][k]), "%s: %s" % (what, k)
    del g
    lay.close()
