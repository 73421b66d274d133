"""Decode steps launched back to back, with no host synchronisation between
them (as in serving and in the benchmark's CUDA graphs), through the C ABI
against the oracle ("IndexMem" technical summary §2.B, Output; "MomentKV"
technical summary, Method §2, §4, for the moment readout).

Each step loads cache rows below its hinted length minus one, b and M before
its launch-dependency wait and keeps those copies only if the workspace's
decode tag matches the length it finds after the wait. The chain is checked
on every output while it runs (tag hits), across split changes (the early
stages are dropped), after direct writes followed by imem_decode_invalidate,
after a library call that clears the tag, and when the steps are replayed
from a CUDA graph."""
import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import synth
from oracle import indexmem_oracle as om
from oracle import momentkv_oracle as mk

from .parity import Case, check_decode, check_memory, ill_conditioned, to_np
from .test_gpu_parity import _decode_case

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


class _Ref:
    """The oracle's copy of one decode chain's state (gated readout)."""

    def __init__(self, case, st, lens, M0, b0, gate_override=None):
        cap = st.K_ret.shape[1]
        self.case = case
        self.gate_override = gate_override
        self.KR = np.zeros((case.batch, cap) + case.in_cpu["K"].shape[2:])
        self.VR = np.zeros_like(self.KR)
        for bi in range(case.batch):
            self.KR[bi, :lens[bi]] = to_np(case.in_cpu["K"][bi, :lens[bi]])
            self.VR[bi, :lens[bi]] = to_np(case.in_cpu["V"][bi, :lens[bi]])
        self.clen = np.array(lens)
        self.M, self.b = M0, b0
        self.W_phi = case.w_cpu["W_phi"].numpy().astype(np.float64)
        self.w_gate = case.w_cpu["w_gate"].numpy().astype(np.float64)
        self.group = case.shape.n_q_heads // case.shape.n_kv_heads

    def check(self, outs, s0, what):
        for i, out in enumerate(outs):
            s = s0 + i
            qc, knc, vnc = (to_np(self.case.dec_cpu[k][s]) for k in ("q", "k_new", "v_new"))
            o_ref, new_len, _, _, _ = om.decode_step(qc, knc, vnc, self.KR, self.VR, self.clen,
                                                     self.M, self.b, self.W_phi, self.w_gate,
                                                     gate_override=self.gate_override)
            for bi in range(self.case.batch):
                self.KR[bi, self.clen[bi]] = knc[bi]
                self.VR[bi, self.clen[bi]] = vnc[bi]
            self.clen = new_len
            mask = (None if self.gate_override is not None
                    else ill_conditioned(self.b, qc, self.W_phi, self.group))
            check_decode(to_np(out), o_ref, mask, "%s step %d" % (what, s))


def _run(lay, st, case, s0, n):
    outs = [torch.empty_like(case.dec_dev["q"][0]) for _ in range(n)]
    for i in range(n):
        s = s0 + i
        lay.decode(case.dec_dev["q"][s], case.dec_dev["k_new"][s], case.dec_dev["v_new"][s], st,
                   out=outs[i])
    return outs


@pytest.mark.parametrize("name,batch,lens,cap,steps,gate", [
    # one wave: cp.async staging, rows and memory loaded before the wait
    ("c1", 4, [1024, 1000, 700, 1], 1024 + 3 * 48, 48, None),
    # several waves: TMA staging (rows issued after the wait); attention
    # alone (gate 0), which also keeps 1024 readouts clear of cancelling
    # denominators
    ("c1", 32, [300] * 31 + [17], 300 + 3 * 20, 20, 0.0),
])
def test_back_to_back_chain(cuda_device, name, batch, lens, cap, steps, gate):
    case = Case(W[name], cuda_device, L=max(lens), batch=batch, n_decode=3 * steps)
    lay, st, M0, b0 = _decode_case(case, cap, lens, gate)
    ref = _Ref(case, st, lens, M0, b0, gate)
    # 1. a chain of steps, one launch after the other
    outs = _run(lay, st, case, 0, steps)
    lay.sync()
    ref.check(outs, 0, "%s chain" % name)
    assert np.array_equal(st.cache_len.cpu().numpy(), ref.clen)
    # 2. direct writes between two steps (rows below the length and the
    # memory), announced with imem_decode_invalidate
    g = torch.Generator(device=cuda_device)
    g.manual_seed(5)
    half = int(ref.clen.min()) // 2
    new_rows = torch.randn(batch, half, *st.K_ret.shape[2:], generator=g, device=cuda_device)
    st.K_ret[:, :half] = new_rows.to(st.K_ret.dtype)
    st.M.mul_(0.5)
    lay.invalidate_decode(batch)
    ref.KR[:, :half] = to_np(st.K_ret[:, :half])
    ref.M = to_np(st.M)
    outs = _run(lay, st, case, steps, steps)
    lay.sync()
    ref.check(outs, steps, "%s after direct writes" % name)
    # 3. the same chain from a CUDA graph (programmatic launch edges)
    s0 = 2 * steps
    outs = [torch.empty_like(case.dec_dev["q"][0]) for _ in range(steps)]
    stream = torch.cuda.Stream(cuda_device)
    stream.wait_stream(torch.cuda.current_stream(cuda_device))
    len_before = st.cache_len.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(steps):
            lay.decode(case.dec_dev["q"][s0 + i], case.dec_dev["k_new"][s0 + i],
                       case.dec_dev["v_new"][s0 + i], st, out=outs[i], stream=stream)
    assert torch.equal(st.cache_len, len_before)   # capture ran nothing
    graph.replay()
    torch.cuda.synchronize(cuda_device)
    ref.check(outs, s0, "%s graph" % name)
    assert np.array_equal(st.cache_len.cpu().numpy(), ref.clen)
    del graph
    lay.close()


def test_library_call_between_chains_clears_the_tag(cuda_device):
    # a chain leaves tag = 1 + length; a prefill of other data into the same
    # state and workspace then ends at that same length. The prefill's calls
    # clear the tag, so the next step reads the new cache and memory.
    B, L, batch, steps = 96, 512, 2, 2
    case_a = Case(W["c1"], cuda_device, L=L, batch=batch, n_decode=steps)
    case_b = Case(W["c1"], cuda_device, L=L, batch=batch, n_decode=1, seed=11)
    lay = case_a.layer()
    st = lay.new_state(batch, L, B, B + steps, cuda_device)
    d = case_a.in_dev
    lay.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st, B)
    lay.update_memory(d["K"], d["V"], st, B, chunk=64)
    st.cache_len.fill_(B - steps)                    # a shorter cache for the first chain
    lay.invalidate_decode(batch)
    _run(lay, st, case_a, 0, steps)                  # cache_len: B - steps -> B, tag 1 + B
    # the second prefill: the same layer weights, other context
    wl = W["c1"]
    inp_b = synth.make_layer_inputs(wl, case_a.w_cpu, 11, "cpu", L=L, batch=batch)
    db = {k: v.to(cuda_device) for k, v in inp_b.items()}
    lay.score_and_evict(db["X"], db["Q"], db["K"], db["V"], st, B)
    M_before, b_before = st.M.clone(), st.bstab.clone()   # the update accumulates onto them
    lay.update_memory(db["K"], db["V"], st, B, chunk=64)
    st.cache_len.fill_(B)
    out = _run(lay, st, case_b, 0, 1)[0]
    lay.sync()
    assert np.all(st.cache_len.cpu().numpy() == B + 1)
    I_gpu = to_np(st.running_max)
    R, E = om.select_budget(I_gpu, B)
    assert np.array_equal(st.idx_retained.cpu().numpy(), R)
    W_phi = case_a.w_cpu["W_phi"].numpy().astype(np.float64)
    w_gate = case_a.w_cpu["w_gate"].numpy().astype(np.float64)
    KR, VR = om.compact(to_np(inp_b["K"]), to_np(inp_b["V"]), R, B + steps)
    M_ref, b_ref = om.memory_update(inp_b["K"], inp_b["V"], E, case_a.w_cpu["W_phi"],
                                    wl.shape.lam, M0=to_np(M_before), b0=to_np(b_before))
    # the memory the step read: the GPU's, checked against the oracle's here;
    # the oracle's decode then reads the GPU's state
    M_gpu, b_gpu = to_np(st.M), to_np(st.bstab)
    check_memory(M_gpu, b_gpu, M_ref, b_ref, "after prefill")
    qc, knc, vnc = (to_np(case_b.dec_cpu[k][0]) for k in ("q", "k_new", "v_new"))
    o_ref, _, _, _, _ = om.decode_step(qc, knc, vnc, KR, VR, np.full(batch, B), M_gpu, b_gpu,
                                       W_phi, w_gate)
    group = wl.shape.n_q_heads // wl.shape.n_kv_heads
    check_decode(to_np(out), o_ref, ill_conditioned(b_gpu, qc, W_phi, group), "after prefill")
    lay.close()


def test_moment_chain_back_to_back(cuda_device):
    # the moment readout stages s_k, s_v and S^T before the wait as well
    from .test_gpu_moment import _decode_setup
    batch, lens, steps = 4, [1024, 900, 512, 3], 40
    cap = 1024 + steps
    case = Case(W["c1"], cuda_device, L=1024 + 64, batch=batch, n_decode=steps)
    lay, st, stats = _decode_setup(case, cap, lens, False)
    KR = np.zeros((batch, cap) + case.in_cpu["K"].shape[2:])
    VR = np.zeros_like(KR)
    for bi in range(batch):
        KR[bi, :lens[bi]] = to_np(case.in_cpu["K"][bi, :lens[bi]])
        VR[bi, :lens[bi]] = to_np(case.in_cpu["V"][bi, :lens[bi]])
    outs = _run(lay, st, case, 0, steps)
    lay.sync()
    clen = np.array(lens)
    for s in range(steps):
        qc, knc, vnc = (to_np(case.dec_cpu[k][s]) for k in ("q", "k_new", "v_new"))
        o_ref, clen_new, _, _, _ = mk.moment_decode_step(qc, knc, vnc, KR, VR, clen, *stats)
        for bi in range(batch):
            KR[bi, clen[bi]] = knc[bi]
            VR[bi, clen[bi]] = vnc[bi]
        clen = clen_new
        check_decode(to_np(outs[s]), o_ref, None, "moment chain step %d" % s)
    assert np.array_equal(st.cache_len.cpu().numpy(), clen)
    lay.close()
