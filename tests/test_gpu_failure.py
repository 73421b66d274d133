"""Failure handling on the GPU without a fault: a bounded device wait that
runs out is reported by imem_sync as IMEM_ERR_TIMEOUT, cleared by it, and the
context keeps working (a decode step then matches the oracle). Inputs outside
what the memory update computes with (an evicted index outside [0, L); with
fp32 inputs a key beyond fp16's range) are caught by the kernel's own checks,
reported as IMEM_ERR_RANGE, and the context keeps working; with bf16 inputs a
key beyond fp16's range is computed correctly."""
import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import binding as B
from learned_kv_cache_indexmem_b200 import synth
from oracle import indexmem_oracle as om

from .parity import Case, check_decode, ill_conditioned, to_np

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_cleared(cuda_device):
    case = Case(synth.WORKLOADS["c1"], cuda_device, L=128, batch=1, n_decode=1)
    lay = case.layer()
    B.selftest_wait(lay.ctx, 2_000_000)          # ~1 ms at the SM clock
    with pytest.raises(B.IndexMemError) as ei:
        lay.sync()
    assert ei.value.name == "IMEM_ERR_TIMEOUT"
    lay.sync()                                   # cleared: no error now
    # the context keeps working: one decode step against the oracle
    st = lay.new_state(1, 128, 1, 70, cuda_device)
    st.K_ret[0, :64] = case.in_dev["K"][0, :64]
    st.V_ret[0, :64] = case.in_dev["V"][0, :64]
    st.cache_len.fill_(64)
    lay.workspace(1, 128, 1, cuda_device)
    q, kn, vn = (case.dec_dev[k][0] for k in ("q", "k_new", "v_new"))
    out = lay.decode(q, kn, vn, st)
    lay.sync()
    KR = np.zeros((1, 70) + tuple(case.in_cpu["K"].shape[2:]))
    VR = np.zeros_like(KR)
    KR[0, :64] = to_np(case.in_cpu["K"][0, :64])
    VR[0, :64] = to_np(case.in_cpu["V"][0, :64])
    W_phi = case.w_cpu["W_phi"].numpy().astype(np.float64)
    qc, knc, vnc = (to_np(case.dec_cpu[k][0]) for k in ("q", "k_new", "v_new"))
    M0, b0 = to_np(st.M), to_np(st.bstab)
    o_ref, _, _, _, _ = om.decode_step(qc, knc, vnc, KR, VR, np.array([64]), M0, b0, W_phi,
                                       case.w_cpu["w_gate"])
    group = case.shape.n_q_heads // case.shape.n_kv_heads
    check_decode(to_np(out), o_ref, ill_conditioned(b0, qc, W_phi, group), "after timeout")
    with pytest.raises(B.IndexMemError) as ei:
        B.selftest_wait(lay.ctx, 0)
    assert ei.value.name == "IMEM_ERR_INVALID_ARG"
    lay.close()


def test_memory_update_out_of_range_inputs_are_reported(cuda_device):
    # bf16 inputs: the keys enter the tensor-core sums as bf16 hi + lo halves
    # (fp32's range), so a key far beyond fp16's range is computed, not refused
    wl = synth.WORKLOADS["c1"]
    s = wl.shape
    case = Case(wl, cuda_device, L=256, batch=2, n_decode=1)
    lay = case.layer()
    ws = lay.workspace(2, 256, 1, cuda_device)
    K = case.in_dev["K"].clone()
    E = synth.make_index_subset(2, 256, 100, 3, cuda_device)
    M = torch.zeros(2, s.n_kv_heads, s.mem_r, s.head_dim, device=cuda_device)
    b = torch.zeros(2, s.n_kv_heads, s.mem_r, device=cuda_device)
    K[1, int(E[1, 40]), 3, 17] = 1.0e5
    B.update_memory(lay.ctx, 2, 256, K, case.in_dev["V"], E, 100, 64, M, b, ws)
    lay.sync()
    M_ref, b_ref = om.memory_update(K.cpu(), case.in_cpu["V"], E.cpu().numpy(),
                                    case.w_cpu["W_phi"], s.lam)
    from .parity import check_memory
    check_memory(to_np(M), to_np(b), M_ref, b_ref, "bf16 key 1e5")
    # an evicted index at L: no row is read, the error is reported
    E2 = E.clone()
    E2[0, 99] = 256
    B.update_memory(lay.ctx, 2, 256, case.in_dev["K"], case.in_dev["V"], E2, 100, 64, M, b, ws)
    with pytest.raises(B.IndexMemError) as ei:
        lay.sync()
    assert ei.value.name == "IMEM_ERR_RANGE"
    # the same index through the allocation-free entry point and its status word
    B.update_memory_static(2, 256, s.n_kv_heads, s.head_dim, s.mem_r, s.lam, B.BF16,
                           case.in_dev["K"], case.in_dev["V"], E2, 100, 64, case.w_dev["W_phi"],
                           M, b)
    with pytest.raises(B.IndexMemError) as ei:
        B.static_status()
    assert ei.value.name == "IMEM_ERR_RANGE"
    B.static_status()                            # cleared
    # in-range inputs afterwards: no error, result as the oracle's
    M.zero_(); b.zero_()
    B.update_memory(lay.ctx, 2, 256, case.in_dev["K"], case.in_dev["V"], E, 100, 64, M, b, ws)
    lay.sync()
    M_ref, b_ref = om.memory_update(case.in_cpu["K"], case.in_cpu["V"], E.cpu().numpy(),
                                    case.w_cpu["W_phi"], s.lam)
    check_memory(to_np(M), to_np(b), M_ref, b_ref, "after range errors")
    lay.close()
    # fp32 inputs keep fp16 tensor-core operands: a key beyond fp16's range is
    # reported as IMEM_ERR_RANGE
    wl0 = synth.WORKLOADS["c0"]
    s0 = wl0.shape
    case0 = Case(wl0, cuda_device, L=256, batch=1, n_decode=1)
    lay0 = case0.layer()
    ws0 = lay0.workspace(1, 256, 1, cuda_device)
    K0 = case0.in_dev["K"].clone()
    E0 = synth.make_index_subset(1, 256, 100, 4, cuda_device)
    K0[0, int(E0[0, 7]), 1, 5] = 1.0e5
    M0 = torch.zeros(1, s0.n_kv_heads, s0.mem_r, s0.head_dim, device=cuda_device)
    b0 = torch.zeros(1, s0.n_kv_heads, s0.mem_r, device=cuda_device)
    B.update_memory(lay0.ctx, 1, 256, K0, case0.in_dev["V"], E0, 100, 64, M0, b0, ws0)
    with pytest.raises(B.IndexMemError) as ei:
        lay0.sync()
    assert ei.value.name == "IMEM_ERR_RANGE"
    lay0.close()
