"""Failure handling on the GPU without a fault: a bounded device wait that
runs out is reported by imem_sync as IMEM_ERR_TIMEOUT, cleared by it, and the
context keeps working (a decode step then matches the oracle)."""
import numpy as np
import pytest

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
