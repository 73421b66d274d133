"""The MomentKV readout mode ("MomentKV" technical summary, Method §1, §2, §4)
through the C ABI against the moment oracle: the statistics (tensor-core
memory kernel with the identity map, value sums from its loader warps) and the
decode step's mix of retained attention and the first-order evicted estimate."""
import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import binding as B
from learned_kv_cache_indexmem_b200 import synth
from learned_kv_cache_indexmem_b200.layer import IndexMemLayer
from oracle import indexmem_oracle as om
from oracle import momentkv_oracle as mk

from .parity import MEM_TOL, Case, check_decode, to_np

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


def _layer(case):
    return IndexMemLayer.from_shape(case.shape, case.w_dev, readout="moment")


def _check_stats(st, ref, what):
    n_e, s_k, s_v, S = ref
    assert np.array_equal(to_np(st.n_e), n_e), what
    gpu = {"S^T": to_np(st.M), "s_k": to_np(st.bstab), "s_v": to_np(st.s_v)}
    want = {"S^T": np.swapaxes(S, -1, -2), "s_k": s_k, "s_v": s_v}
    for name in gpu:
        for bi in range(s_k.shape[0]):
            for h in range(s_k.shape[1]):
                r = want[name][bi, h]
                err = np.linalg.norm(gpu[name][bi, h] - r)
                assert err <= MEM_TOL * max(np.linalg.norm(r), 1e-30), "%s %s seq %d head %d" % (
                    what, name, bi, h)


@pytest.mark.parametrize("name,L,Bud,batch", [("c0", 1024, 128, 1), ("c1", 700, 100, 2),
                                              ("c1", 333, 1, 1)])
def test_moment_statistics_parity(cuda_device, name, L, Bud, batch):
    case = Case(W[name], cuda_device, L=L, batch=batch, n_decode=1)
    lay = _layer(case)
    st = lay.new_state(batch, L, Bud, Bud + 4, cuda_device)
    d = case.in_dev
    lay.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st, Bud)
    lay.update_memory(d["K"], d["V"], st, Bud, chunk=128)
    lay.sync()
    E = to_np(st.idx_evicted).astype(np.int64)
    ref = mk.moment_stats(case.in_cpu["K"], case.in_cpu["V"], E)
    _check_stats(st, ref, "%s first call" % name)
    # a second call accumulates: fold in the retained rows as well
    R = st.idx_retained.clone()
    ws = lay.workspace(batch, L, Bud, cuda_device)
    B.update_moments(lay.ctx, batch, L, d["K"], d["V"], R, Bud, 64, st.M, st.bstab, st.s_v,
                     st.n_e, ws)
    lay.sync()
    ref2 = mk.moment_stats(case.in_cpu["K"], case.in_cpu["V"], to_np(R).astype(np.int64),
                           stats0=ref)
    _check_stats(st, ref2, "%s second call" % name)
    assert np.all(to_np(st.n_e) == L)
    lay.close()


def _decode_setup(case, cap, lens, empty_stats):
    """Retained cache = the first lens rows of the layer's K/V; statistics of
    the rows after them (drawn from the same layer), held as fp32 on both sides."""
    lay = _layer(case)
    dev, b_ = case.device, case.batch
    st = lay.new_state(b_, case.L, 1, cap, dev)
    K, V = case.in_cpu["K"], case.in_cpu["V"]
    d = case.shape.head_dim
    Hkv = case.shape.n_kv_heads
    n_e = np.zeros(b_)
    s_k = np.zeros((b_, Hkv, d))
    s_v = np.zeros((b_, Hkv, d))
    S = np.zeros((b_, Hkv, d, d))
    for bi in range(b_):
        n = lens[bi]
        st.K_ret[bi, :n] = case.in_dev["K"][bi, :n]
        st.V_ret[bi, :n] = case.in_dev["V"][bi, :n]
        if not empty_stats:
            E = np.arange(n, case.L)[None]
            one = mk.moment_stats(K[bi:bi + 1], V[bi:bi + 1], E)
            n_e[bi], s_k[bi], s_v[bi], S[bi] = (x[0] for x in one)
    st.cache_len[:] = torch.tensor(lens, dtype=torch.int32, device=dev)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).float()
    st.M.copy_(f32(np.swapaxes(S, -1, -2)))
    st.bstab.copy_(f32(s_k))
    st.s_v.copy_(f32(s_v))
    st.n_e.copy_(f32(n_e))
    lay.workspace(b_, case.L, 1, dev)
    # the oracle reads the same fp32-rounded statistics
    stats = (to_np(st.n_e), to_np(st.bstab), to_np(st.s_v), np.swapaxes(to_np(st.M), -1, -2))
    return lay, st, stats


@pytest.mark.parametrize("name,batch,lens,cap,steps,empty", [
    ("c0", 1, [128], 144, 8, False),
    ("c1", 3, [410, 37, 1], 420, 6, False),    # ragged; a one-row cache
    ("c1", 1, [410], 410 + 96, 96, False),     # crosses split boundaries
    ("c1", 2, [200, 50], 260, 3, True),        # no evicted tokens: plain attention
])
def test_moment_decode_parity(cuda_device, name, batch, lens, cap, steps, empty):
    L = max(max(lens) + 64, 128)
    case = Case(W[name], cuda_device, L=L, batch=batch, n_decode=steps)
    lay, st, stats = _decode_setup(case, cap, lens, empty)
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
        o_ref, new_len, o_R, _, w_R = mk.moment_decode_step(qc, knc, vnc, KR, VR, clen, *stats)
        for bi in range(batch):
            KR[bi, clen[bi]] = knc[bi]
            VR[bi, clen[bi]] = vnc[bi]
        clen = new_len
        check_decode(to_np(out), o_ref, None, "%s step %d" % (name, s))
        if empty:
            check_decode(to_np(out), o_R, None, "%s step %d (n_e = 0)" % (name, s))
        else:
            assert np.all((w_R > 0) & (w_R < 1))
    assert np.array_equal(st.cache_len.cpu().numpy(), clen)
    lay.close()


def test_moment_path_end_to_end(cuda_device):
    # prefill -> moment statistics -> decode, against the oracle's chain
    L, Bud, batch, steps = 512, 64, 2, 4
    case = Case(W["c1"], cuda_device, L=L, batch=batch, n_decode=steps)
    lay = _layer(case)
    st = lay.new_state(batch, L, Bud, Bud + steps, cuda_device)
    d = case.in_dev
    lay.score_and_evict(d["X"], d["Q"], d["K"], d["V"], st, Bud)
    lay.update_memory(d["K"], d["V"], st, Bud, chunk=128)
    lay.sync()
    R = to_np(st.idx_retained).astype(np.int64)
    E = to_np(st.idx_evicted).astype(np.int64)
    # the selection itself is checked bit-exactly elsewhere; here the chain
    # continues from the GPU's retained and evicted sets
    stats = mk.moment_stats(case.in_cpu["K"], case.in_cpu["V"], E)
    KR, VR = om.compact(to_np(case.in_cpu["K"]), to_np(case.in_cpu["V"]), R, Bud + steps)
    clen = np.full(batch, Bud)
    for s in range(steps):
        q, kn, vn = (case.dec_dev[k][s] for k in ("q", "k_new", "v_new"))
        out = lay.decode(q, kn, vn, st)
        lay.sync()
        qc, knc, vnc = (to_np(case.dec_cpu[k][s]) for k in ("q", "k_new", "v_new"))
        o_ref, new_len, _, _, _ = mk.moment_decode_step(qc, knc, vnc, KR, VR, clen, *stats)
        for bi in range(batch):
            KR[bi, clen[bi]] = knc[bi]
            VR[bi, clen[bi]] = vnc[bi]
        clen = new_len
        check_decode(to_np(out), o_ref, None, "end to end step %d" % s)
    lay.close()


def test_modes_do_not_mix(cuda_device):
    case = Case(W["c1"], cuda_device, L=128, batch=1, n_decode=1)
    gated = case.layer()
    moment = _layer(case)
    st_g = gated.new_state(1, 128, 16, 20, cuda_device)
    st_m = moment.new_state(1, 128, 16, 20, cuda_device)
    wg = gated.workspace(1, 128, 16, cuda_device)
    wm = moment.workspace(1, 128, 16, cuda_device)
    q, kn, vn = (case.dec_dev[k][0] for k in ("q", "k_new", "v_new"))
    out = torch.empty_like(q)
    with pytest.raises(B.IndexMemError) as ei:
        B.decode(moment.ctx, 1, q, kn, vn, st_m.K_ret, st_m.V_ret, st_m.cache_len, 20, st_m.M,
                 st_m.bstab, out, wm)
    assert ei.value.name == "IMEM_ERR_UNSUPPORTED"
    with pytest.raises(B.IndexMemError) as ei:
        B.decode_moment(gated.ctx, 1, q, kn, vn, st_g.K_ret, st_g.V_ret, st_g.cache_len, 20,
                        st_g.M, st_g.bstab, st_m.s_v, st_m.n_e, out, wg)
    assert ei.value.name == "IMEM_ERR_UNSUPPORTED"
    with pytest.raises(B.IndexMemError) as ei:
        B.update_memory(moment.ctx, 1, 128, case.in_dev["K"], case.in_dev["V"], None, 0, 64,
                        st_m.M, st_m.bstab, wm)
    assert ei.value.name == "IMEM_ERR_UNSUPPORTED"
    gated.close()
    moment.close()
