"""The allocation-free memory update (imem_update_memory_static) against the
workspace-based entry point (imem_update_memory).

Some callers cannot allocate device memory -- code that runs inside a host
framework's pre-planned memory arena, or where cudaMalloc is not permitted --
so they can create neither a context nor a workspace. The static entry point
keeps its scratch in a fixed array inside the library instead. This test calls
it through the C ABI twice in a row (the second call on the state the first
left, with a different evicted set, so stale scratch contents would show) and
checks each result against the existing entry point within the memory-state
tolerance of the other parity tests. Two more cases check it against the CPU
oracle directly: the tiny fp32 layer (head dimension 64, r = 32) and the
largest batch its scratch holds (15 sequences x 8 KV heads of dimension 128,
one run per sequence and head). After every call the shared device error word
(imem_static_status) must be clear. It lives in a file of its own that pytest
collects last, and needs nothing from the tests before it.
"""
import numpy as np
import pytest
import torch

from learned_kv_cache_indexmem_b200 import binding, synth
from learned_kv_cache_indexmem_b200.layer import IndexMemLayer
from oracle import indexmem_oracle as om

pytestmark = pytest.mark.gpu

MEM_TOL = 1e-3   # relative Frobenius error per (sequence, KV head), as for update_memory


def _rel_err(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    num = np.sqrt(((a - b) ** 2).reshape(a.shape[0] * a.shape[1], -1).sum(-1))
    den = np.sqrt((b ** 2).reshape(b.shape[0] * b.shape[1], -1).sum(-1))
    return (num / np.maximum(den, 1e-30)).max()


def test_static_update_matches_workspace_update_twice(cuda_device):
    wl = synth.WORKLOADS["c1"]
    s = wl.shape
    batch, L = 3, 1500
    w = synth.make_weights(s, 11, cuda_device)
    inp = synth.make_layer_inputs(wl, w, 11, cuda_device, L=L, batch=batch)
    M0, b0 = synth.make_memory_state(s, batch, 11, cuda_device)
    lay = IndexMemLayer.from_shape(s, w)
    ws = lay.workspace(batch, L, 1, cuda_device)
    M_ref, b_ref = M0.clone(), b0.clone()
    M_st, b_st = M0.clone(), b0.clone()
    for call, (n_e, chunk) in enumerate([(1400, 128), (700, 64)]):
        E = synth.make_index_subset(batch, L, n_e, 100 + call, cuda_device)
        binding.update_memory(lay.ctx, batch, L, inp["K"], inp["V"], E, n_e, chunk, M_ref, b_ref, ws)
        binding.update_memory_static(batch, L, s.n_kv_heads, s.head_dim, s.mem_r, s.lam,
                                     binding.BF16, inp["K"], inp["V"], E, n_e, chunk,
                                     w["W_phi"], M_st, b_st)
        torch.cuda.synchronize()
        lay.sync()
        binding.static_status()                 # no device error recorded
        assert _rel_err(M_st, M_ref) <= MEM_TOL, "call %d: M" % call
        assert _rel_err(b_st, b_ref) <= MEM_TOL, "call %d: b" % call
        assert not torch.equal(M_st, M0)
    lay.close()


@pytest.mark.parametrize("name,batch,L,n_e,chunk", [
    ("c0", 1, 1024, 896, 512),      # fp32, head dimension 64, r = 32
    ("c1", 15, 640, 520, 64),       # the capacity edge: 15 x 8 x 128 x 129 floats
])
def test_static_update_against_oracle(cuda_device, name, batch, L, n_e, chunk):
    wl = synth.WORKLOADS[name]
    s = wl.shape
    dev = cuda_device
    w = synth.make_weights(s, 5, dev)
    inp = synth.make_layer_inputs(wl, w, 5, dev, L=L, batch=batch)
    M0, b0 = synth.make_memory_state(s, batch, 5, dev)
    E = synth.make_index_subset(batch, L, n_e, 9, dev)
    M, b = M0.clone(), b0.clone()
    binding.update_memory_static(batch, L, s.n_kv_heads, s.head_dim, s.mem_r, s.lam,
                                 binding.BF16 if s.dtype == "bf16" else binding.FP32,
                                 inp["K"], inp["V"], E, n_e, chunk, w["W_phi"], M, b)
    binding.static_status()
    M_ref, b_ref = om.memory_update(inp["K"].cpu(), inp["V"].cpu(), E.cpu().numpy(),
                                    w["W_phi"].cpu(), s.lam, M0=M0.cpu(), b0=b0.cpu())
    assert _rel_err(M, torch.from_numpy(M_ref)) <= MEM_TOL, "M"
    assert _rel_err(b, torch.from_numpy(b_ref)) <= MEM_TOL, "b"


def test_static_update_rejects_sizes_beyond_its_scratch(cuda_device):
    s = synth.LLAMA8B
    # 16 sequences x 8 KV heads x 128 x 129 floats exceed the 8 MiB scratch
    K = torch.zeros(16, 64, s.n_kv_heads, s.head_dim, dtype=torch.bfloat16, device=cuda_device)
    E = torch.zeros(16, 8, dtype=torch.int32, device=cuda_device)
    W = torch.zeros(s.mem_r, s.head_dim, device=cuda_device)
    M = torch.zeros(16, s.n_kv_heads, s.mem_r, s.head_dim, device=cuda_device)
    b = torch.zeros(16, s.n_kv_heads, s.mem_r, device=cuda_device)
    with pytest.raises(binding.IndexMemError) as ei:
        binding.update_memory_static(16, 64, s.n_kv_heads, s.head_dim, s.mem_r, s.lam,
                                     binding.BF16, K, K, E, 8, 64, W, M, b)
    assert ei.value.name == "IMEM_ERR_UNSUPPORTED"
    assert not M.any()
