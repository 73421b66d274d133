"""Thin ctypes binding of libindexmem.so (the C ABI in include/indexmem.h).

Argument marshalling only: tensors become device pointers, streams become
their handles, and a non-OK status raises IndexMemError. Every step of the
path runs in the library's CUDA kernels; there is no fallback. The functions
keep the C names without the ``imem_`` prefix.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libindexmem.so")

STATUS = {0: "IMEM_OK", 1: "IMEM_ERR_INVALID_ARG", 2: "IMEM_ERR_SHAPE", 3: "IMEM_ERR_ALIGN",
          4: "IMEM_ERR_UNSUPPORTED", 5: "IMEM_ERR_CUDA", 6: "IMEM_ERR_TIMEOUT",
          7: "IMEM_ERR_RANGE"}
FP32, BF16 = 0, 1
READOUT_GATED, READOUT_MOMENT = 0, 1


class IndexMemError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__("%s failed: %s" % (where, STATUS.get(code, code)))
        self.code = code
        self.name = STATUS.get(code, str(code))


class Config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_q_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("idx_heads", ctypes.c_int), ("idx_dim", ctypes.c_int),
                ("mem_r", ctypes.c_int), ("lambda_", ctypes.c_float),
                ("eps", ctypes.c_float), ("dtype", ctypes.c_int),
                ("gate_override", ctypes.c_float), ("readout", ctypes.c_int)]


class Weights(ctypes.Structure):
    _fields_ = [("W_idx_q", ctypes.c_void_p), ("W_idx_k", ctypes.c_void_p),
                ("w_idx_g", ctypes.c_void_p), ("W_phi", ctypes.c_void_p),
                ("w_gate", ctypes.c_void_p)]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads the library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libindexmem.so not built: run `python -m "
                          "learned_kv_cache_indexmem_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.imem_status_string.restype = ctypes.c_char_p
    lib.imem_status_string.argtypes = [i]
    lib.imem_init.restype = i
    lib.imem_init.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(Weights), ctypes.POINTER(vp)]
    lib.imem_destroy.restype = None
    lib.imem_destroy.argtypes = [vp]
    lib.imem_workspace_size.restype = i
    lib.imem_workspace_size.argtypes = [vp, i, i, i, ctypes.POINTER(ctypes.c_size_t)]
    lib.imem_score_and_evict.restype = i
    lib.imem_score_and_evict.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp, i, i, i, vp, vp, vp,
                                         vp, i, vp, vp]
    lib.imem_update_memory.restype = i
    lib.imem_update_memory.argtypes = [vp, i, i, vp, vp, vp, i, i, vp, vp, vp, vp]
    lib.imem_decode.restype = i
    lib.imem_decode.argtypes = [vp, i, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp]
    lib.imem_sync.restype = i
    lib.imem_sync.argtypes = [vp, vp]
    lib.imem_join.restype = i
    lib.imem_join.argtypes = [vp, vp]
    lib.imem_workspace_size_evict.restype = i
    lib.imem_workspace_size_evict.argtypes = [vp, i, i, i, i, ctypes.POINTER(ctypes.c_size_t)]
    lib.imem_prefill_evict_chunk.restype = i
    lib.imem_prefill_evict_chunk.argtypes = [vp, i, i, i, i, vp, vp, vp, vp, i, i, vp, vp, vp,
                                             vp, vp, i, i, vp, vp, i, vp, vp]
    lib.imem_online_init.restype = i
    lib.imem_online_init.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp, vp, vp, i, vp]
    lib.imem_decode_online.restype = i
    lib.imem_decode_online.argtypes = [vp, i, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i,
                                       vp, vp, vp, vp, vp, vp]
    lib.imem_decode_invalidate.restype = i
    lib.imem_decode_invalidate.argtypes = [vp, i, vp, vp]
    lib.imem_selftest_wait.restype = i
    lib.imem_selftest_wait.argtypes = [vp, ctypes.c_longlong, vp]
    lib.imem_update_moments.restype = i
    lib.imem_update_moments.argtypes = [vp, i, i, vp, vp, vp, i, i, vp, vp, vp, vp, vp, vp]
    lib.imem_decode_moment.restype = i
    lib.imem_decode_moment.argtypes = [vp, i, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp,
                                       vp]
    lib.imem_update_memory_static.restype = i
    lib.imem_update_memory_static.argtypes = [i, i, i, i, i, f, i, vp, vp, vp, i, i, vp, vp, vp, vp]
    lib.imem_static_status.restype = i
    lib.imem_static_status.argtypes = [vp]
    lib.imem_indexer_features.restype = i
    lib.imem_indexer_features.argtypes = [vp, i, i, vp, vp, vp, i, i, vp, vp]
    lib.imem_indexer_score.restype = i
    lib.imem_indexer_score.argtypes = [vp, i, i, vp, i, i, vp, vp]
    lib.imem_select_compact.restype = i
    lib.imem_select_compact.argtypes = [vp, i, i, i, vp, vp, vp, vp, vp, vp, vp, i, vp, vp]
    _lib = lib
    return lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        import torch
        s = torch.cuda.current_stream()
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(code: int, where: str):
    if code != 0:
        raise IndexMemError(code, where)


def status_string(code: int) -> str:
    return load().imem_status_string(code).decode()


def make_config(hidden, n_q_heads, n_kv_heads, head_dim, idx_dim, mem_r, lam, dtype,
                eps=1e-6, gate_override=None, idx_heads=None, readout=None) -> Config:
    return Config(hidden, n_q_heads, n_kv_heads, head_dim,
                  n_q_heads if idx_heads is None else idx_heads, idx_dim, mem_r, lam, eps, dtype,
                  math.nan if gate_override is None else float(gate_override),
                  READOUT_GATED if readout is None else readout)


def init(cfg: Config, W_idx_q, W_idx_k, w_idx_g, W_phi, w_gate) -> int:
    """imem_init: returns the context handle (an int)."""
    lib = load()
    w = Weights(_ptr(W_idx_q), _ptr(W_idx_k), _ptr(w_idx_g), _ptr(W_phi), _ptr(w_gate))
    out = ctypes.c_void_p()
    _check(lib.imem_init(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(out)), "imem_init")
    return out.value


def destroy(ctx: int) -> None:
    load().imem_destroy(ctx)


def workspace_size(ctx: int, batch: int, L: int, B: int) -> int:
    n = ctypes.c_size_t()
    _check(load().imem_workspace_size(ctx, batch, L, B, ctypes.byref(n)), "imem_workspace_size")
    return n.value


def score_and_evict(ctx, batch, L, B, X, Q, K, V, running_max, q_begin, q_end, finalize,
                    idx_retained, idx_evicted, K_ret, V_ret, cap, workspace, stream=None):
    _check(load().imem_score_and_evict(
        ctx, batch, L, B, _ptr(X), _ptr(Q), _ptr(K), _ptr(V), _ptr(running_max), q_begin, q_end,
        int(finalize), _ptr(idx_retained), _ptr(idx_evicted), _ptr(K_ret), _ptr(V_ret), cap,
        _ptr(workspace), _stream(stream)), "imem_score_and_evict")


def update_memory(ctx, batch, L, K, V, idx_evicted, n_evicted, chunk, M, bstab, workspace,
                  stream=None):
    _check(load().imem_update_memory(
        ctx, batch, L, _ptr(K), _ptr(V), _ptr(idx_evicted), n_evicted, chunk, _ptr(M),
        _ptr(bstab), _ptr(workspace), _stream(stream)), "imem_update_memory")


def decode(ctx, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, M, bstab, out, workspace,
           stream=None):
    _check(load().imem_decode(
        ctx, batch, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(K_ret), _ptr(V_ret), _ptr(cache_len),
        cap, _ptr(M), _ptr(bstab), _ptr(out), _ptr(workspace), _stream(stream)), "imem_decode")


def workspace_size_evict(ctx: int, batch: int, L: int, B: int, chunk_max: int) -> int:
    n = ctypes.c_size_t()
    _check(load().imem_workspace_size_evict(ctx, batch, L, B, chunk_max, ctypes.byref(n)),
           "imem_workspace_size_evict")
    return n.value


def prefill_evict_chunk(ctx, batch, L, B, chunk_max, X, Q, K, V, q_begin, q_end, retained,
                        evicted, cand_importance, M, bstab, mem_chunk, finalize, K_ret, V_ret,
                        cap, workspace, stream=None):
    _check(load().imem_prefill_evict_chunk(
        ctx, batch, L, B, chunk_max, _ptr(X), _ptr(Q), _ptr(K), _ptr(V), q_begin, q_end,
        _ptr(retained), _ptr(evicted), _ptr(cand_importance), _ptr(M), _ptr(bstab), mem_chunk,
        int(finalize), _ptr(K_ret), _ptr(V_ret), cap, _ptr(workspace), _stream(stream)),
        "imem_prefill_evict_chunk")


def online_init(ctx, batch, L, B, running_max, idx_retained, workspace, khat_ret, I_ret, pos_ret,
                next_pos, cap, stream=None):
    _check(load().imem_online_init(
        ctx, batch, L, B, _ptr(running_max), _ptr(idx_retained), _ptr(workspace), _ptr(khat_ret),
        _ptr(I_ret), _ptr(pos_ret), _ptr(next_pos), cap, _stream(stream)), "imem_online_init")


def decode_online(ctx, batch, B, x_new, q, k_new, v_new, K_ret, V_ret, khat_ret, I_ret, pos_ret,
                  next_pos, cache_len, cap, M, bstab, out, evicted, workspace, stream=None):
    _check(load().imem_decode_online(
        ctx, batch, B, _ptr(x_new), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(K_ret), _ptr(V_ret),
        _ptr(khat_ret), _ptr(I_ret), _ptr(pos_ret), _ptr(next_pos), _ptr(cache_len), cap, _ptr(M),
        _ptr(bstab), _ptr(out), _ptr(evicted), _ptr(workspace), _stream(stream)),
        "imem_decode_online")


def decode_invalidate(ctx, batch, workspace, stream=None):
    """imem_decode_invalidate: clears the workspace's decode tags (after the
    caller wrote a retained cache, its length or the memory by other means)."""
    _check(load().imem_decode_invalidate(ctx, batch, _ptr(workspace), _stream(stream)),
           "imem_decode_invalidate")


def selftest_wait(ctx, limit_cycles, stream=None):
    """imem_selftest_wait: a bounded device wait that runs out (failure path)."""
    _check(load().imem_selftest_wait(ctx, int(limit_cycles), _stream(stream)), "imem_selftest_wait")


def update_moments(ctx, batch, L, K, V, idx_evicted, n_evicted, chunk, S_T, s_k, s_v, n_e,
                   workspace, stream=None):
    _check(load().imem_update_moments(
        ctx, batch, L, _ptr(K), _ptr(V), _ptr(idx_evicted), n_evicted, chunk, _ptr(S_T),
        _ptr(s_k), _ptr(s_v), _ptr(n_e), _ptr(workspace), _stream(stream)), "imem_update_moments")


def decode_moment(ctx, batch, q, k_new, v_new, K_ret, V_ret, cache_len, cap, S_T, s_k, s_v, n_e,
                  out, workspace, stream=None):
    _check(load().imem_decode_moment(
        ctx, batch, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(K_ret), _ptr(V_ret), _ptr(cache_len),
        cap, _ptr(S_T), _ptr(s_k), _ptr(s_v), _ptr(n_e), _ptr(out), _ptr(workspace),
        _stream(stream)), "imem_decode_moment")


def update_memory_static(batch, L, n_kv_heads, head_dim, mem_r, lam, dtype, K, V, idx_evicted,
                         n_evicted, chunk, W_phi, M, bstab, stream=None):
    """imem_update_memory_static: the memory update without a context or a
    workspace, for callers that cannot allocate device memory (its scratch is a
    fixed array inside the library; see include/indexmem.h)."""
    _check(load().imem_update_memory_static(
        batch, L, n_kv_heads, head_dim, mem_r, lam, dtype, _ptr(K), _ptr(V), _ptr(idx_evicted),
        n_evicted, chunk, _ptr(W_phi), _ptr(M), _ptr(bstab), _stream(stream)),
        "imem_update_memory_static")


def indexer_features(ctx, batch, L, X, Q, running_max, q_begin, q_end, workspace, stream=None):
    _check(load().imem_indexer_features(ctx, batch, L, _ptr(X), _ptr(Q), _ptr(running_max),
                                        q_begin, q_end, _ptr(workspace), _stream(stream)),
           "imem_indexer_features")


def indexer_score(ctx, batch, L, running_max, q_begin, q_end, workspace, stream=None):
    _check(load().imem_indexer_score(ctx, batch, L, _ptr(running_max), q_begin, q_end,
                                     _ptr(workspace), _stream(stream)), "imem_indexer_score")


def select_compact(ctx, batch, L, B, running_max, K, V, idx_retained, idx_evicted, K_ret, V_ret,
                   cap, workspace, stream=None):
    _check(load().imem_select_compact(ctx, batch, L, B, _ptr(running_max), _ptr(K), _ptr(V),
                                      _ptr(idx_retained), _ptr(idx_evicted), _ptr(K_ret),
                                      _ptr(V_ret), cap, _ptr(workspace), _stream(stream)),
           "imem_select_compact")


def static_status(stream=None) -> None:
    """imem_static_status: raises if a call of update_memory_static on this
    device recorded a device error since the last query (and clears it)."""
    _check(load().imem_static_status(_stream(stream)), "imem_static_status")


def join(ctx, stream=None) -> None:
    """imem_join: `stream` waits for a pre-eviction memory update still
    running on the context's second stream."""
    _check(load().imem_join(ctx, _stream(stream)), "imem_join")


def sync(ctx, stream=None) -> None:
    _check(load().imem_sync(ctx, _stream(stream)), "imem_sync")
