"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/indexmem.h declares, and rejects invalid calls with the
documented status before touching the device."""
import ctypes
import math
import os
import re

import pytest

from learned_kv_cache_indexmem_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(imem_[a-z_]+)\s*\(", txt))
    return names


def test_library_exports_every_declared_symbol():
    lib = B.load()
    names = _declared()
    assert {"imem_init", "imem_destroy", "imem_workspace_size", "imem_score_and_evict",
            "imem_update_memory", "imem_decode", "imem_sync", "imem_status_string"} <= names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for code, name in B.STATUS.items():
        assert B.status_string(code) == name
    assert B.status_string(99) == "IMEM_ERR_UNKNOWN"


def _cfg(**kw):
    base = dict(hidden=512, n_q_heads=8, n_kv_heads=2, head_dim=64, idx_dim=32, mem_r=32,
                lam=0.99, dtype=B.FP32)
    base.update(kw)
    return B.make_config(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), "IMEM_ERR_UNSUPPORTED"),
    (dict(idx_dim=48), "IMEM_ERR_UNSUPPORTED"),
    (dict(n_kv_heads=3), "IMEM_ERR_SHAPE"),
    (dict(n_q_heads=32, n_kv_heads=2), "IMEM_ERR_UNSUPPORTED"),   # group 16
    (dict(hidden=500), "IMEM_ERR_UNSUPPORTED"),
    (dict(mem_r=200), "IMEM_ERR_UNSUPPORTED"),
    (dict(lam=0.0), "IMEM_ERR_INVALID_ARG"),
    (dict(lam=1.5), "IMEM_ERR_INVALID_ARG"),
    (dict(dtype=7), "IMEM_ERR_INVALID_ARG"),
    (dict(idx_heads=4), "IMEM_ERR_UNSUPPORTED"),
    (dict(readout=5), "IMEM_ERR_INVALID_ARG"),
    (dict(readout=B.READOUT_MOMENT, mem_r=32, lam=1.0), "IMEM_ERR_UNSUPPORTED"),   # r != d
    (dict(readout=B.READOUT_MOMENT, mem_r=64, lam=0.99), "IMEM_ERR_UNSUPPORTED"),  # decay
])
def test_init_rejects_bad_config_before_any_device_work(kw, code):
    with pytest.raises(B.IndexMemError) as ei:
        B.init(_cfg(**kw), 16, 16, 16, 16, 16)
    assert ei.value.name == code


def test_init_rejects_null_and_misaligned_weights():
    with pytest.raises(B.IndexMemError) as ei:
        B.init(_cfg(), 0, 16, 16, 16, 16)
    assert ei.value.name == "IMEM_ERR_INVALID_ARG"
    with pytest.raises(B.IndexMemError) as ei:
        B.init(_cfg(), 16, 18, 16, 16, 16)
    assert ei.value.name == "IMEM_ERR_ALIGN"


def test_null_context_is_invalid_for_every_call():
    lib = B.load()
    n = ctypes.c_size_t()
    assert lib.imem_workspace_size(None, 1, 16, 4, ctypes.byref(n)) == 1
    assert lib.imem_score_and_evict(None, 1, 16, 4, 16, 16, 16, 16, 16, 0, 16, 1, 16, 16, 16, 16,
                                    16, 16, None) == 1
    assert lib.imem_update_memory(None, 1, 16, 16, 16, 16, 4, 64, 16, 16, 16, None) == 1
    assert lib.imem_decode(None, 1, 16, 16, 16, 16, 16, 16, 8, 16, 16, 16, 16, None) == 1
    assert lib.imem_sync(None, None) == 1
    assert lib.imem_join(None, None) == 1
    n2 = ctypes.c_size_t()
    assert lib.imem_workspace_size_evict(None, 1, 16, 4, 8, ctypes.byref(n2)) == 1
    assert lib.imem_prefill_evict_chunk(None, 1, 16, 4, 8, 16, 16, 16, 16, 0, 8, 16, 16, None, 16,
                                        16, 64, 0, None, None, 8, 16, None) == 1
    assert lib.imem_online_init(None, 1, 16, 4, 16, 16, 16, 16, 16, 16, 16, 8, None) == 1
    assert lib.imem_decode_online(None, 1, 4, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 16, 8, 16,
                                  16, 16, 16, 16, None) == 1
    assert lib.imem_selftest_wait(None, 1000, None) == 1
    assert lib.imem_decode_invalidate(None, 1, 16, None) == 1
    assert lib.imem_update_moments(None, 1, 16, 16, 16, 16, 4, 64, 16, 16, 16, 16, 16, None) == 1
    assert lib.imem_decode_moment(None, 1, 16, 16, 16, 16, 16, 16, 8, 16, 16, 16, 16, 16, 16,
                                  None) == 1
    assert lib.imem_indexer_features(None, 1, 16, 16, 16, 16, 0, 16, 16, None) == 1
    assert lib.imem_indexer_score(None, 1, 16, 16, 0, 16, 16, None) == 1
    assert lib.imem_select_compact(None, 1, 16, 4, 16, 16, 16, 16, 16, 16, 16, 8, 16,
                                   None) == 1
    lib.imem_destroy(None)   # accepted
    out = ctypes.c_void_p(123)
    assert lib.imem_init(None, None, ctypes.byref(out)) == 1 and out.value is None
