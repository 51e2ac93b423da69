"""Host-only checks of the C ABI: the library loads without a GPU, exports every entry
point declared in include/dsa.h, and rejects bad arguments before launching anything.
No call here reaches a CUDA API (every case returns during host-side validation)."""
import ctypes
import os
import re

import pytest

import attention_lightning_indexer_b200 as dsa
from attention_lightning_indexer_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(dsa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_entry_point():
    lib = dsa.load()
    declared = _declared_functions()
    assert "dsa_forward" in declared and "dsa_topk" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(_native.EXPORTED)
    assert lib.dsa_abi_version() == 2


def test_status_strings():
    lib = dsa.load()
    for code in range(7):
        assert lib.dsa_status_string(code)
    assert lib.dsa_status_string(99) == b"unknown status"


def _problem(**kw):
    args = dict(batch=1, total_q=128, total_k=128, max_len_q=128, max_len_k=128, topk=64)
    args.update(kw)
    return dsa.make_problem(**args)


FAKE = ctypes.c_void_p(1 << 20)     # aligned, never dereferenced: validation fails first


def test_null_problem_and_bad_sizes_are_rejected():
    lib = dsa.load()
    assert lib.dsa_topk(None, FAKE, 128, 0, 1, FAKE, None) == 1
    p = _problem(topk=0)
    assert lib.dsa_topk(ctypes.byref(p), FAKE, 128, 0, 1, FAKE, None) == 1
    p = _problem()
    assert lib.dsa_topk(ctypes.byref(p), FAKE, 126, 0, 1, FAKE, None) == 1      # ld % 4 != 0
    assert lib.dsa_topk(ctypes.byref(p), FAKE, 128, 100, 29, FAKE, None) == 1   # rows past total_q
    assert lib.dsa_topk(ctypes.byref(p), ctypes.c_void_p((1 << 20) + 4), 128, 0, 1, FAKE, None) == 1  # misaligned
    p = _problem(total_q=200)                                                   # T > S without cu arrays
    assert lib.dsa_sparse_mla_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None) == 1


def test_unsupported_shapes_are_reported():
    lib = dsa.load()
    for kw in (dict(n_heads=64), dict(d_qk=192), dict(n_idx_heads=32), dict(idx_dim=64), dict(topk=4096)):
        p = _problem(**kw)
        assert lib.dsa_sparse_mla_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None) == 2, kw


def test_dense_form_with_index_rows_limits_the_key_count():
    lib = dsa.load()
    p = _problem(total_q=64, total_k=20000, max_len_q=64, max_len_k=20000, topk=64)
    assert lib.dsa_dense_mla_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, None) == 2
    p = _problem()
    assert lib.dsa_dense_mla_fwd(ctypes.byref(p), None, FAKE, None, FAKE, FAKE, None) == 1   # q missing


def test_workspace_query_and_too_small_workspace():
    lib = dsa.load()
    p = _problem(total_q=1000, total_k=1000, max_len_q=1000, max_len_k=1000, topk=128)
    full = lib.dsa_forward_workspace_size(ctypes.byref(p), 0)
    chunked = lib.dsa_forward_workspace_size(ctypes.byref(p), 100)
    assert full >= 1000 * 1000 * 4 + 1000 * 128 * 4
    assert chunked < full
    args = [ctypes.byref(p)] + [FAKE] * 7 + [0, None, FAKE, FAKE, FAKE, ctypes.c_size_t(full - 1), None]
    assert lib.dsa_forward(*args) == 3
    args[12] = ctypes.c_void_p((1 << 20) + 16)                          # not 256-byte aligned
    args[13] = ctypes.c_size_t(full)
    assert lib.dsa_forward(*args) == 3
    assert lib.dsa_forward_workspace_size(None, 0) == 0


def test_binding_refuses_host_tensors():
    import torch

    p = _problem()
    with pytest.raises(ValueError):
        dsa.dsa_topk(p, torch.zeros(128, 128), torch.zeros(128, 64, dtype=torch.int32))
