"""The C-ABI library loads, exports every function that include/msa.h declares,
and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "msa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_0-9]+)\s*\(", text)))


def load_build_module():
    """The build script, loaded by path (importing the package needs the built library)."""
    import importlib.util
    path = os.path.join(ROOT, "routed_sparse_attention_msa_b200", "_build.py")
    spec = importlib.util.spec_from_file_location("msa_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module")
def msa():
    load_build_module().build()
    import routed_sparse_attention_msa_b200 as m
    return m


def test_every_declared_symbol_is_exported(msa):
    names = _declared()
    assert len(names) >= 12
    lib = ctypes.CDLL(msa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(msa.EXPORTS)


def test_version_and_status_strings(msa):
    assert msa.version() == 1
    for code, name in msa.STATUS.items():
        assert msa._lib.msa_status_string(code).decode() == name


def test_encode_plan_host_only(msa):
    off = np.array([0, 64, 127, 127, 320, 321], np.int64)
    n, dco, mx = msa.encode_plan(off, 64)
    assert n == 1 + 1 + 0 + 4 + 1
    assert dco.tolist() == [0, 1, 2, 2, 6, 7]
    assert mx == 4
    with pytest.raises(msa.MsaError) as e:
        msa.encode_plan(np.array([0, 10, 5], np.int64), 64)
    assert e.value.code == 1 and "decreases" in str(e.value)


def test_route_rejects_bad_arguments_before_launch(msa):
    b = msa.BankLayerC(10, 20, 8, 8, 64, 2, 1, 1, 1, 1, 1, 1, 0, 0)  # d = 64: unsupported
    n = ctypes.c_size_t()
    rc = msa._lib.msa_route_workspace(ctypes.byref(b), 1, 1, 16, ctypes.byref(n))
    assert rc == 3
    b.d = 128
    rc = msa._lib.msa_route_workspace(ctypes.byref(b), 1, 1, 16, ctypes.byref(n))
    assert rc == 0 and n.value > 0
    # a sequence without rows is an argument error (checked on the host)
    qso = np.array([0, 0, 2], np.int32)
    rc = msa._lib.msa_route(ctypes.byref(b), 1, qso.ctypes.data, 2, 2, 16, 1e-8, 1, 1, None, 1, 1 << 30, None)
    assert rc == 1 and "no query rows" in msa._lib.msa_last_error().decode()
    # too small a workspace
    qso = np.array([0, 2], np.int32)
    rc = msa._lib.msa_route(ctypes.byref(b), 1, qso.ctypes.data, 1, 2, 16, 1e-8, 1, 1, None, 1, 16, None)
    assert rc == 2


def test_attend_rejects_bad_group(msa):
    q = np.zeros(1, np.int32)
    a = msa.AttendArgsC(1, q.ctypes.data, q.ctypes.data, 1, 0, 24, 8, 128, 0, 1, 1, q.ctypes.data, 1, 1, 1, 0,
                        0, 16.0, 1e6, 0.0, 1, 0, 0)
    n = ctypes.c_size_t()
    assert msa._lib.msa_attend_workspace(ctypes.byref(a), ctypes.byref(n)) == 3  # 24 / 8 = 3


def test_gather_capacity_check(msa):
    b = msa.BankLayerC(10, 20, 8, 8, 128, 4, 1, 1, 1, 1, 1, 1, 0, 0)
    g = msa.GatherArgsC(ctypes.pointer(b), 1, 2, 16, 1, 1, 50, 0, 0, 0, 0, 0, 0, 0, 0, 0)
    rc = msa._lib.msa_gather(ctypes.byref(g), None)
    assert rc == 6  # cap 50 < n_seq * min(top_k, n_docs) * max_doc_chunks = 2 * 10 * 4
