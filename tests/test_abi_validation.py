"""Argument checks of every C-ABI entry point, on the host, without a GPU.

The interface promises that a call which returns an error other than
MSA_ERR_CUDA has enqueued nothing. With no GPU in the process, any CUDA call
the library makes fails, so a call that reaches the device before checking its
arguments returns MSA_ERR_CUDA (4) instead of the code tested here: each case
below therefore also shows that the check comes before any CUDA work.
"""
import ctypes
import os
import subprocess
import sys

import numpy as np
import pytest

from tests.test_abi import load_build_module

INVALID, WORKSPACE, UNSUPPORTED, CAPACITY = 1, 2, 3, 6
FAKE = 0x1000  # a non-NULL pointer that is never dereferenced by the checks


def _gpu_visible() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:  # pragma: no cover
        return False


# The cases below hand the library pointers that only the host checks keep
# from reaching a kernel. In a process that can see a GPU they would run on
# the device if a check ever moved, so there they are skipped and re-run as a
# whole in a child process with no GPU visible (the last test of this file).
_HOST_ONLY = os.environ.get("CUDA_VISIBLE_DEVICES") == "" or not _gpu_visible()
host_only = pytest.mark.skipif(not _HOST_ONLY, reason="runs in a child process with no GPU visible")


@pytest.fixture(scope="module")
def msa():
    load_build_module().build()
    import routed_sparse_attention_msa_b200 as m
    return m


def _last(msa):
    return msa._lib.msa_last_error().decode()


# ---------------------------------------------------------------- route

def _bank(msa, **kw):
    b = msa.BankLayerC(n_docs=10, n_chunks=20, hr=8, hkv=8, d=128, max_doc_chunks=4, doc_chunk_off=FAKE,
                       chunk_doc=FAKE, kbar_r=FAKE, kr_inv_norm=FAKE, kbar=FAKE, vbar=FAKE, content_on_host=0,
                       reserved=0)
    for k, v in kw.items():
        setattr(b, k, v)
    return b


ROUTE_CASES = [
    # (bank fields, call fields, expected code, message fragment)
    (dict(n_docs=0), {}, INVALID, "n_docs"),
    (dict(n_chunks=-1), {}, INVALID, "n_chunks"),
    (dict(d=64), {}, UNSUPPORTED, "d = 64"),
    (dict(hr=3), {}, UNSUPPORTED, "hr = 3"),
    (dict(hr=18), {}, UNSUPPORTED, "hr = 18"),
    (dict(kbar_r=None), {}, INVALID, "routing arrays"),
    (dict(kr_inv_norm=None), {}, INVALID, "routing arrays"),
    ({}, dict(n_seq=0), UNSUPPORTED, "n_seq = 0"),
    ({}, dict(top_k=0), INVALID, "top_k = 0"),
    (dict(n_docs=10000), dict(top_k=5000), UNSUPPORTED, "> 4096"),
    ({}, dict(qr=None), INVALID, "NULL pointer"),
    ({}, dict(top_ids=None), INVALID, "NULL pointer"),
    ({}, dict(eps=0.0), INVALID, "eps"),
    ({}, dict(eps=float("nan")), INVALID, "eps"),
    ({}, dict(q_seq_off=[0, 3]), INVALID, "end at n_rows"),
    ({}, dict(q_seq_off=[1, 2], n_rows=2), INVALID, "start at 0"),
    ({}, dict(q_seq_off=[0, 2, 2], n_seq=2), INVALID, "sequence 1 has no query rows"),
    ({}, dict(ws_bytes=16), WORKSPACE, "workspace"),
    ({}, dict(ws=None), WORKSPACE, "workspace"),
]


@host_only
@pytest.mark.parametrize("bank_kw, call_kw, code, frag", ROUTE_CASES)
def test_route_argument_checks(msa, bank_kw, call_kw, code, frag):
    b = _bank(msa, **bank_kw)
    c = dict(qr=FAKE, q_seq_off=[0, 2], n_seq=1, n_rows=2, top_k=16, eps=1e-8, top_ids=FAKE, top_scores=FAKE,
             ws=FAKE, ws_bytes=1 << 30)
    c.update(call_kw)
    qso = np.array(c["q_seq_off"], np.int32)
    rc = msa._lib.msa_route(ctypes.byref(b), c["qr"], qso.ctypes.data, c["n_seq"], c["n_rows"], c["top_k"], c["eps"],
                            c["top_ids"], c["top_scores"], None, c["ws"], c["ws_bytes"], None)
    assert rc == code, _last(msa)
    assert frag in _last(msa)


@host_only
def test_route_workspace_and_static_checks(msa):
    n = ctypes.c_size_t()
    b = _bank(msa)
    assert msa._lib.msa_route_workspace(ctypes.byref(b), 1, 1, 16, None) == INVALID
    assert msa._lib.msa_route_workspace(None, 1, 1, 16, ctypes.byref(n)) == INVALID
    assert msa._lib.msa_route_workspace(ctypes.byref(b), 2, 1, 16, ctypes.byref(n)) == INVALID  # rows < seqs
    assert msa._lib.msa_route_workspace(ctypes.byref(b), 1, 1, 16, ctypes.byref(n)) == 0
    # the static-scratch entry point: the same checks, then its capacity
    qso = np.array([0, 1], np.int32)
    bad = _bank(msa, d=64)
    assert msa._lib.msa_route_static(ctypes.byref(bad), FAKE, qso.ctypes.data, 1, 1, 16, 1e-8, FAKE, FAKE, None,
                                     None) == UNSUPPORTED
    big = _bank(msa, n_docs=4_000_000, n_chunks=8_000_000)
    qso = np.array([0, 1], np.int32)
    rc = msa._lib.msa_route_static(ctypes.byref(big), FAKE, qso.ctypes.data, 1, 1, 16, 1e-8, FAKE, FAKE, None, None)
    assert rc == CAPACITY and "static scratch" in _last(msa)


# ---------------------------------------------------------------- top-k merge

@host_only
def test_topk_merge_checks(msa):
    off = np.zeros(65, np.int64)
    f = msa._lib.msa_topk_merge
    assert f(None, FAKE, off.ctypes.data, 2, 1, 16, 16, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, None, 2, 1, 16, 16, FAKE, FAKE, None) == INVALID
    assert f(FAKE, FAKE, off.ctypes.data, 2, 1, 16, 33, FAKE, FAKE, None) == INVALID  # k_out > n_shards * k
    assert f(FAKE, FAKE, off.ctypes.data, 2, 0, 16, 16, FAKE, FAKE, None) == INVALID  # no sequence
    assert f(FAKE, FAKE, off.ctypes.data, 0, 1, 16, 16, FAKE, FAKE, None) == INVALID  # no shard
    assert f(FAKE, FAKE, off.ctypes.data, 64, 1, 128, 16, FAKE, FAKE, None) == UNSUPPORTED  # 8192 candidates
    assert f(FAKE, FAKE, off.ctypes.data, 65, 1, 1, 16, FAKE, FAKE, None) == UNSUPPORTED  # more than 64 shards
    neg = off.copy()
    neg[1] = -5
    assert f(FAKE, FAKE, neg.ctypes.data, 2, 1, 16, 16, FAKE, FAKE, None) == INVALID
    assert "id_offset[1]" in _last(msa)


# ---------------------------------------------------------------- gather

def _gather(msa, bank, **kw):
    g = msa.GatherArgsC(bank=ctypes.pointer(bank), top_ids=FAKE, n_seq=1, top_k=4, sel_off=FAKE, sel_chunk=FAKE,
                        cap=1 << 20, stage_k=FAKE, stage_v=FAKE, mode=msa.GATHER_DEVICE_PULL, reserved=0,
                        doc_chunk_off_host=FAKE, top_ids_host=FAKE, copy_stream=FAKE, done_event=FAKE,
                        timeout_us=0)
    for k, v in kw.items():
        setattr(g, k, v)
    return g


@pytest.mark.parametrize("bank_kw, call_kw, code, frag", [
    (dict(hkv=0), {}, UNSUPPORTED, "hkv"),
    (dict(kbar=None), {}, INVALID, "content arrays"),
    (dict(max_doc_chunks=-1), {}, INVALID, "max_doc_chunks"),
    ({}, dict(n_seq=0), INVALID, "bad sizes"),
    ({}, dict(top_k=0), INVALID, "bad sizes"),
    ({}, dict(sel_chunk=None), INVALID, "NULL pointer"),
    ({}, dict(cap=15), CAPACITY, "cap = 15"),
    # host-tier arguments are checked before the chunk listing is enqueued
    (dict(content_on_host=1), dict(stage_v=None), INVALID, "staging buffers"),
    (dict(content_on_host=1), dict(mode=7), INVALID, "unknown mode 7"),
    (dict(content_on_host=1), dict(mode=0, done_event=None), INVALID, "copy-engine mode needs"),
    (dict(content_on_host=1), dict(mode=0, top_ids_host=None), INVALID, "copy-engine mode needs"),
])
@host_only
def test_gather_argument_checks(msa, bank_kw, call_kw, code, frag):
    b = _bank(msa, **bank_kw)
    g = _gather(msa, b, **call_kw)
    rc = msa._lib.msa_gather(ctypes.byref(g), None)
    assert rc == code, _last(msa)
    assert frag in _last(msa)
    assert msa._lib.msa_gather(None, None) == INVALID


# ---------------------------------------------------------------- attend

def _attend(msa, **kw):
    h = dict(q_seq_off=[0, 1], q_start=[0], loc_off=[0, 1])
    for k in list(h):
        if k in kw:
            h[k] = kw.pop(k)
    arrs = {k: np.array(v, np.int32) for k, v in h.items()}
    a = msa.AttendArgsC(q=FAKE, q_seq_off=arrs["q_seq_off"].ctypes.data, q_start=arrs["q_start"].ctypes.data,
                        n_seq=1, n_q=1, hq=32, hkv=8, d=128, reserved=0, k_loc=FAKE, v_loc=FAKE,
                        loc_off=arrs["loc_off"].ctypes.data, mem_k=FAKE, mem_v=FAKE, sel_off=FAKE, sel_chunk=FAKE,
                        max_sel=16, pos_offset=16.0, rope_theta=1e6, scale=0.0, out=FAKE, out_f32=FAKE, lse=FAKE)
    for k, v in kw.items():
        setattr(a, k, v)
    return a, arrs  # the arrays must outlive the call


ATTEND_CASES = [
    (dict(d=64), UNSUPPORTED, "d = 64"),
    (dict(hq=20), INVALID, "multiple of hkv"),
    (dict(hkv=0), INVALID, "multiple of hkv"),
    (dict(hq=48, hkv=8), UNSUPPORTED, "hq / hkv = 6"),
    (dict(hq=256, hkv=8), UNSUPPORTED, "hq / hkv = 32"),
    (dict(n_seq=0), UNSUPPORTED, "n_seq = 0"),
    (dict(q=None), INVALID, "NULL pointer"),
    (dict(out=None), INVALID, "NULL pointer"),
    (dict(q_seq_off=[0, 2]), INVALID, "end at n_q"),
    (dict(loc_off=[1, 1]), INVALID, "loc_off[0]"),
    (dict(q_seq_off=[0, 2, 1], q_start=[0, 0], loc_off=[0, 1, 2], n_seq=2), INVALID, "decrease at sequence 1"),
    (dict(q_start=[-1]), INVALID, "q_start[0] < 0"),
    (dict(k_loc=None), INVALID, "local K/V"),
    (dict(max_sel=-1), INVALID, "max_sel"),
    (dict(mem_v=None), INVALID, "memory K/V"),
    (dict(rope_theta=1.0), INVALID, "rope_theta"),
    # the routed form (top_ids instead of a gather listing)
    (dict(top_ids=FAKE), INVALID, "exactly one"),
    (dict(sel_off=None), INVALID, "exactly one"),
    (dict(sel_off=None, top_ids=FAKE, doc_chunk_off=FAKE, n_docs=5, top_k=4), INVALID, "no sel_chunk"),
    (dict(sel_off=None, sel_chunk=None, top_ids=FAKE, n_docs=5, top_k=4), INVALID, "doc_chunk_off"),
    (dict(sel_off=None, sel_chunk=None, top_ids=FAKE, doc_chunk_off=FAKE, n_docs=5, top_k=0), INVALID, "top_k = 0"),
    (dict(sel_off=None, sel_chunk=None, top_ids=FAKE, doc_chunk_off=FAKE, n_docs=5, top_k=5000), INVALID,
     "top_k = 5000"),
    (dict(sel_off=None, sel_chunk=None, top_ids=FAKE, doc_chunk_off=FAKE, n_docs=-1, top_k=4), INVALID, "n_docs"),
]


@host_only
@pytest.mark.parametrize("kw, code, frag", ATTEND_CASES)
def test_attend_argument_checks(msa, kw, code, frag):
    a, keep = _attend(msa, **dict(kw))
    n = ctypes.c_size_t()
    for rc in (msa._lib.msa_attend_workspace(ctypes.byref(a), ctypes.byref(n)),
               msa._lib.msa_attend(ctypes.byref(a), FAKE, 1 << 30, None),
               msa._lib.msa_attend_backward_workspace(ctypes.byref(a), ctypes.byref(n)),
               msa._lib.msa_attend_backward(ctypes.byref(a), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                            None)):
        assert rc == code, _last(msa)
        assert frag in _last(msa)


@host_only
def test_attend_valid_arguments_need_a_workspace(msa):
    a, keep = _attend(msa)
    n = ctypes.c_size_t()
    assert msa._lib.msa_attend_workspace(ctypes.byref(a), ctypes.byref(n)) == 0 and n.value > 0
    assert msa._lib.msa_attend_workspace(ctypes.byref(a), None) == INVALID
    assert msa._lib.msa_attend(ctypes.byref(a), FAKE, n.value - 1, None) == WORKSPACE
    assert msa._lib.msa_attend(ctypes.byref(a), None, n.value, None) == WORKSPACE
    # no query rows: nothing to do, nothing enqueued
    z, keep2 = _attend(msa, q_seq_off=[0, 0], n_q=0)
    assert msa._lib.msa_attend(ctypes.byref(z), FAKE, 1 << 30, None) == 0


@host_only
def test_more_than_256_sequences_are_served_in_groups(msa):
    """Route and attention take any number of sequences (groups of 256 run in
    turn); their argument checks cover every sequence; the attention backward
    stays at 256."""
    S = 300
    qso = np.arange(S + 1, dtype=np.int32)
    b = _bank(msa)
    n = ctypes.c_size_t()
    n256 = ctypes.c_size_t()
    assert msa._lib.msa_route_workspace(ctypes.byref(b), S, S, 16, ctypes.byref(n)) == 0
    assert msa._lib.msa_route_workspace(ctypes.byref(b), 256, S, 16, ctypes.byref(n256)) == 0
    assert n.value == n256.value  # one group's layout
    bad = qso.copy()
    bad[271] = bad[270]  # sequence 270 has no rows: found before anything is enqueued
    assert msa._lib.msa_route(ctypes.byref(b), FAKE, bad.ctypes.data, S, S, 16, ctypes.c_float(1e-8), FAKE, FAKE,
                              None, FAKE, 1 << 30, None) == INVALID
    assert "sequence 270" in _last(msa)
    a, keep2 = _attend(msa, q_seq_off=qso, q_start=np.zeros(S, np.int32), loc_off=qso, n_seq=S, n_q=S)
    assert msa._lib.msa_attend_workspace(ctypes.byref(a), ctypes.byref(n)) == 0 and n.value > 0
    assert msa._lib.msa_attend_backward_workspace(ctypes.byref(a), ctypes.byref(n)) == UNSUPPORTED
    assert "n_seq = 300" in _last(msa)
    # the workspace of the whole call is the larger of its two groups' (256 and 44 sequences, the
    # second with longer local contexts so that it needs more)
    lo = np.r_[np.arange(257) * 2, 512 + np.arange(1, 45) * 60].astype(np.int32)
    whole, k4 = _attend(msa, q_seq_off=qso, q_start=np.r_[np.ones(256), np.full(44, 59)].astype(np.int32),
                        loc_off=lo, n_seq=S, n_q=S)
    g1, k5 = _attend(msa, q_seq_off=qso[:257], q_start=np.ones(256, np.int32), loc_off=lo[:257], n_seq=256, n_q=256)
    g2, k6 = _attend(msa, q_seq_off=qso[256:] - 256, q_start=np.full(44, 59, np.int32), loc_off=lo[256:] - lo[256],
                     n_seq=44, n_q=44)
    sizes = []
    for a_ in (whole, g1, g2):
        assert msa._lib.msa_attend_workspace(ctypes.byref(a_), ctypes.byref(n)) == 0
        sizes.append(n.value)
    assert sizes[0] == max(sizes[1], sizes[2]) and sizes[1] != sizes[2]
    neg, keep3 = _attend(msa, q_seq_off=qso, q_start=np.r_[np.zeros(280), -1, np.zeros(19)].astype(np.int32),
                         loc_off=qso, n_seq=S, n_q=S)
    assert msa._lib.msa_attend(ctypes.byref(neg), FAKE, 1 << 30, None) == INVALID
    assert "q_start[280]" in _last(msa)


@host_only
def test_attend_routed_form_is_forward_only(msa):
    a, keep = _attend(msa, sel_off=None, sel_chunk=None, top_ids=FAKE, doc_chunk_off=FAKE, n_docs=5, top_k=4)
    n = ctypes.c_size_t()
    assert msa._lib.msa_attend_workspace(ctypes.byref(a), ctypes.byref(n)) == 0 and n.value > 0
    assert msa._lib.msa_attend_backward_workspace(ctypes.byref(a), ctypes.byref(n)) == UNSUPPORTED
    assert msa._lib.msa_attend_backward(ctypes.byref(a), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                        None) == UNSUPPORTED
    assert "routed form" in _last(msa)


@host_only
def test_attend_backward_checks(msa):
    a, keep = _attend(msa)
    f = msa._lib.msa_attend_backward
    assert f(ctypes.byref(a), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == INVALID
    assert f(ctypes.byref(a), FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == INVALID  # dk_loc
    assert f(ctypes.byref(a), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None) == INVALID  # dmem_v
    assert f(ctypes.byref(a), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == WORKSPACE
    a.lse = None
    assert f(ctypes.byref(a), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == INVALID
    assert "out_f32 and lse" in _last(msa)


# ---------------------------------------------------------------- encode, norms, backward of route

def _encode(msa, **kw):
    e = msa.EncodeArgsC(k_tok=FAKE, v_tok=FAKE, kr_tok=FAKE, doc_tok_off=FAKE, n_docs=2, n_tok=100, n_chunks=3,
                        hkv=8, hr=8, d=128, chunk=64, rope_theta=1e6, eps=1e-8, kbar=FAKE, vbar=FAKE, kbar_r=FAKE,
                        kr_inv_norm=FAKE, doc_chunk_off=FAKE, chunk_doc=FAKE, rope_mode=0, reserved=0)
    for k, v in kw.items():
        setattr(e, k, v)
    return e


@pytest.mark.parametrize("kw, code, frag", [
    (dict(d=96), UNSUPPORTED, "d = 96"),
    (dict(hkv=17), UNSUPPORTED, "hkv = 17"),
    (dict(hr=0), UNSUPPORTED, "hr = 0"),
    (dict(chunk=0), INVALID, "chunk = 0"),
    (dict(chunk=2048), INVALID, "chunk = 2048"),
    (dict(n_docs=0), INVALID, "bad sizes"),
    (dict(n_tok=-1), INVALID, "bad sizes"),
    (dict(rope_theta=0.5), INVALID, "rope_theta"),
    (dict(eps=0.0), INVALID, "eps"),
    (dict(doc_chunk_off=None), INVALID, "NULL offsets"),
    (dict(rope_mode=2), INVALID, "rope_mode = 2"),
    (dict(kr_inv_norm=None), INVALID, "NULL tensor"),
])
@host_only
def test_encode_argument_checks(msa, kw, code, frag):
    e = _encode(msa, **kw)
    assert msa._lib.msa_encode(ctypes.byref(e), None) == code, _last(msa)
    assert frag in _last(msa)
    assert msa._lib.msa_encode(None, None) == INVALID


@host_only
def test_bank_norms_and_route_backward_checks(msa):
    f = msa._lib.msa_bank_norms
    assert f(FAKE, 10, 8, 64, 1e-8, FAKE, None) == UNSUPPORTED
    assert f(FAKE, 10, 0, 128, 1e-8, FAKE, None) == INVALID
    assert f(FAKE, -1, 8, 128, 1e-8, FAKE, None) == INVALID
    assert f(FAKE, 10, 8, 128, 0.0, FAKE, None) == INVALID
    assert f(None, 10, 8, 128, 1e-8, FAKE, None) == INVALID
    b = _bank(msa)
    qso = np.array([0, 2], np.int32)
    g = msa._lib.msa_route_backward
    args = lambda **kw: {**dict(qr=FAKE, qso=qso.ctypes.data, n_seq=1, n_rows=2, eps=1e-8, n_pairs=4, dqr=FAKE), **kw}
    def call(**kw):
        c = args(**kw)
        return g(ctypes.byref(b), c["qr"], c["qso"], c["n_seq"], c["n_rows"], c["eps"], FAKE, FAKE, FAKE,
                 c["n_pairs"], c["dqr"], FAKE, FAKE, FAKE, None)
    assert call(n_pairs=-1) == INVALID
    assert call(n_seq=0) == INVALID
    assert call(eps=-1.0) == INVALID
    assert call(n_rows=3) == INVALID
    assert call(qso=None) == INVALID
    assert call(dqr=None) == INVALID and "NULL pointer" in _last(msa)
    empty = np.array([0, 0, 2], np.int32)
    assert call(qso=empty.ctypes.data, n_seq=2) == INVALID and "no rows" in _last(msa)


@pytest.mark.skipif(_HOST_ONLY, reason="this process already runs the checks without a GPU")
def test_argument_checks_in_a_process_without_gpu():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider", os.path.abspath(__file__)],
                       cwd=root, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
