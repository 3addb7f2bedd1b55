"""CPU oracle for the MSA routing + sparse attention step (ctypes binding).

TEST INFRASTRUCTURE ONLY. The tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` call it; the library's own path never imports
it. It shares no code with the CUDA library: ``msa_oracle.c`` is plain C,
single-threaded, fp64 sums, loops in the order of the definitions.

Definitions followed (page title, section):
  * "MSA: Memory Sparse Attention" (project README), Overall Design,
    Architecture and Figure 2: chunk-mean pooled K/V/K_r, cosine routing
    (head mean, then the max over query tokens), top-k documents, the selected
    pooled K/V joined to the query's own recent K/V; parallel (document-wise)
    RoPE from 0 and global RoPE offset by k.
  * same page, Inference Pipeline and Figure 3: offline encoding of
    (K-bar, V-bar, K-bar_r), online routing, loading only the selected K/V.
  * "MSA-arXiv26" (paper digest), 核心方法: the same steps.

Every function here is pinned by ``tests/test_oracle.py`` against closed forms,
invariants, library routines and brute force; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa_oracle.so")
_SRC = os.path.join(_HERE, "msa_oracle.c")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmsa_oracle.so`` with gcc."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "msa_oracle.h"))
    ):
        cmd = [
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
            "-fno-fast-math", "-Wall", "-o", LIB_PATH, _SRC, "-lm",
        ]
        subprocess.run(cmd, check=True)
    return LIB_PATH


def use_library(path: str | None) -> None:
    """Point the binding at another build of ``msa_oracle.c`` (the mutation
    test loads deliberately broken copies); ``None`` restores the default."""
    global _lib, _lib_path
    _lib = None
    _lib_path = path


_lib_path = None


def _load():
    global _lib
    if _lib is None:
        if _lib_path is None:
            build()
        lib = ctypes.CDLL(_lib_path or LIB_PATH)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_double.restype = f64
        lib.orc_double_to_bf16.argtypes = [f64]
        lib.orc_double_to_bf16.restype = ctypes.c_uint16
        lib.orc_double_array_to_bf16.argtypes = [P, i64, P]
        lib.orc_double_array_to_bf16.restype = None
        lib.orc_rope.argtypes = [P, i32, f64, f64]
        lib.orc_rope.restype = i32
        lib.orc_encode.argtypes = [P, P, P, P, i64, i32, i32, i32, i32, f64, f64, i32,
                                   P, P, P, P, P, P, i64]
        lib.orc_encode.restype = i32
        lib.orc_route.argtypes = [P, P, i64, i32, i32, P, P, i32, f64, i32, P, P, P]
        lib.orc_route.restype = i32
        lib.orc_gather.argtypes = [P, i32, i32, P, P, P, i64]
        lib.orc_gather.restype = i64
        lib.orc_attend.argtypes = [P, P, P, i32, i32, i32, i32, P, P, P, P, P, P, P,
                                   f64, f64, f64, P, P]
        lib.orc_attend.restype = i32
        lib.orc_route_f64.argtypes = [P, P, i64, i32, i32, P, P, i32, f64, i32, P, P, P]
        lib.orc_route_f64.restype = i32
        lib.orc_route_backward.argtypes = [P, P, i64, i32, i32, P, P, i32, f64, P, P, P, i32, P, P, P, P]
        lib.orc_route_backward.restype = i32
        lib.orc_attend_f64.argtypes = [P, P, P, i32, i32, i32, i32, P, P, P, P, P, P, P, f64, f64, f64, P, P,
                                       P, P, P, P, P, P]
        lib.orc_attend_f64.restype = i32
        _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bfloat16 values travel as uint16 bit patterns"
    return a


# ------------------------------------------------------------------ bfloat16

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even), via the oracle."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().orc_double_array_to_bf16(_p(x), x.size, _p(out))
    return out


def rope(x: np.ndarray, pos: float, theta: float) -> np.ndarray:
    """Rotary embedding of one vector (half-split pairing); returns a copy."""
    v = np.array(x, dtype=np.float64, copy=True)
    rc = _load().orc_rope(_p(v), v.size, float(pos), float(theta))
    if rc != 0:
        raise ValueError(f"orc_rope failed ({rc})")
    return v


# ------------------------------------------------------------------- encode

def encode(k_tok, v_tok, kr_tok, doc_tok_off, chunk=64, rope_theta=1e6, eps=1e-8, rope_mode=0):
    """Offline encode of one layer. Per-token arrays are uint16 bfloat16 bits
    shaped [n_tok, heads, d]. rope_mode 0 rotates tokens before pooling, 1
    rotates the pooled chunk at its chunk index. Returns the pooled outputs."""
    k_tok, v_tok, kr_tok = _u16(k_tok), _u16(v_tok), _u16(kr_tok)
    off = np.ascontiguousarray(doc_tok_off, dtype=np.int64)
    n_docs = off.size - 1
    hkv, d = k_tok.shape[1], k_tok.shape[2]
    hr = kr_tok.shape[1]
    lens = np.diff(off)
    n_chunks = int(((lens + chunk - 1) // chunk).sum())
    kbar = np.empty((n_chunks, hkv, d), np.uint16)
    vbar = np.empty((n_chunks, hkv, d), np.uint16)
    kbar_r = np.empty((n_chunks, hr, d), np.uint16)
    inv = np.empty((n_chunks, hr), np.float64)
    dco = np.empty(n_docs + 1, np.int64)
    cdoc = np.empty(max(n_chunks, 1), np.int32)
    rc = _load().orc_encode(_p(k_tok), _p(v_tok), _p(kr_tok), _p(off), n_docs, hkv, hr, d,
                            chunk, float(rope_theta), float(eps), int(rope_mode), _p(kbar), _p(vbar), _p(kbar_r),
                            _p(inv), _p(dco), _p(cdoc), n_chunks)
    if rc != 0:
        raise ValueError(f"orc_encode failed ({rc})")
    return dict(kbar=kbar, vbar=vbar, kbar_r=kbar_r, kr_inv_norm=inv,
                doc_chunk_off=dco, chunk_doc=cdoc[:n_chunks])


# -------------------------------------------------------------------- route

def route(kbar_r, doc_chunk_off, qr, q_seq_off, top_k, eps=1e-8, want_scores=True):
    """Routing of one layer. Returns (top_ids [S,k], top_scores [S,k], doc_scores [S,D])."""
    kbar_r, qr = _u16(kbar_r), _u16(qr)
    dco = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    qso = np.ascontiguousarray(q_seq_off, dtype=np.int32)
    n_docs = dco.size - 1
    hr, d = qr.shape[1], qr.shape[2]
    n_seq = qso.size - 1
    k = min(int(top_k), n_docs)
    ids = np.empty((n_seq, k), np.int32)
    sc = np.empty((n_seq, k), np.float64)
    ds = np.empty((n_seq, n_docs), np.float64) if want_scores else None
    rc = _load().orc_route(_p(kbar_r), _p(dco), n_docs, hr, d, _p(qr), _p(qso), n_seq,
                           float(eps), int(top_k), _p(ds), _p(ids), _p(sc))
    if rc != 0:
        raise ValueError(f"orc_route failed ({rc})")
    return ids, sc, ds


# ------------------------------------------------------------------- gather

def gather(top_ids, doc_chunk_off):
    """Selected chunk lists. Returns (sel_off [S+1], sel_chunk [n])."""
    ids = np.ascontiguousarray(top_ids, dtype=np.int32)
    dco = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    n_seq, k = ids.shape
    cap = int(sum(int(dco[i + 1] - dco[i]) for i in ids.ravel())) + 1
    sel_off = np.empty(n_seq + 1, np.int64)
    sel = np.empty(cap, np.int64)
    n = _load().orc_gather(_p(ids), n_seq, k, _p(dco), _p(sel_off), _p(sel), cap)
    if n < 0:
        raise ValueError(f"orc_gather failed ({n})")
    return sel_off, sel[:n]


# ------------------------------------------------------------------- attend

def attend(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk,
           pos_offset, rope_theta=1e6, scale=None):
    """Sparse attention. Returns (out [n_q, hq, d] float64, lse [n_q, hq] float64)."""
    q, k_loc, v_loc = _u16(q), _u16(k_loc), _u16(v_loc)
    mem_k, mem_v = _u16(mem_k), _u16(mem_v)
    qso = np.ascontiguousarray(q_seq_off, dtype=np.int32)
    qst = np.ascontiguousarray(q_start, dtype=np.int32)
    lo = np.ascontiguousarray(loc_off, dtype=np.int32)
    so = np.ascontiguousarray(sel_off, dtype=np.int64)
    sc = np.ascontiguousarray(sel_chunk, dtype=np.int64)
    if sc.size == 0:
        sc = np.zeros(1, np.int64)
    n_q, hq, d = q.shape
    hkv = k_loc.shape[1] if k_loc.size else mem_k.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if k_loc.size == 0:
        k_loc = np.zeros((1, hkv, d), np.uint16)
        v_loc = np.zeros((1, hkv, d), np.uint16)
    out = np.empty((n_q, hq, d), np.float64)
    lse = np.empty((n_q, hq), np.float64)
    rc = _load().orc_attend(_p(q), _p(qso), _p(qst), qso.size - 1, hq, hkv, d, _p(k_loc),
                            _p(v_loc), _p(lo), _p(mem_k), _p(mem_v), _p(so), _p(sc),
                            float(pos_offset), float(rope_theta), float(scale), _p(out), _p(lse))
    if rc != 0:
        raise ValueError(f"orc_attend failed ({rc})")
    return out, lse


# ------------------------------------------------- fp64 inputs and gradients

def _f64(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    return bf16_to_f64(a) if a.dtype == np.uint16 else np.ascontiguousarray(a, dtype=np.float64)


def route_scores_f64(kbar_r, doc_chunk_off, qr, q_seq_off, eps=1e-8):
    """Document scores [S, D] from fp64 inputs (same arithmetic as ``route``)."""
    kr, q = _f64(kbar_r), _f64(qr)
    dco = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    qso = np.ascontiguousarray(q_seq_off, dtype=np.int32)
    n_docs, n_seq = dco.size - 1, qso.size - 1
    ds = np.empty((n_seq, n_docs), np.float64)
    ids = np.empty((n_seq, 1), np.int32)
    sc = np.empty((n_seq, 1), np.float64)
    rc = _load().orc_route_f64(_p(kr), _p(dco), n_docs, q.shape[1], q.shape[2], _p(q), _p(qso), n_seq, float(eps),
                               1, _p(ds), _p(ids), _p(sc))
    if rc != 0:
        raise ValueError(f"orc_route_f64 failed ({rc})")
    return ds


def route_backward(kbar_r, doc_chunk_off, qr, q_seq_off, pair_seq, pair_doc, pair_dscore, eps=1e-8):
    """Gradients of sum_p dscore_p * score(seq_p, doc_p): (dqr [T, hr, d],
    dkr [P, hr, d], argmax_chunk [P], argmax_row [P])."""
    kr, q = _f64(kbar_r), _f64(qr)
    dco = np.ascontiguousarray(doc_chunk_off, dtype=np.int64)
    qso = np.ascontiguousarray(q_seq_off, dtype=np.int32)
    ps = np.ascontiguousarray(pair_seq, dtype=np.int32)
    pd = np.ascontiguousarray(pair_doc, dtype=np.int32)
    pg = np.ascontiguousarray(pair_dscore, dtype=np.float64)
    T, hr, d = q.shape
    dq = np.zeros((T, hr, d))
    dk = np.empty((ps.size, hr, d))
    ac = np.empty(ps.size, np.int64)
    ar = np.empty(ps.size, np.int32)
    rc = _load().orc_route_backward(_p(kr), _p(dco), dco.size - 1, hr, d, _p(q), _p(qso), qso.size - 1, float(eps),
                                    _p(ps), _p(pd), _p(pg), ps.size, _p(dq), _p(dk), _p(ac), _p(ar))
    if rc != 0:
        raise ValueError(f"orc_route_backward failed ({rc})")
    return dq, dk, ac, ar


def attend_f64(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk, pos_offset,
               rope_theta=1e6, scale=None, dout=None):
    """Attention from fp64 inputs; with ``dout`` also the gradients. Returns
    (out, lse) or (out, lse, dq, dk_loc, dv_loc, dmem_k, dmem_v)."""
    q, kl, vl, mk, mv = (_f64(x) for x in (q, k_loc, v_loc, mem_k, mem_v))
    qso = np.ascontiguousarray(q_seq_off, dtype=np.int32)
    qst = np.ascontiguousarray(q_start, dtype=np.int32)
    lo = np.ascontiguousarray(loc_off, dtype=np.int32)
    so = np.ascontiguousarray(sel_off, dtype=np.int64)
    sc = np.ascontiguousarray(sel_chunk, dtype=np.int64)
    if sc.size == 0:
        sc = np.zeros(1, np.int64)
    n_q, hq, d = q.shape
    hkv = kl.shape[1] if kl.size else mk.shape[1]
    if kl.size == 0:
        kl = np.zeros((1, hkv, d))
        vl = np.zeros((1, hkv, d))
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.empty((n_q, hq, d))
    lse = np.empty((n_q, hq))
    grads = None
    if dout is not None:
        go = np.ascontiguousarray(dout, dtype=np.float64)
        n_sel = int(so[-1])
        grads = [np.zeros((n_q, hq, d)), np.zeros(kl.shape), np.zeros(vl.shape),
                 np.zeros((max(n_sel, 1), hkv, d)), np.zeros((max(n_sel, 1), hkv, d))]
    rc = _load().orc_attend_f64(_p(q), _p(qso), _p(qst), qso.size - 1, hq, hkv, d, _p(kl), _p(vl), _p(lo), _p(mk),
                                _p(mv), _p(so), _p(sc), float(pos_offset), float(rope_theta), float(scale), _p(out),
                                _p(lse), _p(go) if grads else None, *([_p(g) for g in grads] if grads else [None] * 5))
    if rc != 0:
        raise ValueError(f"orc_attend_f64 failed ({rc})")
    if grads is None:
        return out, lse
    n_sel = int(so[-1])
    return (out, lse, grads[0], grads[1][: max(int(lo[-1]), 0)], grads[2][: max(int(lo[-1]), 0)],
            grads[3][:n_sel], grads[4][:n_sel])
