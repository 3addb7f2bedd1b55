"""Python binding of ``libmsa.so``, the C-ABI library of the MSA routing +
sparse attention step on B200 (declarations: ``include/msa.h``).

Argument marshalling only: tensors contribute their device pointers, the
current CUDA stream is passed through, host-side metadata (offsets) is passed
as host arrays. Every step of the path runs in the library's kernels; there is
no fallback. Importing this module fails if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmsa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python routed_sparse_attention_msa_b200/_build.py` "
        "(or __graft_entry__.build()); there is no non-CUDA implementation")

_lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
i32, i64, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float

MSA_OK = 0
STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_WORKSPACE", 3: "MSA_ERR_UNSUPPORTED",
          4: "MSA_ERR_CUDA", 5: "MSA_ERR_TIMEOUT", 6: "MSA_ERR_CAPACITY"}
GATHER_COPY_ENGINE = 0
GATHER_DEVICE_PULL = 1


class MsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = _lib.msa_last_error().decode()
        super().__init__(f"{where}: {STATUS.get(code, code)}: {msg}")


class BankLayerC(ctypes.Structure):
    _fields_ = [("n_docs", i64), ("n_chunks", i64), ("hr", i32), ("hkv", i32), ("d", i32),
                ("max_doc_chunks", i32), ("doc_chunk_off", P), ("chunk_doc", P), ("kbar_r", P),
                ("kr_inv_norm", P), ("kbar", P), ("vbar", P), ("content_on_host", i32), ("reserved", i32)]


class EncodeArgsC(ctypes.Structure):
    _fields_ = [("k_tok", P), ("v_tok", P), ("kr_tok", P), ("doc_tok_off", P), ("n_docs", i64),
                ("n_tok", i64), ("n_chunks", i64), ("hkv", i32), ("hr", i32), ("d", i32), ("chunk", i32),
                ("rope_theta", f32), ("eps", f32), ("kbar", P), ("vbar", P), ("kbar_r", P),
                ("kr_inv_norm", P), ("doc_chunk_off", P), ("chunk_doc", P), ("rope_mode", i32), ("reserved", i32)]


class GatherArgsC(ctypes.Structure):
    _fields_ = [("bank", ctypes.POINTER(BankLayerC)), ("top_ids", P), ("n_seq", i32), ("top_k", i32),
                ("sel_off", P), ("sel_chunk", P), ("cap", i64), ("stage_k", P), ("stage_v", P),
                ("mode", i32), ("reserved", i32), ("doc_chunk_off_host", P), ("top_ids_host", P),
                ("copy_stream", P), ("done_event", P), ("timeout_us", i64)]


class AttendArgsC(ctypes.Structure):
    _fields_ = [("q", P), ("q_seq_off", P), ("q_start", P), ("n_seq", i32), ("n_q", i32), ("hq", i32),
                ("hkv", i32), ("d", i32), ("reserved", i32), ("k_loc", P), ("v_loc", P), ("loc_off", P),
                ("mem_k", P), ("mem_v", P), ("sel_off", P), ("sel_chunk", P), ("max_sel", i64),
                ("pos_offset", f32), ("rope_theta", f32), ("scale", f32), ("out", P), ("out_f32", P),
                ("lse", P), ("top_ids", P), ("doc_chunk_off", P), ("n_docs", i64), ("top_k", i32),
                ("reserved2", i32)]


def _sig(name, args, res=ctypes.c_int):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_sig("msa_status_string", [ctypes.c_int], ctypes.c_char_p)
_sig("msa_last_error", [], ctypes.c_char_p)
_sig("msa_version", [])
_sig("msa_debug_set_score_kernel", [ctypes.c_int])
_sig("msa_debug_set_pf_block", [ctypes.c_int])
_sig("msa_debug_set_pf_pair", [ctypes.c_int])
_sig("msa_debug_wait_probe", [ctypes.c_void_p])
_sig("msa_debug_set_attend_kernel", [ctypes.c_int])
_sig("msa_debug_set_attend_splits", [ctypes.c_int])
_sig("msa_debug_set_topk_part", [ctypes.c_int])
_sig("msa_debug_set_tc_split_blocks", [ctypes.c_int])
_sig("msa_debug_set_dec_bulk", [ctypes.c_int])
_sig("msa_debug_set_dec_rot_keys", [ctypes.c_int])
_sig("msa_debug_tc_available", [])
_sig("msa_debug_launch_count", [], ctypes.c_longlong)
_sig("msa_debug_score_events", [P, P], None)
_sig("msa_encode_plan", [P, i64, i32, P, P, P])
_sig("msa_encode", [ctypes.POINTER(EncodeArgsC), P])
_sig("msa_bank_norms", [P, i64, i32, i32, f32, P, P])
_sig("msa_route_workspace", [ctypes.POINTER(BankLayerC), i32, i32, i32, ctypes.POINTER(ctypes.c_size_t)])
_sig("msa_route", [ctypes.POINTER(BankLayerC), P, P, i32, i32, i32, f32, P, P, P, P, ctypes.c_size_t, P])
_sig("msa_route_static", [ctypes.POINTER(BankLayerC), P, P, i32, i32, i32, f32, P, P, P, P])
_sig("msa_topk_merge", [P, P, P, i32, i32, i32, i32, P, P, P])
_sig("msa_gather", [ctypes.POINTER(GatherArgsC), P])
_sig("msa_attend_workspace", [ctypes.POINTER(AttendArgsC), ctypes.POINTER(ctypes.c_size_t)])
_sig("msa_attend", [ctypes.POINTER(AttendArgsC), P, ctypes.c_size_t, P])
_sig("msa_sync_check", [P])
_sig("msa_route_backward", [ctypes.POINTER(BankLayerC), P, P, i32, i32, f32, P, P, P, i32, P, P, P, P, P])
_sig("msa_attend_backward_workspace", [ctypes.POINTER(AttendArgsC), ctypes.POINTER(ctypes.c_size_t)])
_sig("msa_attend_backward", [ctypes.POINTER(AttendArgsC), P, P, P, P, P, P, P, ctypes.c_size_t, P])

EXPORTS = ["msa_status_string", "msa_last_error", "msa_version", "msa_encode_plan", "msa_encode",
           "msa_bank_norms", "msa_route_workspace", "msa_route", "msa_route_static", "msa_topk_merge", "msa_gather", "msa_attend_workspace",
           "msa_attend", "msa_sync_check", "msa_route_backward", "msa_attend_backward_workspace",
           "msa_attend_backward"]


def _check(code: int, where: str) -> None:
    if code != MSA_OK:
        raise MsaError(code, where)


def _ptr(t) -> int:
    if t is None:
        return 0
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return int(t.data_ptr())


def _host_i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _stream(stream=None) -> int:
    if stream is not None:
        return int(stream)
    import torch
    return int(torch.cuda.current_stream().cuda_stream)


def version() -> int:
    return _lib.msa_version()


def tc_available() -> bool:
    """True if the tensor-core scoring kernel is compiled into the library."""
    return bool(_lib.msa_debug_tc_available())


def launch_count() -> int:
    """Kernels this library has launched in the process so far."""
    return int(_lib.msa_debug_launch_count())


def score_events(begin, end) -> None:
    """Record torch.cuda.Events ``begin``/``end`` around the scoring kernel of
    the calling thread's next route call (both must already exist)."""
    _lib.msa_debug_score_events(int(begin.cuda_event), int(end.cuda_event))


def set_attend_kernel(which: str) -> str:
    """'auto', 'split' (split-K kernel), 'tc' (tensor cores, many rows),
    'tc_dec' (tensor cores with the keys as M) or 'dec' (the decoding kernel
    that 'auto' picks when a sequence's query vectors fill less than half a
    128-vector tile); returns the previous setting. Testing control."""
    names = ["auto", "split", "tc", "tc_dec", "dec"]
    return names[_lib.msa_debug_set_attend_kernel(names.index(which))]


def set_attend_splits(n: int) -> int:
    """Force the split-K attention's key splits (1..64; 0 = planned); returns
    the previous setting. Workspace sizes follow it: query attend_workspace
    after changing it. Benchmarking control."""
    return int(_lib.msa_debug_set_attend_splits(int(n)))


def set_dec_bulk(on: bool) -> bool:
    """Move the decoding attention kernel's rows by bulk copies (True) or by
    16-byte cp.async pieces (False); returns the previous setting. Testing
    control."""
    return bool(_lib.msa_debug_set_dec_bulk(1 if on else 0))


def set_tc_split_blocks(n: int) -> int:
    """Fewest 64-key blocks per key split of the many-row tensor-core attention
    (1..64); returns the previous setting. Benchmarking control."""
    return int(_lib.msa_debug_set_tc_split_blocks(int(n)))


def set_topk_part(n: int) -> int:
    """Documents per CTA of the k <= 16 top-k (1024..16384, a power of two; 0:
    the planned 2,048); returns the previous setting. Workspace sizes follow
    it. Benchmarking control."""
    return int(_lib.msa_debug_set_topk_part(int(n)))


def set_dec_rot_keys(n: int) -> int:
    """Largest per-CTA share of local keys the decoding attention kernel rotates
    itself (0..256; 0: a separate rotation kernel always does); returns the
    previous setting. Workspace sizes follow it. Testing control."""
    return int(_lib.msa_debug_set_dec_rot_keys(int(n)))


def wait_probe() -> None:
    """Launch a kernel whose bounded wait runs out (nothing arrives on its
    barrier); the next sync_check raises with MSA_ERR_TIMEOUT. Testing control
    for the failure path."""
    _check(_lib.msa_debug_wait_probe(_stream(None)), "wait_probe")


def set_pf_pair(on: bool) -> bool:
    """Run the many-row scorer's 192-row blocks on CTA pairs (one M = 256 MMA
    over two SMs) or on single CTAs; returns the previous setting. Testing
    control."""
    return bool(_lib.msa_debug_set_pf_pair(1 if on else 0))


def set_pf_block(rows: int) -> int:
    """Force the many-row scorer's query-row block (64, 128, 160 or 192; 0 =
    choose by padding); returns the previous setting. Testing control."""
    return _lib.msa_debug_set_pf_block(int(rows))


def set_score_kernel(which: str) -> str:
    """'auto', 'simt' (CUDA cores), 'tc' (tensor cores, per-head accumulators)
    or 'tc_rows' (tensor cores, folded scales, for many query rows); returns
    the previous setting."""
    names = ["auto", "simt", "tc", "tc_rows"]
    return names[_lib.msa_debug_set_score_kernel(names.index(which))]


# ------------------------------------------------------------------ encode

def encode_plan(doc_tok_off_host, chunk: int = 64):
    """Host planning. Returns (n_chunks, doc_chunk_off_host int64 [D+1], max_doc_chunks)."""
    off = np.ascontiguousarray(doc_tok_off_host, dtype=np.int64)
    n_docs = off.size - 1
    n = ctypes.c_int64()
    dco = np.empty(n_docs + 1, np.int64)
    mx = ctypes.c_int32()
    _check(_lib.msa_encode_plan(off.ctypes.data, n_docs, chunk, ctypes.addressof(n), dco.ctypes.data,
                                ctypes.addressof(mx)), "msa_encode_plan")
    return n.value, dco, mx.value


def encode(k_tok, v_tok, kr_tok, doc_tok_off, n_chunks: int, out: dict, chunk: int = 64,
           rope_theta: float = 1e6, eps: float = 1e-8, rope_mode: int = 0, stream=None) -> None:
    """Encode one layer. Per-token tensors [n_tok, heads, 128] bf16 on the device,
    doc_tok_off int64 device; ``out`` holds device tensors kbar, vbar, kbar_r,
    kr_inv_norm, doc_chunk_off, chunk_doc."""
    a = EncodeArgsC(_ptr(k_tok), _ptr(v_tok), _ptr(kr_tok), _ptr(doc_tok_off), doc_tok_off.numel() - 1,
                    k_tok.shape[0], n_chunks, k_tok.shape[1], kr_tok.shape[1], k_tok.shape[2], chunk,
                    rope_theta, eps, _ptr(out["kbar"]), _ptr(out["vbar"]), _ptr(out["kbar_r"]),
                    _ptr(out["kr_inv_norm"]), _ptr(out["doc_chunk_off"]), _ptr(out["chunk_doc"]), rope_mode, 0)
    _check(_lib.msa_encode(ctypes.byref(a), _stream(stream)), "msa_encode")


def bank_norms(kbar_r, kr_inv_norm, eps: float = 1e-8, stream=None) -> None:
    C, hr, d = kbar_r.shape
    _check(_lib.msa_bank_norms(_ptr(kbar_r), C, hr, d, eps, _ptr(kr_inv_norm), _stream(stream)),
           "msa_bank_norms")


# -------------------------------------------------------------------- bank

@dataclass
class BankLayer:
    """Tensors of one routing layer (device unless content_on_host)."""
    doc_chunk_off: object   # int64 [D+1] device
    chunk_doc: object       # int32 [C] device
    kbar_r: object          # bf16 [C, hr, 128] device
    kr_inv_norm: object     # fp32 [C, hr] device
    kbar: object = None     # bf16 [C, hkv, 128] device or pinned host
    vbar: object = None
    content_on_host: bool = False
    max_doc_chunks: int = 0

    def c(self) -> BankLayerC:
        C, hr, d = self.kbar_r.shape
        hkv = self.kbar.shape[1] if self.kbar is not None else 0
        return BankLayerC(self.doc_chunk_off.numel() - 1, C, hr, hkv, d, self.max_doc_chunks,
                          _ptr(self.doc_chunk_off), _ptr(self.chunk_doc), _ptr(self.kbar_r),
                          _ptr(self.kr_inv_norm), _ptr(self.kbar), _ptr(self.vbar),
                          int(self.content_on_host), 0)


# ------------------------------------------------------------------- route

def route_workspace(bank: BankLayer, n_seq: int, n_rows: int, top_k: int) -> int:
    b = bank.c()
    n = ctypes.c_size_t()
    _check(_lib.msa_route_workspace(ctypes.byref(b), n_seq, n_rows, top_k, ctypes.byref(n)),
           "msa_route_workspace")
    return n.value


def route(bank: BankLayer, qr, q_seq_off_host, top_k: int, top_ids, top_scores, workspace,
          all_doc_scores=None, eps: float = 1e-8, stream=None) -> None:
    """Route one layer. qr bf16 [T, hr, 128] device; q_seq_off host [S+1];
    top_ids int32 / top_scores fp32 [S, min(top_k, D)] device."""
    b = bank.c()
    qso = _host_i32(q_seq_off_host)
    _check(_lib.msa_route(ctypes.byref(b), _ptr(qr), qso.ctypes.data, qso.size - 1, qr.shape[0], top_k, eps,
                          _ptr(top_ids), _ptr(top_scores), _ptr(all_doc_scores), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(stream)), "msa_route")


def topk_merge(ids, scores, id_offset_host, k_out: int, top_ids, top_scores, stream=None) -> None:
    """Merge per-shard top-k lists ids/scores [G, S, k] (device; local ids, -1 =
    padding) with each shard's first global document id (host [G]) into the
    global top-k_out [S, k_out]."""
    G, S, k = ids.shape
    off = np.ascontiguousarray(np.asarray(id_offset_host, dtype=np.int64))
    _check(_lib.msa_topk_merge(_ptr(ids), _ptr(scores), off.ctypes.data, G, S, k, k_out, _ptr(top_ids),
                               _ptr(top_scores), _stream(stream)), "msa_topk_merge")


ROUTE_STATIC_SCRATCH_BYTES = 4 << 20  # MSA_ROUTE_STATIC_SCRATCH_BYTES


def route_static(bank: BankLayer, qr, q_seq_off_host, top_k: int, top_ids, top_scores, all_doc_scores=None,
                 eps: float = 1e-8, stream=None) -> None:
    """Route one layer without a workspace, for callers that may not allocate
    device memory: the library's fixed device scratch is used instead. Same
    results as ``route``. Calls on one device must not overlap on the GPU."""
    b = bank.c()
    qso = _host_i32(q_seq_off_host)
    _check(_lib.msa_route_static(ctypes.byref(b), _ptr(qr), qso.ctypes.data, qso.size - 1, qr.shape[0], top_k, eps,
                                 _ptr(top_ids), _ptr(top_scores), _ptr(all_doc_scores), _stream(stream)),
           "msa_route_static")


# ------------------------------------------------------------------ gather

def gather(bank: BankLayer, top_ids, top_k: int, sel_off, sel_chunk, stage_k=None, stage_v=None,
           mode: int = GATHER_COPY_ENGINE, doc_chunk_off_host=None, top_ids_host=None, copy_stream=None,
           done_event=None, timeout_us: int = 10_000_000, stream=None) -> None:
    b = bank.c()
    n_seq = top_ids.shape[0]
    if done_event is not None and int(done_event.cuda_event) == 0:
        done_event.record(copy_stream)  # torch creates the CUDA event lazily, on first record
    a = GatherArgsC(ctypes.pointer(b), _ptr(top_ids), n_seq, top_k, _ptr(sel_off), _ptr(sel_chunk),
                    sel_chunk.numel(), _ptr(stage_k), _ptr(stage_v), mode, 0, _ptr(doc_chunk_off_host),
                    _ptr(top_ids_host), int(copy_stream.cuda_stream) if copy_stream is not None else 0,
                    int(done_event.cuda_event) if done_event is not None else 0, timeout_us)
    _check(_lib.msa_gather(ctypes.byref(a), _stream(stream)), "msa_gather")


# ------------------------------------------------------------------ attend

def _attend_args(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk,
                 max_sel, pos_offset, rope_theta, scale, out, out_f32, lse, routed=None):
    """routed = (top_ids [n_seq, top_k] int32, doc_chunk_off [n_docs + 1] int64), both on the
    device, for the routed form (sel_off and sel_chunk None)."""
    qso, qst, lo = _host_i32(q_seq_off), _host_i32(q_start), _host_i32(loc_off)
    top_ids, dco = routed if routed is not None else (None, None)
    a = AttendArgsC(_ptr(q), qso.ctypes.data, qst.ctypes.data, qso.size - 1, q.shape[0], q.shape[1],
                    (k_loc if k_loc is not None else mem_k).shape[1], q.shape[2], 0, _ptr(k_loc), _ptr(v_loc),
                    lo.ctypes.data, _ptr(mem_k), _ptr(mem_v), _ptr(sel_off), _ptr(sel_chunk), int(max_sel),
                    float(pos_offset), float(rope_theta), float(scale), _ptr(out), _ptr(out_f32), _ptr(lse),
                    _ptr(top_ids), _ptr(dco), dco.numel() - 1 if dco is not None else 0,
                    top_ids.shape[1] if top_ids is not None else 0, 0)
    return a, (qso, qst, lo)


def attend_workspace(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk,
                     max_sel, pos_offset=16.0, rope_theta=1e6, scale=0.0, routed=None) -> int:
    a, keep = _attend_args(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk,
                           max_sel, pos_offset, rope_theta, scale, q, None, None, routed)
    n = ctypes.c_size_t()
    _check(_lib.msa_attend_workspace(ctypes.byref(a), ctypes.byref(n)), "msa_attend_workspace")
    return n.value


def attend(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk, max_sel,
           out, workspace, out_f32=None, lse=None, pos_offset=16.0, rope_theta=1e6, scale=0.0,
           stream=None, routed=None) -> None:
    """With routed = (top_ids, doc_chunk_off) and sel_off = sel_chunk = None, the call lists
    the selected documents' chunks itself (the routed form of msa_attend)."""
    a, keep = _attend_args(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk,
                           max_sel, pos_offset, rope_theta, scale, out, out_f32, lse, routed)
    _check(_lib.msa_attend(ctypes.byref(a), _ptr(workspace), workspace.numel() * workspace.element_size(),
                           _stream(stream)), "msa_attend")


def route_backward(bank: BankLayer, qr, q_seq_off_host, pair_seq, pair_doc, pair_dscore, dqr, dkr, argmax_chunk,
                   argmax_row, eps: float = 1e-8, stream=None) -> None:
    """Gradient of sum dscore * score(seq, doc) over (seq, doc, dscore) triples
    (device arrays). dqr [T, hr, 128] fp32 is accumulated (zero it first)."""
    b = bank.c()
    qso = _host_i32(q_seq_off_host)
    _check(_lib.msa_route_backward(ctypes.byref(b), _ptr(qr), qso.ctypes.data, qso.size - 1, qr.shape[0], eps,
                                   _ptr(pair_seq), _ptr(pair_doc), _ptr(pair_dscore), pair_seq.numel(), _ptr(dqr),
                                   _ptr(dkr), _ptr(argmax_chunk), _ptr(argmax_row), _stream(stream)),
           "msa_route_backward")


def attend_backward_workspace(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk,
                              max_sel, out_f32, lse, pos_offset=16.0, rope_theta=1e6, scale=0.0) -> int:
    a, keep = _attend_args(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk,
                           max_sel, pos_offset, rope_theta, scale, q, out_f32, lse)
    n = ctypes.c_size_t()
    _check(_lib.msa_attend_backward_workspace(ctypes.byref(a), ctypes.byref(n)), "msa_attend_backward_workspace")
    return n.value


def attend_backward(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk, max_sel,
                    out_f32, lse, dout, dq, dk_loc, dv_loc, dmem_k, dmem_v, workspace, pos_offset=16.0,
                    rope_theta=1e6, scale=0.0, stream=None) -> None:
    """Gradients of ``attend`` given the forward's fp32 output and lse."""
    a, keep = _attend_args(q, q_seq_off, q_start, k_loc, v_loc, loc_off, mem_k, mem_v, sel_off, sel_chunk,
                           max_sel, pos_offset, rope_theta, scale, q, out_f32, lse)
    _check(_lib.msa_attend_backward(ctypes.byref(a), _ptr(dout), _ptr(dq), _ptr(dk_loc), _ptr(dv_loc), _ptr(dmem_k),
                                    _ptr(dmem_v), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)), "msa_attend_backward")


def sync_check(stream=None) -> None:
    _check(_lib.msa_sync_check(_stream(stream)), "msa_sync_check")
