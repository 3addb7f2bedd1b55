"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds none of the method's arithmetic: it draws numbers, lays out
document structures and builds query vectors with prescribed cosines. Both the
CUDA library (through device buffers) and the CPU oracle (through host arrays)
receive what it produces; neither side computes its own inputs.

The generator (``synth.cu``) is SplitMix64 used counter-style, so any slice of
a multi-gigabyte tensor can be regenerated bit-identically on the host.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa_synth.so")
_SRC = os.path.join(_HERE, "synth.cu")

SEED = 0x4D5341  # "MSA"

_lib = None


def build(force: bool = False) -> str:
    """Compile ``synth/libmsa_synth.so`` (host generator + sm_100a fill kernel)."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(_SRC):
        cmd = [
            "nvcc", "-O2", "-shared", "-std=c++17",
            "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-fmad=false",
            "-Xcompiler", "-fPIC,-fopenmp,-ffp-contract=off",
            "-o", LIB_PATH, _SRC, "-lgomp",
        ]
        subprocess.run(cmd, check=True)
    return LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB_PATH)
        P, i64, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64
        lib.synth_normal_bf16_host.argtypes = [P, i64, u64, u64, i64, ctypes.c_float]
        lib.synth_normal_bf16_host.restype = ctypes.c_int
        lib.synth_normal_bf16_device.argtypes = [P, i64, u64, u64, i64, ctypes.c_float, P]
        lib.synth_normal_bf16_device.restype = ctypes.c_int
        lib.synth_u64_host.argtypes = [P, i64, u64, u64, i64]
        lib.synth_u64_host.restype = ctypes.c_int
        _lib = lib
    return _lib


# ------------------------------------------------------------ tensor streams

def tid(kind: str, layer: int = 0, extra: int = 0) -> int:
    """Stream id of one synthetic tensor (independent streams per kind/layer)."""
    base = {
        "kbar_r": 0x100, "kbar": 0x200, "vbar": 0x300,
        "k_tok": 0x400, "v_tok": 0x500, "kr_tok": 0x600,
        "q_noise": 0x700, "q_att": 0x800, "k_loc": 0x900, "v_loc": 0xA00,
        "doc_len": 0xB00, "plant": 0xC00,
    }[kind]
    return (base << 32) | (layer << 16) | extra


def normal_bf16_host(n: int, tensor_id: int, index0: int = 0, sigma: float = 1.0,
                     seed: int = SEED) -> np.ndarray:
    """Draws index0..index0+n-1 of a stream as bfloat16 bit patterns (uint16)."""
    out = np.empty(int(n), np.uint16)
    if n:
        _load().synth_normal_bf16_host(out.ctypes.data_as(ctypes.c_void_p), int(n), seed,
                                       tensor_id, int(index0), float(sigma))
    return out


def normal_bf16_device(ptr: int, n: int, tensor_id: int, index0: int = 0, sigma: float = 1.0,
                       stream: int = 0, seed: int = SEED) -> None:
    """Same values as ``normal_bf16_host``, written to device memory at ``ptr``."""
    rc = _load().synth_normal_bf16_device(ctypes.c_void_p(ptr), int(n), seed, tensor_id,
                                          int(index0), float(sigma), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"synthetic fill kernel failed (cudaError {rc})")


def normal_bf16_host_into(ptr: int, n: int, tensor_id: int, index0: int = 0, sigma: float = 1.0,
                          seed: int = SEED) -> None:
    """Like ``normal_bf16_host`` but writes into existing host memory at ``ptr``."""
    _load().synth_normal_bf16_host(ctypes.c_void_p(ptr), int(n), seed, tensor_id, int(index0), float(sigma))


def u64_host(n: int, tensor_id: int, index0: int = 0, seed: int = SEED) -> np.ndarray:
    out = np.empty(int(n), np.uint64)
    if n:
        _load().synth_u64_host(out.ctypes.data_as(ctypes.c_void_p), int(n), seed, tensor_id,
                               int(index0))
    return out


def uniform01(n: int, tensor_id: int, index0: int = 0, seed: int = SEED) -> np.ndarray:
    """Uniform doubles in (0, 1] from the top 53 bits of each draw."""
    r = u64_host(n, tensor_id, index0, seed)
    return ((r >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bfloat16 bits (nearest, ties to even) for building inputs."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(
        np.float32).astype(np.float64)


# ------------------------------------------------------- document structure

def doc_offsets_uniform(n_docs: int, length: int) -> np.ndarray:
    return np.arange(n_docs + 1, dtype=np.int64) * int(length)


def doc_offsets_lognormal(total: int, mu: float, sigma: float, lo: int, hi: int,
                          multiple: int = 1, stream: int = 0) -> np.ndarray:
    """Document lengths drawn log-normally (Box-Muller on SplitMix64 uniforms),
    clipped to [lo, hi], rounded up to ``multiple``, drawn until they reach
    ``total`` tokens; the last document is cut so the sum is exactly ``total``."""
    lens = []
    acc = 0
    i = 0
    batch = 4096
    while acc < total:
        u = uniform01(2 * batch, tid("doc_len", extra=stream), index0=2 * i)
        u1, u2 = u[0::2], u[1::2]
        z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
        ln = np.clip(np.exp(mu + sigma * z), lo, hi)
        ln = (np.ceil(ln / multiple) * multiple).astype(np.int64)
        for v in ln:
            v = int(min(v, total - acc))
            lens.append(v)
            acc += v
            if acc >= total:
                break
        i += batch
    return np.concatenate([[0], np.cumsum(np.asarray(lens, np.int64))]).astype(np.int64)


def chunk_index(doc_tok_off: np.ndarray, chunk: int):
    """The chunk structure of a synthetic bank: chunks per document, the
    document-to-chunk offsets and each chunk's document."""
    lens = np.diff(doc_tok_off)
    nch = (lens + chunk - 1) // chunk
    dco = np.concatenate([[0], np.cumsum(nch)]).astype(np.int64)
    cdoc = np.repeat(np.arange(lens.size, dtype=np.int32), nch)
    return dco, cdoc


# ------------------------------------------------ queries with planted docs

def plant_row(keys: np.ndarray, cos_targets: np.ndarray, noise: np.ndarray,
              magnitude: float):
    """One routing query row [hr, d] whose cosine with each planted key
    ``keys[j]`` ([m, hr, d]) is prescribed in every head (before bfloat16
    rounding): the minimum-norm vector with those inner products against the
    unit keys, completed to unit length by a noise direction orthogonal to
    them, then scaled by ``magnitude``. If the targets cannot all be met in a
    head (squared norm of the minimum-norm vector above 0.95) that head's
    targets are scaled down together. Returns (row, designed mean-over-heads
    cosine of each planted key)."""
    m, hr, d = keys.shape
    out = np.empty((hr, d))
    c = np.asarray(cos_targets, np.float64)
    scales = np.empty(hr)
    for h in range(hr):
        K = keys[:, h, :] / np.linalg.norm(keys[:, h, :], axis=1, keepdims=True)
        G = K @ K.T
        a = np.linalg.solve(G, c)
        n0 = float(c @ a)
        sh = min(1.0, math.sqrt(0.95 / n0))
        q0 = (K.T @ a) * sh
        n0 *= sh * sh
        r = noise[h] - K.T @ np.linalg.lstsq(K.T, noise[h], rcond=None)[0]
        r /= np.linalg.norm(r)
        out[h] = (q0 + math.sqrt(1.0 - n0) * r) * magnitude
        scales[h] = sh
    return out, c * scales.mean()


def planted_targets(k: int, n_needles: int, per_row: int) -> np.ndarray:
    """Cosine targets of the k planted documents of one sequence: needles
    first, then graded decoys, all well above the noise maximum and spaced
    apart. ``per_row`` is how many planted documents share one query row."""
    if per_row <= 1:
        needles = np.full(n_needles, 0.99) - 0.002 * np.arange(n_needles)
        decoys = np.linspace(0.9, 0.35, max(k - n_needles, 0)) if k > n_needles else np.zeros(0)
        return np.concatenate([needles, decoys])[:k]
    # Several planted documents in one row: their squared cosines must sum
    # below 1, so the needle is lower and decoys are packed just above noise.
    needles = np.full(n_needles, 0.36) - 0.01 * np.arange(n_needles)
    decoys = 0.19 + 0.005 * np.arange(max(k - n_needles, 0))[::-1]
    return np.concatenate([needles, decoys])[:k]


@dataclass
class Plan:
    """Planted documents of one routing call: ``docs[s]`` are sequence s's
    planted document ids (needles first), ``chunks[s]`` the planted chunk of
    each, ``cos[s]`` the designed scores."""
    docs: list = field(default_factory=list)
    chunks: list = field(default_factory=list)
    cos: list = field(default_factory=list)


def make_routing_queries(kbar_r_rows, doc_chunk_off: np.ndarray, rows_per_seq: list[int],
                         top_k: int, n_needles: int, hr: int, d: int, layer: int,
                         call: int = 0, magnitude: float | None = None):
    """Build Qr [T, hr, d] (bfloat16 bits) and q_seq_off for one routing call.

    ``kbar_r_rows(c)`` returns the pooled routing key of chunk c as float64
    [hr, d] (regenerated on the host). Each sequence gets top_k planted
    documents (distinct, chosen at random, each with one random chunk); if the
    sequence has at least top_k rows, row j carries planted document j alone,
    otherwise the planted documents are spread over the rows and superposed.
    Remaining rows are N(0,1) noise."""
    n_docs = doc_chunk_off.size - 1
    n_seq = len(rows_per_seq)
    T = int(sum(rows_per_seq))
    if magnitude is None:
        magnitude = math.sqrt(d)
    q_seq_off = np.concatenate([[0], np.cumsum(rows_per_seq)]).astype(np.int32)
    noise = bits_to_f64(normal_bf16_host(T * hr * d, tid("q_noise", layer, call))).reshape(T, hr, d)
    qr = noise.copy()
    plan = Plan()
    k = min(top_k, n_docs)
    nonempty = np.nonzero(np.diff(doc_chunk_off) > 0)[0]
    u = u64_host(64 * (k + 1) * n_seq + 64, tid("plant", layer, call))
    ui = 0
    for s in range(n_seq):
        rows = rows_per_seq[s]
        chosen: list[int] = []
        while len(chosen) < min(k, nonempty.size):
            cand = int(nonempty[int(u[ui] % np.uint64(nonempty.size))])
            ui += 1
            if cand not in chosen:
                chosen.append(cand)
        chunks = []
        for doc in chosen:
            nch = int(doc_chunk_off[doc + 1] - doc_chunk_off[doc])
            chunks.append(int(doc_chunk_off[doc]) + int(u[ui] % np.uint64(nch)))
            ui += 1
        per_row = max(1, math.ceil(len(chosen) / rows))
        targets = planted_targets(len(chosen), min(n_needles, len(chosen)), per_row)
        base = int(q_seq_off[s])
        for r in range(min(rows, len(chosen))):
            idx = list(range(r, len(chosen), rows))  # planted docs carried by this row
            keys = np.stack([kbar_r_rows(chunks[j]) for j in idx])
            qr[base + r], targets[idx] = plant_row(keys, targets[idx], noise[base + r], magnitude)
        plan.docs.append(chosen)
        plan.chunks.append(chunks)
        plan.cos.append(targets)
    return bf16_bits(qr.reshape(T, hr, d)), q_seq_off, plan


# ---------------------------------------------------------------- workloads

@dataclass
class Workload:
    """One synthetic workload shaped like the pages' memory banks."""
    name: str
    doc_tok_off: np.ndarray
    chunk: int = 64
    hr: int = 8
    hkv: int = 8
    hq: int = 32
    d: int = 128
    n_layers: int = 1
    n_seq: int = 1
    route_rows: int = 1        # routing rows per sequence in the timed call
    prefill_rows: int = 0      # routing rows per sequence at prefill (0: none)
    top_k: int = 16
    n_needles: int = 1
    loc_len: int = 1           # local (query + generated) tokens per sequence
    attn_rows: int = 1         # attention query rows per sequence
    content_on_host: bool = False
    rope_theta: float = 1e6
    eps: float = 1e-8

    @property
    def n_docs(self) -> int:
        return self.doc_tok_off.size - 1

    @property
    def memory_tokens(self) -> int:
        return int(self.doc_tok_off[-1])

    def index(self):
        return chunk_index(self.doc_tok_off, self.chunk)


def workload(name: str) -> Workload:
    """The five workloads: tiny, 1m, 10m, 100m (routing + attention) and encode."""
    if name == "tiny":
        # 256 docs x 512 tokens, chunk 64 -> 2048 chunks; 32 query rows, 3 needles.
        return Workload("tiny", doc_offsets_uniform(256, 512), n_layers=1, n_seq=1,
                        route_rows=32, top_k=16, n_needles=3, loc_len=32, attn_rows=32)
    if name == "1m":
        # 2048 docs x 512 tokens (16384 chunks/layer), 18 layers, 128-row prefill, decode.
        return Workload("1m", doc_offsets_uniform(2048, 512), n_layers=18, n_seq=1,
                        route_rows=1, prefill_rows=128, top_k=16, n_needles=1,
                        loc_len=129, attn_rows=1)
    if name == "10m":
        # log-normal documents (mean 1K tokens, clipped 64..8K), 16 sequences of 64 tokens.
        off = doc_offsets_lognormal(10_000_000, math.log(1024) - 0.5, 1.0, 64, 8192, 1, stream=3)
        return Workload("10m", off, n_layers=18, n_seq=16, route_rows=1, prefill_rows=64,
                        top_k=16, n_needles=1, loc_len=65, attn_rows=1)
    if name == "100m":
        # 1,562,500 chunks/layer, 18 layers of K-bar_r resident; content on the host.
        off = doc_offsets_lognormal(100_000_000, math.log(1024) - 0.5, 1.0, 64, 8192, 64, stream=4)
        return Workload("100m", off, n_layers=18, n_seq=1, route_rows=1, top_k=16,
                        n_needles=1, loc_len=128, attn_rows=1, content_on_host=True)
    if name == "encode":
        # 10M tokens in documents of 4096 (the last one 1664), 8 kv + 8 routing heads.
        lens = [4096] * 2441 + [1664]
        off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        return Workload("encode", off, n_layers=18)
    raise KeyError(name)
