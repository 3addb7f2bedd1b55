"""Memory Parallel routing: the memory bank's documents split into contiguous
shards, one per GPU. Each GPU scores its shard with ``route`` (local document
ids), the k candidates of every sequence are all-gathered, and every rank
merges them with ``topk_merge`` into the global top-k, identical to routing
the unsharded bank.

["MSA: Memory Sparse Attention", Inference Pipeline: Memory Parallel splits
the routing keys over GPUs, each scores the query against its part, and the
results are reduced;
"MSA-arXiv26", 核心方法 / Memory Parallel inference]

Host-side planning and collective plumbing only; the scoring and the merge
run in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

import routed_sparse_attention_msa_b200 as msa


def shard_ranges(doc_chunk_off: np.ndarray, n_shards: int) -> list[tuple[int, int]]:
    """Contiguous document ranges [d0, d1) with chunk counts as even as whole
    documents allow."""
    dco = np.asarray(doc_chunk_off, np.int64)
    n_docs, total = dco.size - 1, int(dco[-1])
    bounds = [0]
    for g in range(1, n_shards):
        d = int(np.searchsorted(dco, g * total / n_shards, side="left"))
        bounds.append(min(max(d, bounds[-1]), n_docs))
    bounds.append(n_docs)
    return [(bounds[g], bounds[g + 1]) for g in range(n_shards)]


@dataclass
class Shard:
    layer: "msa.BankLayer"
    doc_begin: int
    doc_end: int

    @property
    def n_docs(self) -> int:
        return self.doc_end - self.doc_begin


def make_shard(bank: "msa.BankLayer", doc_chunk_off_host: np.ndarray, d0: int, d1: int) -> Shard:
    """The bank of documents [d0, d1) as a bank of its own: views of the
    routing keys, norms and content, and rebased document offsets and chunk
    owners."""
    import torch
    dco = np.asarray(doc_chunk_off_host, np.int64)
    c0, c1 = int(dco[d0]), int(dco[d1])
    local_dco = torch.from_numpy(dco[d0:d1 + 1] - c0).to(bank.kbar_r.device)
    nch = np.diff(dco[d0:d1 + 1])
    local_cdoc = torch.from_numpy(np.repeat(np.arange(d1 - d0, dtype=np.int32), nch)).to(bank.kbar_r.device)
    layer = msa.BankLayer(local_dco, local_cdoc, bank.kbar_r[c0:c1], bank.kr_inv_norm[c0:c1],
                          None if bank.kbar is None else bank.kbar[c0:c1],
                          None if bank.vbar is None else bank.vbar[c0:c1], bank.content_on_host,
                          int(nch.max()) if nch.size else 0)
    return Shard(layer, d0, d1)


def route_local(shard: Shard, qr, q_seq_off_host, top_k: int, ids_out, scores_out, workspace, eps=1e-8):
    """Route one shard into fixed [S, top_k] buffers, padding with id -1 when
    the shard has fewer than top_k documents."""
    kk = min(top_k, shard.n_docs)
    if kk < top_k:
        ids_out.fill_(-1)
        scores_out.fill_(float("-inf"))
    if kk == 0:  # a shard without documents contributes only padding
        return
    if kk == top_k:
        msa.route(shard.layer, qr, q_seq_off_host, top_k, ids_out, scores_out, workspace, eps=eps)
    else:  # a shard with fewer documents than top_k: route into a compact buffer, then place it
        import torch
        ti = torch.empty((ids_out.shape[0], kk), dtype=torch.int32, device=ids_out.device)
        ts = torch.empty((ids_out.shape[0], kk), dtype=torch.float32, device=ids_out.device)
        msa.route(shard.layer, qr, q_seq_off_host, top_k, ti, ts, workspace, eps=eps)
        ids_out[:, :kk] = ti
        scores_out[:, :kk] = ts


def gather_candidates(ids, scores, group=None):
    """All-gather every rank's [S, k] candidates into [G, S, k] (torch.distributed).
    NCCL gathers the device tensors directly (over NVLink); a gloo group gathers
    host copies, and the result is returned on the candidates' device."""
    import torch
    import torch.distributed as dist
    G = dist.get_world_size(group)
    dev = ids.device
    staged = dist.get_backend(group) == "gloo" and dev.type == "cuda"
    src_i = ids.contiguous().cpu() if staged else ids.contiguous()
    src_s = scores.contiguous().cpu() if staged else scores.contiguous()
    li = [torch.empty_like(src_i) for _ in range(G)]
    ls = [torch.empty_like(src_s) for _ in range(G)]
    dist.all_gather(li, src_i, group=group)
    dist.all_gather(ls, src_s, group=group)
    all_i, all_s = torch.stack(li), torch.stack(ls)
    if staged:
        all_i, all_s = all_i.to(dev), all_s.to(dev)
    return all_i, all_s


def route_memory_parallel(shard: Shard, doc_offsets: list[int], qr, q_seq_off_host, top_k: int, top_ids,
                          top_scores, workspace, group=None, eps=1e-8):
    """One rank's part of a Memory Parallel route: local scoring, all-gather of
    the candidates, merge. Every rank ends with the global [S, k] result."""
    import torch
    S = len(q_seq_off_host) - 1
    ids = torch.empty((S, top_k), dtype=torch.int32, device=qr.device)
    sc = torch.empty((S, top_k), dtype=torch.float32, device=qr.device)
    route_local(shard, qr, q_seq_off_host, top_k, ids, sc, workspace, eps)
    all_ids, all_sc = gather_candidates(ids, sc, group)
    msa.topk_merge(all_ids, all_sc, doc_offsets, top_ids.shape[1], top_ids, top_scores)
