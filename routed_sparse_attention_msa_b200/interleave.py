"""Memory Interleave: multi-hop retrieval that alternates routing and
context expansion.

["MSA: Memory Sparse Attention", Key Contributions and Inference Pipeline
(Figure 3): generative retrieval -> context expansion -> generation, repeated;
"MSA-arXiv26", 核心方法 / Memory Interleave: generate a document id, fetch the
document, add it to the query, retrieve again, until there is enough
evidence]

Without a model, the step that generates the next document id is a fixed
rule: the best-scoring document of the hop that has not been fetched yet. The
fetched document joins the query as its pooled routing keys (one extra
routing row per chunk, the stand-in for re-encoding the appended text), and
the next hop routes with the grown query. Every hop runs the library's
routing kernels; the loop itself is host logic.
"""
from __future__ import annotations

import numpy as np

import routed_sparse_attention_msa_b200 as msa


def next_document(top_ids_row, taken) -> int:
    """The generated document id of a hop: the highest-ranked document not yet fetched."""
    for d in top_ids_row:
        if int(d) not in taken:
            return int(d)
    return -1


def memory_interleave(bank: "msa.BankLayer", doc_chunk_off_host, qr, top_k: int, hops: int, eps: float = 1e-8):
    """One sequence's multi-hop retrieval. qr: its routing rows [T, hr, 128]
    (device bf16). Returns (fetched document ids per hop, top-k ids of every
    hop [hops, k], the final routing rows)."""
    import torch
    dco = np.asarray(doc_chunk_off_host, np.int64)
    k = min(top_k, int(dco.size - 1))
    fetched: list[int] = []
    per_hop = []
    rows = qr
    for _ in range(hops):
        ids = torch.empty((1, k), dtype=torch.int32, device=qr.device)
        sc = torch.empty((1, k), dtype=torch.float32, device=qr.device)
        ws = torch.empty(msa.route_workspace(bank, 1, rows.shape[0], top_k), dtype=torch.uint8, device=qr.device)
        msa.route(bank, rows, [0, rows.shape[0]], top_k, ids, sc, ws, eps=eps)
        top = ids.cpu().numpy()[0]  # the model reads the ranking to generate the next id
        per_hop.append(top)
        d = next_document(top, set(fetched))
        if d < 0:
            break
        fetched.append(d)
        c0, c1 = int(dco[d]), int(dco[d + 1])
        rows = torch.cat([rows, bank.kbar_r[c0:c1]], dim=0)  # the fetched document joins the query
    return fetched, np.stack(per_hop), rows
