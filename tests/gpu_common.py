"""Helpers for the GPU tests: synthetic banks on the device, host copies for
the oracle, and the comparison rules for top-k results."""
from __future__ import annotations

import numpy as np

import synth

try:
    import torch
except Exception:  # pragma: no cover
    torch = None


def stream():
    return int(torch.cuda.current_stream().cuda_stream)


def dev_normal(shape, tensor_id, sigma=1.0, index0=0):
    t = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    synth.normal_bf16_device(t.data_ptr(), t.numel(), tensor_id, index0, sigma, stream=stream())
    return t


def host_normal(shape, tensor_id, sigma=1.0, index0=0):
    n = int(np.prod(shape))
    return synth.normal_bf16_host(n, tensor_id, index0, sigma).reshape(shape)


def bits(t) -> np.ndarray:
    """bfloat16 device tensor -> uint16 bit patterns on the host."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


class DevBank:
    """One synthetic routing layer on the device (content in HBM or pinned host)."""

    def __init__(self, doc_tok_off, layer, hr=8, hkv=8, content=True, on_host=False, chunk=64):
        import routed_sparse_attention_msa_b200 as msa
        self.doc_tok_off = np.asarray(doc_tok_off, np.int64)
        self.dco, self.cdoc = synth.chunk_index(self.doc_tok_off, chunk)
        self.C = int(self.dco[-1])
        self.hr, self.hkv, self.layer = hr, hkv, layer
        self.kbar_r = dev_normal((self.C, hr, 128), synth.tid("kbar_r", layer))
        self.inv = torch.empty((self.C, hr), dtype=torch.float32, device="cuda")
        msa.bank_norms(self.kbar_r, self.inv)
        self.kbar = self.vbar = None
        if content:
            if on_host:
                self.kbar = torch.empty((self.C, hkv, 128), dtype=torch.bfloat16, pin_memory=True)
                self.vbar = torch.empty((self.C, hkv, 128), dtype=torch.bfloat16, pin_memory=True)
                synth.normal_bf16_host_into(self.kbar.data_ptr(), self.kbar.numel(), synth.tid("kbar", layer))
                synth.normal_bf16_host_into(self.vbar.data_ptr(), self.vbar.numel(), synth.tid("vbar", layer))
            else:
                self.kbar = dev_normal((self.C, hkv, 128), synth.tid("kbar", layer))
                self.vbar = dev_normal((self.C, hkv, 128), synth.tid("vbar", layer))
        nch = np.diff(self.dco)
        self.layer_c = msa.BankLayer(
            doc_chunk_off=torch.from_numpy(self.dco).cuda(), chunk_doc=torch.from_numpy(self.cdoc).cuda(),
            kbar_r=self.kbar_r, kr_inv_norm=self.inv, kbar=self.kbar, vbar=self.vbar,
            content_on_host=on_host, max_doc_chunks=int(nch.max()) if nch.size else 0)

    @property
    def n_docs(self):
        return self.dco.size - 1

    def host_kbar_r(self):
        return host_normal((self.C, self.hr, 128), synth.tid("kbar_r", self.layer))

    def host_chunk_kbar_r(self, c):
        return synth.bits_to_f64(host_normal((self.hr, 128), synth.tid("kbar_r", self.layer),
                                             index0=c * self.hr * 128))

    def host_content(self):
        return (host_normal((self.C, self.hkv, 128), synth.tid("kbar", self.layer)),
                host_normal((self.C, self.hkv, 128), synth.tid("vbar", self.layer)))


def route_gpu(bank: DevBank, qr_bits, q_seq_off, top_k, want_all=True):
    import routed_sparse_attention_msa_b200 as msa
    S = len(q_seq_off) - 1
    k = min(top_k, bank.n_docs)
    qr = from_bits(qr_bits)
    ids = torch.empty((S, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((S, k), dtype=torch.float32, device="cuda")
    alls = torch.empty((S, bank.n_docs), dtype=torch.float32, device="cuda") if want_all else None
    ws = torch.empty(msa.route_workspace(bank.layer_c, S, qr.shape[0], top_k), dtype=torch.uint8, device="cuda")
    msa.route(bank.layer_c, qr, q_seq_off, top_k, ids, sc, ws, all_doc_scores=alls)
    msa.sync_check()
    return ids.cpu().numpy(), sc.cpu().numpy(), (alls.cpu().numpy() if want_all else None)


def gap_at_k(scores_row: np.ndarray, k: int) -> float:
    if k >= scores_row.size:
        return np.inf
    s = np.sort(scores_row)[::-1]
    return float(s[k - 1] - s[k])


def check_topk(g_ids, g_sc, o_ids, o_sc, o_all, tol=1e-3, exact_gap=1e-2, order_gap=1e-4):
    """Compare a GPU top-k with the oracle's. Returns the number of sequences
    compared bit-exactly. Where the oracle's gap at rank k is >= exact_gap the
    id sets must be identical, and the order too where adjacent selected
    scores differ by more than order_gap; elsewhere the GPU's selection must
    be valid (each pick's oracle score within tol of the oracle's rank score)."""
    S, k = o_ids.shape
    assert g_ids.shape == (S, k)
    n_exact = 0
    for s in range(S):
        picked = o_all[s][g_ids[s]]
        np.testing.assert_allclose(g_sc[s], picked, atol=tol, rtol=0)
        np.testing.assert_allclose(picked, o_sc[s], atol=tol, rtol=0)
        assert len(set(g_ids[s].tolist())) == k
        if gap_at_k(o_all[s], k) >= exact_gap:
            assert set(g_ids[s].tolist()) == set(o_ids[s].tolist()), s
            n_exact += 1
            for i in range(k):
                lo = o_sc[s][i] - (o_sc[s][i + 1] if i + 1 < k else -np.inf)
                hi = (o_sc[s][i - 1] if i > 0 else np.inf) - o_sc[s][i]
                if min(lo, hi) > order_gap:
                    assert g_ids[s][i] == o_ids[s][i], (s, i)
    return n_exact
