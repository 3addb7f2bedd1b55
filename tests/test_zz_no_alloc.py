"""msa_route_static: routing for callers that cannot allocate device memory.

Callers such as a serving process whose framework owns all of HBM through its
own pool, or a latency-critical loop that cannot accept cudaMalloc's implicit
synchronisation, may not allocate a routing workspace. msa_route_static uses
the library's fixed device scratch instead. These tests call it through the C
ABI and check, on two calls in a row with different queries, that it returns
what msa_route (with a caller-provided workspace) returns, within the
tolerance of the other routing tests (ids exact, scores within 1e-3).
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

import synth
from tests.gpu_common import DevBank, from_bits

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _route_both(msa, bank, qr_bits, qso, k):
    S, kk = len(qso) - 1, min(k, bank.n_docs)
    qr = from_bits(qr_bits)
    out = []
    for fn in ("route", "route_static"):
        ids = torch.full((S, kk), -1, dtype=torch.int32, device="cuda")
        sc = torch.full((S, kk), float("nan"), dtype=torch.float32, device="cuda")
        alls = torch.full((S, bank.n_docs), float("nan"), dtype=torch.float32, device="cuda")
        if fn == "route":
            ws = torch.empty(msa.route_workspace(bank.layer_c, S, qr.shape[0], k), dtype=torch.uint8, device="cuda")
            msa.route(bank.layer_c, qr, qso, k, ids, sc, ws, all_doc_scores=alls)
        else:
            msa.route_static(bank.layer_c, qr, qso, k, ids, sc, all_doc_scores=alls)
        msa.sync_check()
        out.append((ids.cpu().numpy(), sc.cpu().numpy(), alls.cpu().numpy()))
    return out


def test_route_static_matches_route_on_two_calls_in_a_row():
    import routed_sparse_attention_msa_b200 as msa
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, 0, content=False)
    for call, rows in enumerate(([32], [1, 5, 2])):
        qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, rows, 16, 3, 8, 128, 0,
                                                   call=10 + call)
        (ids_a, sc_a, all_a), (ids_b, sc_b, all_b) = _route_both(msa, bank, qr, qso, 16)
        np.testing.assert_array_equal(ids_b, ids_a)
        np.testing.assert_allclose(sc_b, sc_a, atol=1e-3, rtol=0)
        np.testing.assert_allclose(all_b, all_a, atol=1e-3, rtol=0)
        for s in range(len(rows)):
            assert set(ids_b[s].tolist()) == set(plan.docs[s])


def test_route_static_rejects_calls_beyond_its_scratch():
    """A call whose scratch need exceeds the array is refused on the host with
    MSA_ERR_CAPACITY. Every pointer is a real device buffer of the right size,
    so the call would be valid (and in bounds) if the capacity check ever moved."""
    import routed_sparse_attention_msa_b200 as msa
    # 256 sequences x 4,200 documents need 4.3 MB of per-document keys: more than the 4 MiB scratch.
    n_docs, n_seq, k = 4200, 256, 16
    bank = DevBank(np.arange(n_docs + 1, dtype=np.int64) * 64, 1, content=False)
    need = msa.route_workspace(bank.layer_c, n_seq, n_seq, k)
    assert need > msa.ROUTE_STATIC_SCRATCH_BYTES
    qr = torch.zeros((n_seq, 8, 128), dtype=torch.bfloat16, device="cuda")
    ids = torch.full((n_seq, k), -1, dtype=torch.int32, device="cuda")
    sc = torch.zeros((n_seq, k), dtype=torch.float32, device="cuda")
    qso = np.arange(n_seq + 1, dtype=np.int32)
    with pytest.raises(msa.MsaError) as ei:
        msa.route_static(bank.layer_c, qr, qso, k, ids, sc)
    assert ei.value.code == 6  # MSA_ERR_CAPACITY
    assert "static scratch" in str(ei.value)
    msa.sync_check()
    assert bool((ids == -1).all())  # nothing was enqueued
