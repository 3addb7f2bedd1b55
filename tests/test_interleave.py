"""Memory Interleave on the GPU against the same loop run with the oracle."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_common import DevBank, from_bits

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _oracle_interleave(kr_host, dco, qr_bits, k, hops):
    """The interleave loop on the oracle. The generated id of a hop is the
    best-ranked document of that hop's top-k not fetched before (written out
    here, independently of the library's loop)."""
    fetched, per_hop, rows = [], [], qr_bits
    for _ in range(hops):
        ids, sc, ds = oracle.route(kr_host, dco, rows, [0, rows.shape[0]], k)
        per_hop.append((ids[0], ds[0]))
        fresh = [int(x) for x in ids[0] if int(x) not in fetched]
        assert fresh, "every top-k document already fetched"
        d = fresh[0]
        fetched.append(d)
        rows = np.concatenate([rows, kr_host[dco[d]:dco[d + 1]]])
    return fetched, per_hop


@pytest.mark.parametrize("rows", [1, 8])
def test_memory_interleave_matches_oracle_loop(rows):
    from routed_sparse_attention_msa_b200.interleave import memory_interleave
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, 5, content=False)
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, [rows], 16, 2, 8, 128, 5)
    fetched, per_hop, final_rows = memory_interleave(bank.layer_c, bank.dco, from_bits(qr), 16, hops=4)
    o_fetched, o_per_hop = _oracle_interleave(bank.host_kbar_r(), bank.dco, qr, 16, 4)
    assert fetched == o_fetched
    for h, (ids, ds) in enumerate(o_per_hop):
        s = np.sort(ds)[::-1]
        if s[15] - s[16] >= 1e-2:  # unique top-k set at this hop
            assert set(per_hop[h].tolist()) == set(ids.tolist())
    # the first hop retrieves the planted needles, later hops follow the fetched documents
    assert fetched[0] in plan.docs[0][:2]
    assert len(set(fetched)) == 4
    # every fetched document joined the query as one routing row per chunk
    assert final_rows.shape[0] == rows + sum(int(bank.dco[d + 1] - bank.dco[d]) for d in fetched)
