"""Memory Parallel routing: the bank split into document shards, each routed
on its own, the candidates merged; the result must equal routing the whole
bank (ids and scores bit for bit) and agree with the oracle.

On one GPU the shards run one after another (no kernel waits on another);
the collective step is tested with gloo ranks in tests/test_dist_cpu.py.
"""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_common import DevBank, check_topk, from_bits, route_gpu

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _sharded(msa, mp, bank, qr_bits, qso, k, n_shards):
    ranges = mp.shard_ranges(bank.dco, n_shards)
    S = len(qso) - 1
    qr = from_bits(qr_bits)
    all_ids = torch.empty((n_shards, S, k), dtype=torch.int32, device="cuda")
    all_sc = torch.empty((n_shards, S, k), dtype=torch.float32, device="cuda")
    for g, (d0, d1) in enumerate(ranges):
        sh = mp.make_shard(bank.layer_c, bank.dco, d0, d1)
        if sh.n_docs == 0:
            all_ids[g].fill_(-1)
            all_sc[g].fill_(float("-inf"))
            continue
        ws = torch.empty(msa.route_workspace(sh.layer, S, qr.shape[0], k), dtype=torch.uint8, device="cuda")
        mp.route_local(sh, qr, qso, k, all_ids[g], all_sc[g], ws)
    kk = min(k, bank.n_docs)
    ids = torch.empty((S, kk), dtype=torch.int32, device="cuda")
    sc = torch.empty((S, kk), dtype=torch.float32, device="cuda")
    msa.topk_merge(all_ids, all_sc, [d0 for d0, _ in ranges], kk, ids, sc)
    msa.sync_check()
    return ids.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("workload,n_shards,rows", [("tiny", 2, [32]), ("tiny", 7, [1, 3]), ("10m", 8, [1] * 16),
                                                    ("1m", 3, [128])])
def test_sharded_route_equals_unsharded(workload, n_shards, rows):
    import routed_sparse_attention_msa_b200 as msa
    from routed_sparse_attention_msa_b200 import memory_parallel as mp
    w = synth.workload(workload)
    bank = DevBank(w.doc_tok_off, 0, content=False)
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, rows, w.top_k, w.n_needles,
                                               8, 128, 0)
    ids1, sc1, _ = route_gpu(bank, qr, qso, w.top_k, want_all=False)
    ids2, sc2 = _sharded(msa, mp, bank, qr, qso, w.top_k, n_shards)
    np.testing.assert_array_equal(ids2, ids1)
    np.testing.assert_array_equal(sc2, sc1)
    for s in range(len(rows)):
        assert set(ids2[s].tolist()) == set(plan.docs[s])


def test_sharded_route_k_larger_than_a_shard_matches_oracle():
    import routed_sparse_attention_msa_b200 as msa
    from routed_sparse_attention_msa_b200 import memory_parallel as mp
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, 1, content=False)
    qr, qso, _ = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, [4], 16, 2, 8, 128, 1)
    # 40 shards of ~6 documents: k = 16 exceeds every shard (padding path), k_out = 16
    ids, sc = _sharded(msa, mp, bank, qr, qso, 16, 40)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    check_topk(ids, sc, o_ids, o_sc, o_all)
