"""Memory Parallel routing across ranks: two processes, each owning one
document shard of the bank, route their shard, all-gather the candidates
(gloo, through host copies) and merge them with the top-k merge kernel. Both
ranks must end with ids and scores bit-identical to routing the unsharded
bank, and agree with the oracle.

The two processes share the one GPU; no kernel waits on the other process
(the only exchange is the host-side all-gather)."""
import datetime
import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, workload, rows, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import routed_sparse_attention_msa_b200 as msa
    from routed_sparse_attention_msa_b200 import memory_parallel as mp
    import synth
    from tests.gpu_common import DevBank, from_bits, route_gpu

    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        w = synth.workload(workload)
        bank = DevBank(w.doc_tok_off, 2, content=False)  # every rank regenerates the same bank
        qr_bits, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, rows, w.top_k,
                                                        w.n_needles, 8, 128, 2)
        ranges = mp.shard_ranges(bank.dco, world)
        d0, d1 = ranges[rank]
        shard = mp.make_shard(bank.layer_c, bank.dco, d0, d1)
        S, k = len(rows), w.top_k
        qr = from_bits(qr_bits)
        ws = torch.empty(max(msa.route_workspace(shard.layer, S, qr.shape[0], k), 256), dtype=torch.uint8,
                         device="cuda")
        ids = torch.empty((S, k), dtype=torch.int32, device="cuda")
        sc = torch.empty((S, k), dtype=torch.float32, device="cuda")
        mp.route_memory_parallel(shard, [a for a, _ in ranges], qr, qso, k, ids, sc, ws)
        msa.sync_check()
        full_ids, full_sc, _ = route_gpu(bank, qr_bits, qso, k, want_all=False)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), ids=ids.cpu().numpy(), sc=sc.cpu().numpy(),
                 full_ids=full_ids, full_sc=full_sc, qr=qr_bits, qso=np.asarray(qso), dco=bank.dco,
                 planted=np.asarray(plan.docs))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("workload,rows", [("tiny", [32]), ("10m", [1] * 16)])
def test_memory_parallel_two_ranks(tmp_path, workload, rows):
    import torch.multiprocessing as tmp
    import oracle
    from tests.gpu_common import DevBank
    import synth

    world, port = 2, _free_port()
    ctx = tmp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, workload, rows, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=600)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0, p.exitcode
    r0, r1 = (np.load(tmp_path / f"rank{r}.npz") for r in range(world))
    for r in (r0, r1):
        np.testing.assert_array_equal(r["ids"], r0["full_ids"])  # bit-identical to the unsharded route
        np.testing.assert_array_equal(r["sc"], r0["full_sc"])
    for s in range(len(rows)):
        assert set(r0["ids"][s].tolist()) == set(r0["planted"][s].tolist())
    # and the oracle agrees (ids exact where the planted gap makes the set unique, scores within 1e-3)
    w = synth.workload(workload)
    kr = synth.normal_bf16_host(int(r0["dco"][-1]) * 8 * 128, synth.tid("kbar_r", 2)).reshape(-1, 8, 128)
    o_ids, o_sc, _ = oracle.route(kr, r0["dco"], r0["qr"], r0["qso"], w.top_k)
    np.testing.assert_array_equal(np.sort(r0["ids"], axis=1), np.sort(o_ids, axis=1))
    np.testing.assert_allclose(r0["sc"], o_sc, atol=1e-3, rtol=0)
