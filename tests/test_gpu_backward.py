"""GPU gradients (attention and routing score) against the oracle's fp64
gradients, which are pinned by finite differences."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_common import DevBank, from_bits, host_normal, route_gpu
from tests.test_gpu_kernels import _attend_case

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def _close(got, want, rel=1e-3):
    """max |got - want| within rel of the largest reference magnitude (fp32
    accumulation against fp64: observed errors are ~1e-6 relative)."""
    scale = max(float(np.abs(want).max()), 1e-12)
    err = float(np.abs(got - want).max())
    assert err <= rel * scale, (err, scale)


@pytest.mark.parametrize("case", [
    dict(rows=(3, 1), n_loc=(5, 2), n_mem=(40, 17), q_start=(2, 1)),
    dict(rows=(1,), n_loc=(129,), n_mem=(300,), q_start=(128,)),
    dict(rows=(1, 1, 1), n_loc=(65, 1, 7), n_mem=(0, 100, 61), q_start=(64, 0, 6)),
    dict(rows=(20,), n_loc=(12,), n_mem=(33,), q_start=(0,)),  # rows beyond the local keys; unseen local keys
])
def test_attend_backward_matches_oracle(case):
    import routed_sparse_attention_msa_b200 as msa
    c = _attend_case(**case, layer=30)
    pos, theta = 16.0, 1e4
    T, hq = c["q"].shape[:2]
    L, hkv = c["k_loc"].shape[:2]
    n_sel = int(c["sel_off"][-1])
    q, kl, vl = from_bits(c["q"]), from_bits(c["k_loc"]), from_bits(c["v_loc"])
    mk, mv = from_bits(c["mem_k"]), from_bits(c["mem_v"])
    sel = torch.from_numpy(c["sel_chunk"] if c["sel_chunk"].size else np.zeros(1, np.int64)).cuda()
    sel_off = torch.from_numpy(c["sel_off"]).cuda()
    max_sel = int(np.diff(c["sel_off"]).max())
    out = torch.empty((T, hq, 128), dtype=torch.bfloat16, device="cuda")
    of = torch.empty((T, hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, hq), dtype=torch.float32, device="cuda")
    args = (q, c["q_seq_off"], c["q_start"], kl, vl, c["loc_off"], mk, mv, sel_off, sel, max_sel)
    ws = torch.empty(msa.attend_workspace(*args, pos_offset=pos, rope_theta=theta), dtype=torch.uint8, device="cuda")
    msa.attend(*args, out, ws, out_f32=of, lse=lse, pos_offset=pos, rope_theta=theta)
    dout_np = host_normal((T, hq, 128), synth.tid("q_att", 31)).astype(np.uint16)
    W = oracle.bf16_to_f64(dout_np)
    dout = torch.from_numpy(W.astype(np.float32)).cuda()
    dq = torch.full((T, hq, 128), float("nan"), device="cuda")
    dkl = torch.full((L, hkv, 128), float("nan"), device="cuda")
    dvl = torch.full((L, hkv, 128), float("nan"), device="cuda")
    dmk = torch.full((max(n_sel, 1), hkv, 128), float("nan"), device="cuda")
    dmv = torch.full((max(n_sel, 1), hkv, 128), float("nan"), device="cuda")
    wsb = torch.empty(msa.attend_backward_workspace(*args, of, lse, pos_offset=pos, rope_theta=theta),
                      dtype=torch.uint8, device="cuda")
    msa.attend_backward(*args, of, lse, dout, dq, dkl, dvl, dmk, dmv, wsb, pos_offset=pos, rope_theta=theta)
    msa.sync_check()
    _, _, o_dq, o_dkl, o_dvl, o_dmk, o_dmv = oracle.attend_f64(**c, pos_offset=pos, rope_theta=theta, dout=W)
    _close(dq.cpu().numpy(), o_dq)
    _close(dkl.cpu().numpy(), o_dkl)
    _close(dvl.cpu().numpy(), o_dvl)
    if n_sel:
        _close(dmk.cpu().numpy()[:n_sel], o_dmk)
        _close(dmv.cpu().numpy()[:n_sel], o_dmv)


@pytest.mark.parametrize("rows", [[32], [1, 16, 3], [1] * 4])
def test_route_backward_matches_oracle(rows):
    import routed_sparse_attention_msa_b200 as msa
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, 2, content=False)
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, rows, 8, 1, 8, 128, 2, call=3)
    # triples: every planted document of every sequence, with random dL/dscore
    ps = np.concatenate([[s] * len(plan.docs[s]) for s in range(len(rows))]).astype(np.int32)
    pd = np.concatenate([plan.docs[s] for s in range(len(rows))]).astype(np.int32)
    pg = np.linspace(-1.5, 1.2, ps.size)
    T = sum(rows)
    dqr = torch.zeros((T, 8, 128), dtype=torch.float32, device="cuda")
    dkr = torch.empty((ps.size, 8, 128), dtype=torch.float32, device="cuda")
    ac = torch.empty(ps.size, dtype=torch.int64, device="cuda")
    ar = torch.empty(ps.size, dtype=torch.int32, device="cuda")
    msa.route_backward(bank.layer_c, from_bits(qr), qso, torch.from_numpy(ps).cuda(), torch.from_numpy(pd).cuda(),
                       torch.from_numpy(pg.astype(np.float32)).cuda(), dqr, dkr, ac, ar)
    msa.sync_check()
    o_dq, o_dk, o_ac, o_ar = oracle.route_backward(bank.host_kbar_r(), bank.dco, qr, qso, ps, pd, pg)
    np.testing.assert_array_equal(ac.cpu().numpy(), o_ac)
    np.testing.assert_array_equal(ar.cpu().numpy(), o_ar)
    _close(dqr.cpu().numpy(), o_dq)
    _close(dkr.cpu().numpy(), o_dk)
