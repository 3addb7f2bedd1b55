"""GPU parity of msa_attend's routed form: the call takes the route's top-k
document ids and the bank's chunk offsets and lists the memory rows itself.

Every attention kernel must give exactly what it gives on the gather listing of
the same documents (same rows in the same order: bit-identical outputs), and
both must match the CPU oracle run on the listing that oracle.gather writes.
Covers the decoding kernel's in-kernel listing (top_k <= 256) and the listing
into the workspace (the other kernels, and top_k > 256), documents with no
chunks, ids outside the bank (they list nothing), and max_sel below a
sequence's row count (the call stays inside its buffers)."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_common import DevBank, bits, check_topk, from_bits, host_normal, route_gpu

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def msa():
    import routed_sparse_attention_msa_b200 as m
    return m


@pytest.fixture(params=["split", "tc", "tc_dec", "dec", "dec_rope", "dec_bulk"])
def attend_kernel(request, msa):
    """dec: the decoding kernel rotating its local keys itself; dec_rope: the
    same kernel after the separate rotation kernel; dec_bulk: the decoding
    kernel moving its rows by bulk copies."""
    old = msa.set_attend_kernel(request.param.split("_")[0] if request.param.startswith("dec") else request.param)
    old_r = msa.set_dec_rot_keys(0 if request.param == "dec_rope" else 256)
    old_b = msa.set_dec_bulk(request.param == "dec_bulk")
    yield request.param
    msa.set_dec_bulk(old_b)
    msa.set_dec_rot_keys(old_r)
    msa.set_attend_kernel(old)


def _docs(n_docs, seed):
    """Chunk counts of a bank: ragged, every 7th document empty."""
    rng = np.random.default_rng(seed)
    cnt = rng.integers(1, 9, n_docs)
    cnt[::7] = 0
    return np.concatenate([[0], np.cumsum(cnt)]).astype(np.int64)


def _case(rows, n_loc, q_start, k, n_docs=400, bad=False, hq=32, hkv=8, layer=90):
    dco = _docs(n_docs, layer)
    C = int(dco[-1])
    S, T, L = len(rows), sum(rows), sum(n_loc)
    rng = np.random.default_rng(layer + 1)
    top = np.stack([rng.choice(n_docs, k, replace=False) for _ in range(S)]).astype(np.int32)
    if bad:  # ids outside the bank list nothing
        top[0, 1] = -1
        top[-1, k - 1] = n_docs
        top[-1, 0] = np.iinfo(np.int32).max
    # the expected listing: the valid ids' chunk ranges in rank order (oracle.gather per sequence)
    offs, chunks = [0], []
    for s in range(S):
        ids = top[s][(top[s] >= 0) & (top[s] < n_docs)]
        _, sel = oracle.gather(ids[None, :], dco) if ids.size else (None, np.zeros(0, np.int64))
        chunks.append(sel)
        offs.append(offs[-1] + sel.size)
    return dict(q=host_normal((T, hq, 128), synth.tid("q_att", layer)),
                q_seq_off=np.concatenate([[0], np.cumsum(rows)]).astype(np.int32),
                q_start=np.array(q_start, np.int32),
                k_loc=host_normal((max(L, 1), hkv, 128), synth.tid("k_loc", layer)),
                v_loc=host_normal((max(L, 1), hkv, 128), synth.tid("v_loc", layer)),
                loc_off=np.concatenate([[0], np.cumsum(n_loc)]).astype(np.int32),
                mem_k=host_normal((max(C, 1), hkv, 128), synth.tid("kbar", layer)),
                mem_v=host_normal((max(C, 1), hkv, 128), synth.tid("vbar", layer)),
                sel_off=np.array(offs, np.int64), sel_chunk=np.concatenate(chunks).astype(np.int64),
                top=top, dco=dco, max_sel=k * 8)


def _run(msa, c, routed, max_sel=None, pos_offset=16.0):
    T, hq = c["q"].shape[:2]
    max_sel = c["max_sel"] if max_sel is None else max_sel
    if routed:
        sel_off = sel = None
        r = (torch.from_numpy(c["top"]).cuda(), torch.from_numpy(c["dco"]).cuda())
    else:
        sel_off = torch.from_numpy(c["sel_off"]).cuda()
        sel = torch.from_numpy(c["sel_chunk"] if c["sel_chunk"].size else np.zeros(1, np.int64)).cuda()
        r = None
    args = (from_bits(c["q"]), c["q_seq_off"], c["q_start"], from_bits(c["k_loc"]), from_bits(c["v_loc"]),
            c["loc_off"], from_bits(c["mem_k"]), from_bits(c["mem_v"]), sel_off, sel, max_sel)
    out = torch.empty((T, hq, 128), dtype=torch.bfloat16, device="cuda")
    of = torch.empty((T, hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, hq), dtype=torch.float32, device="cuda")
    ws = torch.empty(msa.attend_workspace(*args, pos_offset=pos_offset, routed=r), dtype=torch.uint8, device="cuda")
    msa.attend(*args, out, ws, out_f32=of, lse=lse, pos_offset=pos_offset, routed=r)
    msa.sync_check()
    return bits(out), of.cpu().numpy(), lse.cpu().numpy()


def _oracle(c, pos_offset=16.0):
    keys = ("q", "q_seq_off", "q_start", "k_loc", "v_loc", "loc_off", "mem_k", "mem_v", "sel_off", "sel_chunk")
    return oracle.attend(**{k: c[k] for k in keys}, pos_offset=pos_offset)


CASES = {
    "decode": dict(rows=(1, 1, 2), n_loc=(129, 1, 9), q_start=(128, 0, 7), k=16),
    "decode_one_seq": dict(rows=(1,), n_loc=(192,), q_start=(191,), k=16),
    "decode_bad_ids": dict(rows=(1, 1), n_loc=(40, 3), q_start=(39, 2), k=16, bad=True),
    "decode_k300": dict(rows=(1, 2), n_loc=(20, 30), q_start=(19, 28), k=300, n_docs=700),
    "prefill": dict(rows=(64, 9), n_loc=(64, 20), q_start=(0, 11), k=16),
}


@pytest.mark.parametrize("name", list(CASES))
def test_attend_routed_equals_gather_listing(msa, attend_kernel, name):
    c = _case(**CASES[name])
    listed = _run(msa, c, routed=False)
    routed = _run(msa, c, routed=True)
    for a, b in zip(listed, routed):
        np.testing.assert_array_equal(a, b)
    o_out, o_lse = _oracle(c)
    assert np.abs(routed[1] - o_out).max() <= 1e-2
    np.testing.assert_array_equal(routed[0], synth.bf16_bits(routed[1]))
    np.testing.assert_allclose(routed[2], o_lse, atol=1e-3, rtol=0)


@pytest.mark.parametrize("splits", [1, 2, 3, 8])
def test_attend_routed_decoding_splits(msa, splits):
    """The decoding kernel's cluster merge with 1 to 8 splits, on its in-kernel listing."""
    old_k, old_s = msa.set_attend_kernel("dec"), msa.set_attend_splits(splits)
    try:
        c = _case(rows=(1, 1, 1), n_loc=(65, 1, 200), q_start=(64, 0, 199), k=24, layer=91)
        out = _run(msa, c, routed=True)
    finally:
        msa.set_attend_splits(old_s)
        msa.set_attend_kernel(old_k)
    o_out, o_lse = _oracle(c)
    assert np.abs(out[1] - o_out).max() <= 1e-2
    np.testing.assert_allclose(out[2], o_lse, atol=1e-3, rtol=0)


def test_attend_routed_max_sel_below_the_rows(msa, attend_kernel):
    """max_sel smaller than a sequence's rows: the result is unspecified by the
    interface, but the call must stay inside its buffers. With one sequence
    every kernel keeps the first max_sel rows."""
    c = _case(rows=(1,), n_loc=(30,), q_start=(29,), k=16, layer=92)
    n = int(c["sel_off"][1])
    cut = n // 3
    got = _run(msa, c, routed=True, max_sel=cut)
    t = dict(c, sel_off=np.array([0, cut], np.int64), sel_chunk=c["sel_chunk"][:cut])
    o_out, o_lse = _oracle(t)
    assert np.abs(got[1] - o_out).max() <= 1e-2
    np.testing.assert_allclose(got[2], o_lse, atol=1e-3, rtol=0)


def test_tiny_step_route_then_routed_attend(msa):
    """Route -> attend (routed form, no msa_gather) on the tiny workload, against the oracle chain."""
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, 0, content=True)
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, [32], 16, 3, 8, 128, 0)
    ids, sc, _ = route_gpu(bank, qr, qso, 16, want_all=False)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    np.testing.assert_array_equal(ids, o_ids)
    o_off, o_sel = oracle.gather(o_ids, bank.dco)
    kh, vh = bank.host_content()
    T = 32
    q = host_normal((T, 32, 128), synth.tid("q_att", 0))
    kl = host_normal((T, 8, 128), synth.tid("k_loc", 0))
    vl = host_normal((T, 8, 128), synth.tid("v_loc", 0))
    out = torch.empty((T, 32, 128), dtype=torch.bfloat16, device="cuda")
    of = torch.empty((T, 32, 128), dtype=torch.float32, device="cuda")
    r = (torch.from_numpy(ids).cuda(), bank.layer_c.doc_chunk_off)
    args = (from_bits(q), [0, T], [0], from_bits(kl), from_bits(vl), [0, T], bank.kbar, bank.vbar, None, None,
            16 * bank.layer_c.max_doc_chunks)
    ws = torch.empty(msa.attend_workspace(*args, routed=r), dtype=torch.uint8, device="cuda")
    msa.attend(*args, out, ws, out_f32=of, pos_offset=16.0, routed=r)
    msa.sync_check()
    o_out, _ = oracle.attend(q, [0, T], [0], kl, vl, [0, T], kh, vh, o_off, o_sel, pos_offset=16.0)
    assert np.abs(of.cpu().numpy() - o_out).max() <= 1e-2


def test_more_than_256_sequences(msa):
    """300 sequences: the route and the attention run as two groups (256 + 44)
    on one stream and one workspace each; the top-k against the oracle, the
    gather listing for all 300 sequences, and the attention (routed form, one
    decoding row per sequence after 5 local keys) against the oracle chain."""
    S, L = 300, 5
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, 3, content=True)
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, [1] * S, 16, 1, 8, 128, 3)
    ids, sc, alls = route_gpu(bank, qr, qso, 16)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    check_topk(ids, sc, o_ids, o_sc, o_all)
    finite = np.isfinite(o_all)
    np.testing.assert_allclose(alls[finite], o_all[finite], atol=1e-3, rtol=0)
    top_d = torch.from_numpy(ids).cuda()
    # the gather listing of all 300 sequences
    cap = S * 16 * bank.layer_c.max_doc_chunks
    sel_off = torch.empty(S + 1, dtype=torch.int64, device="cuda")
    sel = torch.empty(cap, dtype=torch.int64, device="cuda")
    msa.gather(bank.layer_c, top_d, 16, sel_off, sel)
    msa.sync_check()
    o_off, o_sel = oracle.gather(ids, bank.dco)
    np.testing.assert_array_equal(sel_off.cpu().numpy(), o_off)
    np.testing.assert_array_equal(sel.cpu().numpy()[:o_off[-1]], o_sel)
    # the attention in the routed form
    q = host_normal((S, 32, 128), synth.tid("q_att", 3))
    kl = host_normal((S * L, 8, 128), synth.tid("k_loc", 3))
    vl = host_normal((S * L, 8, 128), synth.tid("v_loc", 3))
    qs, qst, lo = np.arange(S + 1), np.full(S, L - 1), np.arange(S + 1) * L
    r = (top_d, bank.layer_c.doc_chunk_off)
    args = (from_bits(q), qs, qst, from_bits(kl), from_bits(vl), lo, bank.kbar, bank.vbar, None, None,
            16 * bank.layer_c.max_doc_chunks)
    out = torch.empty((S, 32, 128), dtype=torch.bfloat16, device="cuda")
    of = torch.empty((S, 32, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((S, 32), dtype=torch.float32, device="cuda")
    ws = torch.empty(msa.attend_workspace(*args, routed=r), dtype=torch.uint8, device="cuda")
    msa.attend(*args, out, ws, out_f32=of, lse=lse, pos_offset=16.0, routed=r)
    msa.sync_check()
    kh, vh = bank.host_content()
    o_out, o_lse = oracle.attend(q, qs, qst, kl, vl, lo, kh, vh, o_off, o_sel, pos_offset=16.0)
    assert np.abs(of.cpu().numpy() - o_out).max() <= 1e-2
    np.testing.assert_allclose(lse.cpu().numpy(), o_lse, atol=1e-3, rtol=0)
