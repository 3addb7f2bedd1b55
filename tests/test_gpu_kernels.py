"""GPU parity: every kernel of the path, called through the C ABI, against the
CPU oracle on the same seeded inputs (small and ragged sizes spanning several
tiles, with partial tails and degenerate cases)."""
import math

import numpy as np
import pytest

import oracle
import synth
from tests.gpu_common import (DevBank, bf16_ulp, bits, check_topk, dev_normal, from_bits, gap_at_k,
                              host_normal, route_gpu)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def msa():
    import routed_sparse_attention_msa_b200 as m
    return m


@pytest.fixture(params=["simt", "tc", "tc_rows"])
def score_kernel(request, msa):
    if request.param != "simt" and not msa.tc_available():
        pytest.skip("tensor-core scoring kernel not compiled in")
    old = msa.set_score_kernel(request.param)
    yield request.param
    msa.set_score_kernel(old)


# ------------------------------------------------------------- generator

def test_device_generator_matches_host():
    n = (1 << 20) + 77
    t = dev_normal((n,), synth.tid("kbar_r", 5))
    np.testing.assert_array_equal(bits(t), host_normal((n,), synth.tid("kbar_r", 5)))
    t = dev_normal((1000,), synth.tid("kbar", 2), sigma=0.5, index0=123456789)
    np.testing.assert_array_equal(bits(t), host_normal((1000,), synth.tid("kbar", 2), 0.5, 123456789))


def bf16_of(x):
    return synth.bf16_bits(np.asarray(x, np.float64))


# ---------------------------------------------------------------- encode

ENC_LENS = [64, 1, 63, 65, 0, 129, 300, 4096 + 17, 640, 2]


@pytest.mark.parametrize("theta,rope_mode", [(1e6, 0), (1e4, 0), (1e4, 1)])
def test_encode_matches_oracle(msa, theta, rope_mode):
    off = np.concatenate([[0], np.cumsum(ENC_LENS)]).astype(np.int64)
    n = int(off[-1])
    shp = (n, 8, 128)
    k = dev_normal(shp, synth.tid("k_tok", 1))
    v = dev_normal(shp, synth.tid("v_tok", 1))
    r = dev_normal(shp, synth.tid("kr_tok", 1))
    C, dco_h, mx = msa.encode_plan(off, 64)
    out = dict(kbar=torch.empty((C, 8, 128), dtype=torch.bfloat16, device="cuda"),
               vbar=torch.empty((C, 8, 128), dtype=torch.bfloat16, device="cuda"),
               kbar_r=torch.empty((C, 8, 128), dtype=torch.bfloat16, device="cuda"),
               kr_inv_norm=torch.empty((C, 8), dtype=torch.float32, device="cuda"),
               doc_chunk_off=torch.empty(len(ENC_LENS) + 1, dtype=torch.int64, device="cuda"),
               chunk_doc=torch.empty(C, dtype=torch.int32, device="cuda"))
    msa.encode(k, v, r, torch.from_numpy(off).cuda(), C, out, rope_theta=theta, rope_mode=rope_mode)
    msa.sync_check()
    ref = oracle.encode(host_normal(shp, synth.tid("k_tok", 1)), host_normal(shp, synth.tid("v_tok", 1)),
                        host_normal(shp, synth.tid("kr_tok", 1)), off, rope_theta=theta, rope_mode=rope_mode)
    np.testing.assert_array_equal(out["doc_chunk_off"].cpu().numpy(), ref["doc_chunk_off"])
    np.testing.assert_array_equal(out["doc_chunk_off"].cpu().numpy(), dco_h)
    np.testing.assert_array_equal(out["chunk_doc"].cpu().numpy(), ref["chunk_doc"])
    for name in ["kbar", "vbar", "kbar_r"]:
        g = oracle.bf16_to_f64(bits(out[name]))
        o = oracle.bf16_to_f64(ref[name])
        err = np.abs(g - o)
        # one bfloat16 ulp of the final rounding, plus the fp32 accumulation
        # error of a mean of <= 64 terms of size O(1) (<= 64 * 2^-24 * 4)
        tol = bf16_ulp(o) + 2e-5
        worst = int(np.argmax(err - tol))
        assert np.all(err <= tol), (name, float(err.max()), float(o.ravel()[worst]), float(g.ravel()[worst]))
        exact = float(np.mean(g == o))
        assert exact > 0.99, (name, exact)
    np.testing.assert_allclose(out["kr_inv_norm"].cpu().numpy(), ref["kr_inv_norm"], rtol=2e-4)


def test_bank_norms_match_oracle(msa):
    off = np.array([0, 640, 700, 2000], np.int64)
    shp = (2000, 8, 128)
    kr = host_normal(shp, synth.tid("kr_tok", 9))
    ref = oracle.encode(host_normal(shp, synth.tid("k_tok", 9)), host_normal(shp, synth.tid("v_tok", 9)), kr, off)
    kb = from_bits(ref["kbar_r"])
    inv = torch.empty((kb.shape[0], 8), dtype=torch.float32, device="cuda")
    msa.bank_norms(kb, inv)
    msa.sync_check()
    np.testing.assert_allclose(inv.cpu().numpy(), ref["kr_inv_norm"], rtol=1e-5)
    # zero routing key: the norm clamp gives 1 / eps
    z = torch.zeros((3, 8, 128), dtype=torch.bfloat16, device="cuda")
    inv = torch.empty((3, 8), dtype=torch.float32, device="cuda")
    msa.bank_norms(z, inv, eps=1e-6)
    msa.sync_check()
    np.testing.assert_allclose(inv.cpu().numpy(), 1e6, rtol=1e-6)


@pytest.mark.parametrize("chunk", [16, 128])
def test_encode_other_chunk_lengths(msa, chunk):
    """The chunk length is an argument: 16 and 128 against the oracle."""
    lens = [chunk, 1, chunk - 1, chunk + 1, 0, 3 * chunk + 5]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(off[-1])
    shp = (n, 8, 128)
    k = dev_normal(shp, synth.tid("k_tok", 3))
    v = dev_normal(shp, synth.tid("v_tok", 3))
    r = dev_normal(shp, synth.tid("kr_tok", 3))
    C, dco_h, mx = msa.encode_plan(off, chunk)
    out = dict(kbar=torch.empty((C, 8, 128), dtype=torch.bfloat16, device="cuda"),
               vbar=torch.empty((C, 8, 128), dtype=torch.bfloat16, device="cuda"),
               kbar_r=torch.empty((C, 8, 128), dtype=torch.bfloat16, device="cuda"),
               kr_inv_norm=torch.empty((C, 8), dtype=torch.float32, device="cuda"),
               doc_chunk_off=torch.empty(len(lens) + 1, dtype=torch.int64, device="cuda"),
               chunk_doc=torch.empty(C, dtype=torch.int32, device="cuda"))
    msa.encode(k, v, r, torch.from_numpy(off).cuda(), C, out, chunk=chunk)
    msa.sync_check()
    ref = oracle.encode(host_normal(shp, synth.tid("k_tok", 3)), host_normal(shp, synth.tid("v_tok", 3)),
                        host_normal(shp, synth.tid("kr_tok", 3)), off, chunk=chunk)
    np.testing.assert_array_equal(out["doc_chunk_off"].cpu().numpy(), ref["doc_chunk_off"])
    np.testing.assert_array_equal(out["chunk_doc"].cpu().numpy(), ref["chunk_doc"])
    for name in ["kbar", "vbar", "kbar_r"]:
        g = oracle.bf16_to_f64(bits(out[name]))
        o = oracle.bf16_to_f64(ref[name])
        # one bfloat16 ulp plus the fp32 accumulation error of a mean of <= chunk O(1) terms
        tol = bf16_ulp(o) + chunk * 2.0 ** -24 * 4 + 1e-5
        assert np.all(np.abs(g - o) <= tol), (name, float(np.abs(g - o).max()))
        assert float(np.mean(g == o)) > 0.98, name
    np.testing.assert_allclose(out["kr_inv_norm"].cpu().numpy(), ref["kr_inv_norm"], rtol=2e-4)


# ----------------------------------------------------------------- route

def _tiny_bank_and_queries(layer=0, rows=32, call=0, n_needles=3, k=16):
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, layer, content=False)
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, [rows], k, n_needles, 8, 128,
                                               layer, call)
    return bank, qr, qso, plan


def test_route_tiny_matches_oracle(msa, score_kernel):
    bank, qr, qso, plan = _tiny_bank_and_queries()
    ids, sc, alls = route_gpu(bank, qr, qso, 16)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    assert gap_at_k(o_all[0], 16) >= 1e-2
    assert check_topk(ids, sc, o_ids, o_sc, o_all) == 1
    np.testing.assert_array_equal(ids, o_ids)
    np.testing.assert_allclose(alls, o_all, atol=1e-3, rtol=0)
    assert set(ids[0, :3].tolist()) == set(plan.docs[0][:3])


def _ragged_offsets(seed_stream, n_docs=700):
    u = synth.uniform01(n_docs, synth.tid("doc_len", extra=seed_stream))
    lens = (np.exp(3.5 + 2.2 * u) * (u > 0.03)).astype(np.int64)  # ~3% empty documents
    lens[5] = 0
    lens[-1] = 0
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


@pytest.mark.parametrize("rows,k", [((1,), 16), ((1, 5, 2), 7), ((3, 1, 17, 1, 40), 16), ((2, 2), 40)])
def test_route_ragged_matches_oracle(msa, score_kernel, rows, k):
    off = _ragged_offsets(11)
    bank = DevBank(off, 3, content=False)
    T = sum(rows)
    qso = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    qr = host_normal((T, 8, 128), synth.tid("q_noise", 3, 77))
    qr[min(2, T - 1), 1] = 0  # a zero head in one query row (norm clamp)
    ids, sc, alls = route_gpu(bank, qr, qso, k)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, k)
    check_topk(ids, sc, o_ids, o_sc, o_all)
    finite = np.isfinite(o_all)
    np.testing.assert_allclose(alls[finite], o_all[finite], atol=1e-3, rtol=0)
    assert np.all(np.isneginf(alls[~finite]))


def test_route_planted_multi_sequence(msa, score_kernel):
    # 5 sequences with different row counts, each with 16 planted documents
    off = _ragged_offsets(12, 1500)
    bank = DevBank(off, 4, content=False)
    rows = [1, 16, 40, 3, 2]
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, rows, 16, 1, 8, 128, 4)
    ids, sc, alls = route_gpu(bank, qr, qso, 16)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    n_exact = check_topk(ids, sc, o_ids, o_sc, o_all)
    assert n_exact == len(rows)
    for s in range(len(rows)):
        assert set(ids[s].tolist()) == set(plan.docs[s])


def test_route_k_equals_all_documents(msa, score_kernel):
    bank, qr, qso, plan = _tiny_bank_and_queries(rows=4, k=16)
    ids, sc, alls = route_gpu(bank, qr, qso, 10_000)  # clamps to D = 256 (radix path)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 10_000)
    assert ids.shape == (1, 256)
    assert sorted(ids[0].tolist()) == list(range(256))
    check_topk(ids, sc, o_ids, o_sc, o_all)
    assert np.all(np.diff(sc[0]) <= 0)


@pytest.mark.parametrize("rows", [(65,), (128,), (129,), (256,), (257,), (100, 1, 300, 7, 200), (5,) * 60])
def test_route_many_rows_matches_oracle(msa, score_kernel, rows):
    # row blocks of 128 / 256 with ragged tails; sequences that straddle blocks
    off = _ragged_offsets(14, 500)
    bank = DevBank(off, 5, content=False)
    T = sum(rows)
    qso = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    qr = host_normal((T, 8, 128), synth.tid("q_noise", 5, 91))
    qr[3, 2] = 0  # a zero head (norm clamp)
    ids, sc, alls = route_gpu(bank, qr, qso, 16)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    check_topk(ids, sc, o_ids, o_sc, o_all)
    finite = np.isfinite(o_all)
    np.testing.assert_allclose(alls[finite], o_all[finite], atol=1e-3, rtol=0)
    assert np.all(np.isneginf(alls[~finite]))


@pytest.mark.parametrize("block,pair", [(64, False), (128, False), (160, False), (192, False), (192, True)])
def test_route_many_rows_each_block(msa, block, pair):
    # every row-block variant of the many-row scorer, ragged sequences across blocks
    if not msa.tc_available():
        pytest.skip("tensor-core scoring kernel not compiled in")
    off = _ragged_offsets(16, 400)
    bank = DevBank(off, 7, content=False)
    rows = (100, 1, 300, 7, 200)
    qso = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    qr = host_normal((sum(rows), 8, 128), synth.tid("q_noise", 7, 93))
    old_k, old_b, old_p = msa.set_score_kernel("tc_rows"), msa.set_pf_block(block), msa.set_pf_pair(pair)
    try:
        ids, sc, alls = route_gpu(bank, qr, qso, 16)
    finally:
        msa.set_score_kernel(old_k)
        msa.set_pf_block(old_b)
        msa.set_pf_pair(old_p)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    check_topk(ids, sc, o_ids, o_sc, o_all)
    finite = np.isfinite(o_all)
    np.testing.assert_allclose(alls[finite], o_all[finite], atol=1e-3, rtol=0)



def test_route_norm_clamp_large_eps(msa, score_kernel):
    """eps = 0.5: each norm is clamped separately, so short vectors score in
    proportion to their length (the oracle's closed-form pin, on the GPU)."""
    hr, d, D = 8, 128, 256
    e = np.zeros((hr, d))
    e[np.arange(hr), 3 * np.arange(hr)] = 1.0
    kbar = np.stack([2.0 * e, 0.25 * e] + [np.roll(e, 1 + j % 2, axis=1) for j in range(D - 2)])
    qr = np.stack([0.25 * e, 2.0 * e])
    kb = bf16_of(kbar)
    eps = 0.5
    o_ids, o_sc, o_ds = oracle.route(kb, np.arange(D + 1), bf16_of(qr), [0, 1, 2], top_k=3, eps=eps)
    kr = from_bits(kb)
    inv = torch.empty((D, hr), dtype=torch.float32, device="cuda")
    msa.bank_norms(kr, inv, eps=eps)
    bank = msa.BankLayer(doc_chunk_off=torch.arange(D + 1, dtype=torch.int64, device="cuda"),
                         chunk_doc=torch.arange(D, dtype=torch.int32, device="cuda"), kbar_r=kr, kr_inv_norm=inv)
    ids = torch.empty((2, 3), dtype=torch.int32, device="cuda")
    sc = torch.empty((2, 3), dtype=torch.float32, device="cuda")
    ads = torch.empty((2, D), dtype=torch.float32, device="cuda")
    ws = torch.zeros(msa.route_workspace(bank, 2, 2, 3), dtype=torch.uint8, device="cuda")
    msa.route(bank, from_bits(bf16_of(qr)), [0, 1, 2], 3, ids, sc, ws, all_doc_scores=ads, eps=eps)
    msa.sync_check()
    np.testing.assert_allclose(ads.cpu().numpy(), o_ds, atol=1e-6)
    np.testing.assert_array_equal(ids.cpu().numpy(), o_ids)
    np.testing.assert_allclose(sc.cpu().numpy()[:, :2], [[0.5, 0.25], [1.0, 0.5]], atol=1e-6)

@pytest.mark.parametrize("n_docs", [900, 1800, 3500, 5000, 12000, 20000, 41000])
def test_route_topk_paths(msa, n_docs):
    # the top-k's single-CTA variant (up to 2,048 documents) and the multi-CTA merge (2,048 documents
    # per CTA: 2 to 21 CTAs per sequence)
    off = _ragged_offsets(17 + n_docs, n_docs)
    bank = DevBank(off, 8, content=False)
    rows = (1, 3)
    qso = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    qr = host_normal((sum(rows), 8, 128), synth.tid("q_noise", 8, n_docs))
    ids, sc, alls = route_gpu(bank, qr, qso, 16)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    check_topk(ids, sc, o_ids, o_sc, o_all)
    # the selection is the exact top-16 of the GPU's own scores (ties to the lower id)
    for s_ in range(len(rows)):
        order = np.lexsort((np.arange(alls.shape[1]), -alls[s_].astype(np.float64)))[:16]
        np.testing.assert_array_equal(ids[s_], order)


@pytest.mark.parametrize("n_docs,rows", [(300, (200, 1, 90)), (1000, (192,)), (2500, (64,) * 16)])
def test_route_cta_pair_scorer(msa, n_docs, rows):
    # 192-row blocks on CTA pairs: odd and even tile counts, row blocks with ragged tails, planted sets
    off = _ragged_offsets(31 + n_docs, n_docs)
    bank = DevBank(off, 9, content=False)
    old_k, old_b, old_p = msa.set_score_kernel("tc_rows"), msa.set_pf_block(192), msa.set_pf_pair(True)
    try:
        qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, list(rows), 16, 2, 8, 128, 9)
        ids, sc, alls = route_gpu(bank, qr, qso, 16)
    finally:
        msa.set_score_kernel(old_k)
        msa.set_pf_block(old_b)
        msa.set_pf_pair(old_p)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    assert check_topk(ids, sc, o_ids, o_sc, o_all) == len(rows)
    np.testing.assert_allclose(alls, o_all, atol=1e-3, rtol=0)
    for s_ in range(len(rows)):
        assert set(ids[s_].tolist()) == set(plan.docs[s_])


def test_route_many_rows_planted(msa, score_kernel):
    off = _ragged_offsets(15, 1200)
    bank = DevBank(off, 6, content=False)
    rows = [300, 1, 200, 90]
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, rows, 16, 2, 8, 128, 6)
    ids, sc, alls = route_gpu(bank, qr, qso, 16)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    assert check_topk(ids, sc, o_ids, o_sc, o_all) == len(rows)
    for s in range(len(rows)):
        assert set(ids[s].tolist()) == set(plan.docs[s])


# ---------------------------------------------------------------- gather

def test_gather_index_matches_oracle(msa):
    off = _ragged_offsets(13, 300)
    bank = DevBank(off, 6, content=True)
    rng = np.random.default_rng(3)
    top = np.stack([rng.choice(bank.n_docs, 9, replace=False) for _ in range(3)]).astype(np.int32)
    top_d = torch.from_numpy(top).cuda()
    cap = 3 * 9 * bank.layer_c.max_doc_chunks
    sel_off = torch.empty(4, dtype=torch.int64, device="cuda")
    sel = torch.full((cap,), -1, dtype=torch.int64, device="cuda")
    msa.gather(bank.layer_c, top_d, 9, sel_off, sel)
    msa.sync_check()
    o_off, o_sel = oracle.gather(top, bank.dco)
    np.testing.assert_array_equal(sel_off.cpu().numpy(), o_off)
    np.testing.assert_array_equal(sel.cpu().numpy()[: o_off[-1]], o_sel)


@pytest.mark.parametrize("mode", [0, 1])
def test_gather_host_tier(msa, mode):
    off = _ragged_offsets(14, 200)
    bank = DevBank(off, 7, content=True, on_host=True)
    top = np.array([[5, 17, 3, 150], [0, 199, 42, 43]], np.int32)  # 5 and 199 are empty documents
    top_d = torch.from_numpy(top).cuda()
    cap = 2 * 4 * bank.layer_c.max_doc_chunks
    sel_off = torch.empty(3, dtype=torch.int64, device="cuda")
    sel = torch.empty((cap,), dtype=torch.int64, device="cuda")
    sk = torch.zeros((cap, 8, 128), dtype=torch.bfloat16, device="cuda")
    sv = torch.zeros((cap, 8, 128), dtype=torch.bfloat16, device="cuda")
    ids_h = torch.empty(8, dtype=torch.int32).pin_memory()
    cs = torch.cuda.Stream()
    ev = torch.cuda.Event()
    msa.gather(bank.layer_c, top_d, 4, sel_off, sel, sk, sv, mode=mode, doc_chunk_off_host=bank.dco,
               top_ids_host=ids_h, copy_stream=cs, done_event=ev)
    msa.sync_check()
    o_off, o_sel = oracle.gather(top, bank.dco)
    kh, vh = bank.host_content()
    n = int(o_off[-1])
    np.testing.assert_array_equal(bits(sk)[:n], kh[o_sel])
    np.testing.assert_array_equal(bits(sv)[:n], vh[o_sel])


# ---------------------------------------------------------------- attend

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


def _attend_case(rows, n_loc, n_mem, q_start, C=3000, hq=32, hkv=8, layer=20):
    T, L = sum(rows), sum(n_loc)
    q = host_normal((T, hq, 128), synth.tid("q_att", layer))
    kl = host_normal((max(L, 1), hkv, 128), synth.tid("k_loc", layer))
    vl = host_normal((max(L, 1), hkv, 128), synth.tid("v_loc", layer))
    mk = host_normal((C, hkv, 128), synth.tid("kbar", layer))
    mv = host_normal((C, hkv, 128), synth.tid("vbar", layer))
    rng = np.random.default_rng(layer)
    sel = np.concatenate([rng.choice(C, m, replace=False) for m in n_mem] + [np.zeros(0)]).astype(np.int64)
    return dict(q=q, q_seq_off=np.concatenate([[0], np.cumsum(rows)]).astype(np.int32),
                q_start=np.array(q_start, np.int32), k_loc=kl, v_loc=vl,
                loc_off=np.concatenate([[0], np.cumsum(n_loc)]).astype(np.int32), mem_k=mk, mem_v=mv,
                sel_off=np.concatenate([[0], np.cumsum(n_mem)]).astype(np.int64), sel_chunk=sel)


def _attend_gpu(msa, c, pos_offset, theta=1e6, identity=False):
    T, hq = c["q"].shape[:2]
    q = from_bits(c["q"])
    kl, vl = from_bits(c["k_loc"]), from_bits(c["v_loc"])
    if identity:  # memory rows already gathered in order (staging buffer)
        mk, mv = from_bits(c["mem_k"][c["sel_chunk"]]), from_bits(c["mem_v"][c["sel_chunk"]])
        sel = None
    else:
        mk, mv = from_bits(c["mem_k"]), from_bits(c["mem_v"])
        sel = torch.from_numpy(c["sel_chunk"] if c["sel_chunk"].size else np.zeros(1, np.int64)).cuda()
    sel_off = torch.from_numpy(c["sel_off"]).cuda()
    max_sel = int(np.diff(c["sel_off"]).max())
    out = torch.empty((T, hq, 128), dtype=torch.bfloat16, device="cuda")
    of = torch.empty((T, hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, hq), dtype=torch.float32, device="cuda")
    args = (q, c["q_seq_off"], c["q_start"], kl, vl, c["loc_off"], mk, mv, sel_off, sel, max_sel)
    ws = torch.empty(msa.attend_workspace(*args, pos_offset=pos_offset, rope_theta=theta), dtype=torch.uint8,
                     device="cuda")
    msa.attend(*args, out, ws, out_f32=of, lse=lse, pos_offset=pos_offset, rope_theta=theta)
    msa.sync_check()
    return bits(out), of.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("case", [
    dict(rows=(3, 1), n_loc=(5, 2), n_mem=(40, 17), q_start=(2, 1)),           # prefill tail + decode row
    dict(rows=(32,), n_loc=(32,), n_mem=(128,), q_start=(0,)),                   # tiny workload shape
    dict(rows=(1,), n_loc=(129,), n_mem=(1500,), q_start=(128,)),                # many keys: split-K
    dict(rows=(1, 1, 1), n_loc=(65, 1, 7), n_mem=(0, 300, 61), q_start=(64, 0, 6)),  # empty memory
    dict(rows=(5,), n_loc=(3,), n_mem=(9,), q_start=(0,)),                       # rows beyond local keys
    dict(rows=(64, 64, 30), n_loc=(64, 64, 30), n_mem=(250, 130, 0), q_start=(0, 0, 0)),  # prefill, 3 sequences
    dict(rows=(48,), n_loc=(80,), n_mem=(100,), q_start=(32,)),                  # prefill after a local prefix
    dict(rows=(100,), n_loc=(100,), n_mem=(77,), q_start=(0,), hq=8, hkv=8),    # no GQA sharing (group 1)
    dict(rows=(40, 9), n_loc=(40, 9), n_mem=(64, 200), q_start=(0, 0), hq=64, hkv=8),  # group 8
    dict(rows=(32,) * 19, n_loc=(32,) * 19, n_mem=(40,) * 19, q_start=(0,) * 19),  # >= 148 CTAs: no key split
])
def test_attend_matches_oracle(msa, attend_kernel, case):
    c = _attend_case(**case)
    pos = 16.0
    g_out, g_f32, g_lse = _attend_gpu(msa, c, pos)
    o_out, o_lse = oracle.attend(**c, pos_offset=pos)
    err = np.abs(g_f32 - o_out).max()
    assert err <= 1e-2, err
    np.testing.assert_array_equal(g_out, synth.bf16_bits(g_f32))  # bf16 out = nearest-even of the fp32 result
    np.testing.assert_allclose(g_lse, o_lse, atol=1e-3, rtol=0)


def test_attend_block_length_offset_reading(msa, attend_kernel):
    """The alternative reading of the query offset: k retrieved documents x the
    chunk length (pos_offset = 16 * 64) instead of k."""
    c = _attend_case(rows=(2, 1), n_loc=(5, 70), n_mem=(48, 90), q_start=(3, 69), layer=22)
    g_out, g_f32, g_lse = _attend_gpu(msa, c, 1024.0)
    o_out, o_lse = oracle.attend(**c, pos_offset=1024.0)
    assert np.abs(g_f32 - o_out).max() <= 1e-2
    np.testing.assert_allclose(g_lse, o_lse, atol=1e-3, rtol=0)


def test_attend_staged_memory_equals_indexed(msa, attend_kernel):
    c = _attend_case(rows=(2, 1), n_loc=(4, 9), n_mem=(33, 70), q_start=(2, 8), layer=21)
    a = _attend_gpu(msa, c, 16.0)
    b = _attend_gpu(msa, c, 16.0, identity=True)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("kernel", ["split", "dec", "dec_rope", "dec_bulk"])
@pytest.mark.parametrize("splits", [1, 2, 5, 64])
def test_attend_forced_splits(msa, kernel, splits):
    """Key splits forced (split-K: 64 is clamped to one split per 32 keys;
    decoding kernel: 64 is clamped to its 8-CTA cluster, with one split a CTA
    walks every key of its sequence): splits that get no keys, one split,
    uneven splits; the decoding kernel rotating its local keys itself or after
    the separate rotation kernel."""
    old_k, old_s = msa.set_attend_kernel(kernel.split("_")[0]), msa.set_attend_splits(splits)
    old_r = msa.set_dec_rot_keys(0 if kernel == "dec_rope" else 256)
    old_b = msa.set_dec_bulk(kernel == "dec_bulk")
    try:
        c = _attend_case(rows=(1, 1, 2), n_loc=(65, 1, 9), n_mem=(0, 300, 61), q_start=(64, 0, 7), layer=23)
        g_out, g_f32, g_lse = _attend_gpu(msa, c, 16.0)
    finally:
        msa.set_dec_bulk(old_b)
        msa.set_dec_rot_keys(old_r)
        msa.set_attend_splits(old_s)
        msa.set_attend_kernel(old_k)
    o_out, o_lse = oracle.attend(**c, pos_offset=16.0)
    assert np.abs(g_f32 - o_out).max() <= 1e-2
    np.testing.assert_array_equal(g_out, synth.bf16_bits(g_f32))
    np.testing.assert_allclose(g_lse, o_lse, atol=1e-3, rtol=0)


@pytest.mark.parametrize("splits", [1, 2, 3, 8])
def test_attend_tc_cluster_splits(msa, splits):
    """The many-row tensor-core attention with its key blocks split over a
    cluster of 1 to 8 CTAs (merged from each other's shared memory): a
    sequence with 9 key blocks, one with 2 (splits beyond its blocks get
    none), prefill rows after a local prefix."""
    old_k, old_s = msa.set_attend_kernel("tc"), msa.set_attend_splits(splits)
    try:
        c = _attend_case(rows=(64, 40), n_loc=(64, 70), n_mem=(500, 60), q_start=(0, 30), layer=24)
        g_out, g_f32, g_lse = _attend_gpu(msa, c, 16.0)
    finally:
        msa.set_attend_splits(old_s)
        msa.set_attend_kernel(old_k)
    o_out, o_lse = oracle.attend(**c, pos_offset=16.0)
    assert np.abs(g_f32 - o_out).max() <= 1e-2
    np.testing.assert_array_equal(g_out, synth.bf16_bits(g_f32))
    np.testing.assert_allclose(g_lse, o_lse, atol=1e-3, rtol=0)


# ------------------------------------------------------- whole step, tiny

def test_tiny_step_route_gather_attend(msa):
    """Route -> gather -> attend on the tiny workload, against the oracle chain."""
    w = synth.workload("tiny")
    bank = DevBank(w.doc_tok_off, 0, content=True)
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, [32], 16, 3, 8, 128, 0)
    ids, sc, _ = route_gpu(bank, qr, qso, 16, want_all=False)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    np.testing.assert_array_equal(ids, o_ids)
    top_d = torch.from_numpy(ids).cuda()
    cap = 16 * bank.layer_c.max_doc_chunks
    sel_off = torch.empty(2, dtype=torch.int64, device="cuda")
    sel = torch.empty(cap, dtype=torch.int64, device="cuda")
    msa.gather(bank.layer_c, top_d, 16, sel_off, sel)
    o_off, o_sel = oracle.gather(o_ids, bank.dco)
    kh, vh = bank.host_content()
    T = 32
    q = host_normal((T, 32, 128), synth.tid("q_att", 0))
    kl = host_normal((T, 8, 128), synth.tid("k_loc", 0))
    vl = host_normal((T, 8, 128), synth.tid("v_loc", 0))
    out = torch.empty((T, 32, 128), dtype=torch.bfloat16, device="cuda")
    of = torch.empty((T, 32, 128), dtype=torch.float32, device="cuda")
    args = (from_bits(q), [0, T], [0], from_bits(kl), from_bits(vl), [0, T], bank.kbar, bank.vbar, sel_off, sel,
            cap)
    ws = torch.empty(msa.attend_workspace(*args), dtype=torch.uint8, device="cuda")
    msa.attend(*args, out, ws, out_f32=of, pos_offset=16.0)
    msa.sync_check()
    o_out, _ = oracle.attend(q, [0, T], [0], kl, vl, [0, T], kh, vh, o_off, o_sel, pos_offset=16.0)
    assert np.abs(of.cpu().numpy() - o_out).max() <= 1e-2
