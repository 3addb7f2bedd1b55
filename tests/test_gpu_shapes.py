"""GPU parity for every head count and chunk length the C ABI accepts, not only
the configs' 8 routing heads / 8 kv heads / 64-token chunks: routing with
hr in {2, 4, ..., 16} (the CUDA-core scorer), encode with other kv and routing
head counts, attention with kv head counts 4 and 16 (GQA groups 1 to 16) on
every attention kernel, the host-tier gather with other row widths. Each
compares with the CPU oracle on the same seeded inputs."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_common import DevBank, bf16_ulp, bits, check_topk, dev_normal, from_bits, host_normal, route_gpu

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def msa():
    import routed_sparse_attention_msa_b200 as m
    return m


def _ragged_offsets(stream, n_docs):
    u = synth.uniform01(n_docs, synth.tid("doc_len", extra=stream))
    lens = (np.exp(3.5 + 2.2 * u) * (u > 0.03)).astype(np.int64)
    lens[3] = 0
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


# ----------------------------------------------------------------- encode

@pytest.mark.parametrize("hkv,hr", [(4, 2), (16, 16), (16, 4), (4, 16), (1, 8)])
def test_encode_head_counts(msa, hkv, hr):
    lens = [64, 1, 63, 65, 0, 300, 129]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(off[-1])
    k = dev_normal((n, hkv, 128), synth.tid("k_tok", 40 + hkv))
    v = dev_normal((n, hkv, 128), synth.tid("v_tok", 40 + hkv))
    r = dev_normal((n, hr, 128), synth.tid("kr_tok", 40 + hr))
    C, _, _ = msa.encode_plan(off, 64)
    out = dict(kbar=torch.empty((C, hkv, 128), dtype=torch.bfloat16, device="cuda"),
               vbar=torch.empty((C, hkv, 128), dtype=torch.bfloat16, device="cuda"),
               kbar_r=torch.empty((C, hr, 128), dtype=torch.bfloat16, device="cuda"),
               kr_inv_norm=torch.empty((C, hr), dtype=torch.float32, device="cuda"),
               doc_chunk_off=torch.empty(len(lens) + 1, dtype=torch.int64, device="cuda"),
               chunk_doc=torch.empty(C, dtype=torch.int32, device="cuda"))
    msa.encode(k, v, r, torch.from_numpy(off).cuda(), C, out, rope_theta=1e4)
    msa.sync_check()
    ref = oracle.encode(host_normal((n, hkv, 128), synth.tid("k_tok", 40 + hkv)),
                        host_normal((n, hkv, 128), synth.tid("v_tok", 40 + hkv)),
                        host_normal((n, hr, 128), synth.tid("kr_tok", 40 + hr)), off, rope_theta=1e4)
    np.testing.assert_array_equal(out["chunk_doc"].cpu().numpy(), ref["chunk_doc"])
    for name in ["kbar", "vbar", "kbar_r"]:
        g = oracle.bf16_to_f64(bits(out[name]))
        o = oracle.bf16_to_f64(ref[name])
        assert g.shape == o.shape
        tol = bf16_ulp(o) + 2e-5  # one bfloat16 ulp + fp32 accumulation of a mean of <= 64 O(1) terms
        assert np.all(np.abs(g - o) <= tol), (name, float(np.abs(g - o).max()))
        assert float(np.mean(g == o)) > 0.98, name
    np.testing.assert_allclose(out["kr_inv_norm"].cpu().numpy(), ref["kr_inv_norm"], rtol=2e-4)


# ------------------------------------------------------------------ route

@pytest.mark.parametrize("hr", [2, 4, 6, 10, 12, 14, 16])
def test_route_head_counts(msa, hr):
    """Routing heads other than 8 run on the CUDA-core scorer: planted sets,
    scores and selection against the oracle, one- and many-row sequences."""
    off = _ragged_offsets(50 + hr, 900)
    bank = DevBank(off, 30 + hr, hr=hr, content=False)
    rows = [1, 5, 70, 2]
    qr, qso, plan = synth.make_routing_queries(bank.host_chunk_kbar_r, bank.dco, rows, 16, 1, hr, 128, 30 + hr)
    ids, sc, alls = route_gpu(bank, qr, qso, 16)
    o_ids, o_sc, o_all = oracle.route(bank.host_kbar_r(), bank.dco, qr, qso, 16)
    check_topk(ids, sc, o_ids, o_sc, o_all)
    finite = np.isfinite(o_all)
    np.testing.assert_allclose(alls[finite], o_all[finite], atol=1e-3, rtol=0)
    assert np.all(np.isneginf(alls[~finite]))


@pytest.mark.parametrize("which", ["tc", "tc_rows"])
def test_route_tensor_core_scorers_refuse_other_head_counts(msa, which):
    """Forcing a tensor-core scorer with hr != 8 is refused before anything is enqueued."""
    off = _ragged_offsets(70, 50)
    bank = DevBank(off, 70, hr=4, content=False)
    qr = from_bits(host_normal((2, 4, 128), synth.tid("q_noise", 70)))
    ids = torch.empty((1, 4), dtype=torch.int32, device="cuda")
    sc = torch.empty((1, 4), dtype=torch.float32, device="cuda")
    ws = torch.empty(msa.route_workspace(bank.layer_c, 1, 2, 4), dtype=torch.uint8, device="cuda")
    old = msa.set_score_kernel(which)
    try:
        with pytest.raises(msa.MsaError) as ei:
            msa.route(bank.layer_c, qr, [0, 2], 4, ids, sc, ws)
    finally:
        msa.set_score_kernel(old)
    assert ei.value.code == 3  # MSA_ERR_UNSUPPORTED
    msa.sync_check()


# ----------------------------------------------------------------- gather

@pytest.mark.parametrize("hkv", [4, 16])
def test_gather_host_tier_head_counts(msa, hkv):
    off = _ragged_offsets(80 + hkv, 120)
    bank = DevBank(off, 80 + hkv, hkv=hkv, content=True, on_host=True)
    top = np.array([[7, 3, 100], [3, 0, 119]], np.int32)
    top_d = torch.from_numpy(top).cuda()
    cap = 2 * 3 * bank.layer_c.max_doc_chunks
    sel_off = torch.empty(3, dtype=torch.int64, device="cuda")
    sel = torch.empty((cap,), dtype=torch.int64, device="cuda")
    sk = torch.zeros((cap, hkv, 128), dtype=torch.bfloat16, device="cuda")
    sv = torch.zeros((cap, hkv, 128), dtype=torch.bfloat16, device="cuda")
    msa.gather(bank.layer_c, top_d, 3, sel_off, sel, sk, sv, mode=msa.GATHER_DEVICE_PULL)
    msa.sync_check()
    o_off, o_sel = oracle.gather(top, bank.dco)
    kh, vh = bank.host_content()
    n = int(o_off[-1])
    np.testing.assert_array_equal(sel_off.cpu().numpy(), o_off)
    np.testing.assert_array_equal(bits(sk)[:n], kh[o_sel])
    np.testing.assert_array_equal(bits(sv)[:n], vh[o_sel])


# ----------------------------------------------------------------- attend

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


def _attend_case(rows, n_loc, n_mem, q_start, hq, hkv, layer, C=2000):
    T, L = sum(rows), sum(n_loc)
    rng = np.random.default_rng(layer)
    sel = np.concatenate([rng.choice(C, m, replace=False) for m in n_mem] + [np.zeros(0)]).astype(np.int64)
    return dict(q=host_normal((T, hq, 128), synth.tid("q_att", layer)),
                q_seq_off=np.concatenate([[0], np.cumsum(rows)]).astype(np.int32),
                q_start=np.array(q_start, np.int32),
                k_loc=host_normal((max(L, 1), hkv, 128), synth.tid("k_loc", layer)),
                v_loc=host_normal((max(L, 1), hkv, 128), synth.tid("v_loc", layer)),
                loc_off=np.concatenate([[0], np.cumsum(n_loc)]).astype(np.int32),
                mem_k=host_normal((C, hkv, 128), synth.tid("kbar", layer)),
                mem_v=host_normal((C, hkv, 128), synth.tid("vbar", layer)),
                sel_off=np.concatenate([[0], np.cumsum(n_mem)]).astype(np.int64), sel_chunk=sel)


@pytest.mark.parametrize("hq,hkv", [(16, 4), (32, 16), (64, 16), (16, 16), (8, 4), (64, 4)])
@pytest.mark.parametrize("shape", ["decode", "prefill"])
def test_attend_head_counts(msa, attend_kernel, hq, hkv, shape):
    if shape == "decode":
        case = dict(rows=(1, 1, 2), n_loc=(129, 1, 9), n_mem=(300, 0, 61), q_start=(128, 0, 7))
    else:
        case = dict(rows=(64, 9), n_loc=(64, 20), n_mem=(130, 40), q_start=(0, 11))
    c = _attend_case(**case, hq=hq, hkv=hkv, layer=60 + hq + hkv)
    T = c["q"].shape[0]
    sel_off = torch.from_numpy(c["sel_off"]).cuda()
    sel = torch.from_numpy(c["sel_chunk"] if c["sel_chunk"].size else np.zeros(1, np.int64)).cuda()
    out = torch.empty((T, hq, 128), dtype=torch.bfloat16, device="cuda")
    of = torch.empty((T, hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((T, hq), dtype=torch.float32, device="cuda")
    args = (from_bits(c["q"]), c["q_seq_off"], c["q_start"], from_bits(c["k_loc"]), from_bits(c["v_loc"]),
            c["loc_off"], from_bits(c["mem_k"]), from_bits(c["mem_v"]), sel_off, sel, int(np.diff(c["sel_off"]).max()))
    ws = torch.empty(msa.attend_workspace(*args, pos_offset=16.0), dtype=torch.uint8, device="cuda")
    msa.attend(*args, out, ws, out_f32=of, lse=lse, pos_offset=16.0)
    msa.sync_check()
    o_out, o_lse = oracle.attend(**c, pos_offset=16.0)
    err = np.abs(of.cpu().numpy() - o_out).max()
    assert err <= 1e-2, err
    np.testing.assert_array_equal(bits(out), synth.bf16_bits(of.cpu().numpy()))
    np.testing.assert_allclose(lse.cpu().numpy(), o_lse, atol=1e-3, rtol=0)
