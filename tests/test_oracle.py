"""Pins for the CPU oracle (no GPU).

The pages print no worked example, so each oracle function is pinned to
closed forms, invariants, special cases that reduce to a library routine,
hand-derived fixtures and brute-force enumeration; each pin is chosen so that
a plausible slip (a dropped term, a wrong sign or index, a transposed operand)
fails it.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def bf(x):
    return synth.bf16_bits(np.asarray(x, np.float64))


def f64(b):
    return oracle.bf16_to_f64(b)


# --------------------------------------------------------------- bfloat16

def test_bf16_golden_cases():
    with open(os.path.join(GOLDEN, "bf16_rne.txt")) as f:
        rows = [ln.split("|") for ln in f if ln.strip() and not ln.startswith("#")]
    assert len(rows) >= 10
    for val, bits, _ in rows:
        got = int(oracle.f64_to_bf16(np.array([float(val)]))[0])
        assert got == int(bits, 16), (val, hex(got), bits)


def test_bf16_matches_torch_on_float32_values():
    # For values that are exact float32 numbers a single rounding to bfloat16
    # is what torch's float32 -> bfloat16 conversion does.
    x = np.concatenate([
        RNG.standard_normal(20000) * 10.0 ** RNG.integers(-30, 30, 20000),
        (1.0 + np.arange(0, 512) * 2.0 ** -15),  # dense grid around 1 including ties
        np.array([0.0, -0.0, 1e-40, -1e-40, 3.39e38, -3.39e38]),
    ]).astype(np.float32).astype(np.float64)
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    got = oracle.f64_to_bf16(x).view(np.int16)
    np.testing.assert_array_equal(got, want)


def test_bf16_roundtrip_exact():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    vals = f64(bits)
    finite = np.isfinite(vals)
    back = oracle.f64_to_bf16(vals[finite])
    # -0.0 and +0.0 both survive with their sign; every finite pattern round-trips.
    np.testing.assert_array_equal(back, bits[finite])


# -------------------------------------------------------------------- RoPE

THETA = 1e6


def test_rope_position_zero_is_identity():
    x = RNG.standard_normal(128)
    np.testing.assert_array_equal(oracle.rope(x, 0.0, THETA), x)


def test_rope_closed_form_basis_vectors():
    d = 128
    for p in [1.0, 7.0, 4095.0]:
        e0 = np.zeros(d); e0[0] = 1.0
        y = oracle.rope(e0, p, THETA)
        # pair 0 has frequency theta^0 = 1: rotation by p radians into x[64]
        assert y[0] == pytest.approx(math.cos(p), abs=1e-15)
        assert y[64] == pytest.approx(math.sin(p), abs=1e-15)
        assert np.count_nonzero(y) == 2
        # pair 32 has frequency theta^(-1/2)
        e = np.zeros(d); e[96] = 1.0
        y = oracle.rope(e, p, THETA)
        w = p * THETA ** -0.5
        assert y[32] == pytest.approx(-math.sin(w), abs=1e-15)
        assert y[96] == pytest.approx(math.cos(w), abs=1e-15)


def test_rope_preserves_pair_norms_and_composes():
    x = RNG.standard_normal(128)
    y = oracle.rope(x, 123.0, THETA)
    np.testing.assert_allclose(x[:64] ** 2 + x[64:] ** 2, y[:64] ** 2 + y[64:] ** 2, rtol=1e-12)
    z = oracle.rope(oracle.rope(x, 100.0, THETA), 23.0, THETA)
    np.testing.assert_allclose(z, y, atol=1e-12)
    back = oracle.rope(y, -123.0, THETA)
    np.testing.assert_allclose(back, x, atol=1e-12)


def test_rope_relative_position_property():
    q, k = RNG.standard_normal(128), RNG.standard_normal(128)
    a = oracle.rope(q, 50.0, THETA) @ oracle.rope(k, 20.0, THETA)
    b = oracle.rope(q, 1030.0, THETA) @ oracle.rope(k, 1000.0, THETA)
    c = oracle.rope(q, 31.0, THETA) @ oracle.rope(k, 1.0, THETA)
    assert a == pytest.approx(b, abs=1e-9)
    assert a == pytest.approx(c, abs=1e-9)
    assert abs(a - oracle.rope(q, 51.0, THETA) @ oracle.rope(k, 20.0, THETA)) > 1e-6


# ------------------------------------------------------------------ encode

def _rand_tokens(n, h, d, scale=1.0):
    return bf(RNG.standard_normal((n, h, d)) * scale)


def test_encode_chunk_structure_and_partial_chunks():
    lens = [64, 63, 65, 128, 1, 0, 191, 64 * 3 + 1]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(off[-1])
    k, v, kr = _rand_tokens(n, 2, 16), _rand_tokens(n, 2, 16), _rand_tokens(n, 3, 16)
    out = oracle.encode(k, v, kr, off, chunk=64)
    want_counts = [math.ceil(x / 64) for x in lens]
    assert list(np.diff(out["doc_chunk_off"])) == want_counts
    assert list(out["chunk_doc"]) == [j for j, c in enumerate(want_counts) for _ in range(c)]


def test_encode_constant_chunks_pool_exactly():
    # Tokens constant within each chunk (different per chunk, partial chunks
    # included): the mean of V and K_r must be that constant, bit for bit.
    lens = [64, 100, 1, 129]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(off[-1])
    hkv, hr, d = 2, 3, 16
    v = np.empty((n, hkv, d), np.uint16)
    kr = np.empty((n, hr, d), np.uint16)
    consts_v, consts_r = [], []
    for j, L in enumerate(lens):
        for q in range(math.ceil(L / 64)):
            cv = bf(RNG.standard_normal((hkv, d)))
            cr = bf(RNG.standard_normal((hr, d)))
            t0 = int(off[j]) + 64 * q
            t1 = min(int(off[j + 1]), t0 + 64)
            v[t0:t1] = cv
            kr[t0:t1] = cr
            consts_v.append(cv)
            consts_r.append(cr)
    k = _rand_tokens(n, hkv, d)
    out = oracle.encode(k, v, kr, off, chunk=64)
    np.testing.assert_array_equal(out["vbar"], np.stack(consts_v))
    np.testing.assert_array_equal(out["kbar_r"], np.stack(consts_r))


def test_encode_single_token_doc_is_unrotated_copy():
    off = np.array([0, 1], np.int64)
    k, v, kr = _rand_tokens(1, 2, 16), _rand_tokens(1, 2, 16), _rand_tokens(1, 2, 16)
    out = oracle.encode(k, v, kr, off)
    np.testing.assert_array_equal(out["kbar"][0], k[0])
    np.testing.assert_array_equal(out["vbar"][0], v[0])
    np.testing.assert_array_equal(out["kbar_r"][0], kr[0])


def test_encode_positions_restart_in_every_document():
    # Two documents with identical token content must pool identically
    # (document-wise RoPE from 0), whatever their place in the corpus.
    L = 150
    k1, v1, r1 = _rand_tokens(L, 2, 16), _rand_tokens(L, 2, 16), _rand_tokens(L, 2, 16)
    pad = 77
    kp, vp, rp = _rand_tokens(pad, 2, 16), _rand_tokens(pad, 2, 16), _rand_tokens(pad, 2, 16)
    k = np.concatenate([k1, kp, k1]); v = np.concatenate([v1, vp, v1]); r = np.concatenate([r1, rp, r1])
    off = np.array([0, L, L + pad, 2 * L + pad], np.int64)
    out = oracle.encode(k, v, r, off)
    dco = out["doc_chunk_off"]
    a = slice(dco[0], dco[1]); b = slice(dco[2], dco[3])
    np.testing.assert_array_equal(out["kbar"][a], out["kbar"][b])
    np.testing.assert_array_equal(out["vbar"][a], out["vbar"][b])
    # ... and RoPE really is applied: K-bar of the first chunk differs from plain mean of K.
    plain = oracle.f64_to_bf16(f64(k1[:64]).mean(axis=0))
    assert np.count_nonzero(out["kbar"][0] != plain) > 0


def test_encode_rotated_mean_matches_dirichlet_closed_form():
    # n identical tokens x at positions p0..p0+n-1: the mean of the rotations of
    # pair (a, b) by (p0+u)*w equals the rotation of (a, b) by (p0+(n-1)/2)*w
    # scaled by sin(n w / 2) / (n sin(w / 2)).
    d, theta = 128, 1e4
    x = bf(RNG.standard_normal((1, 1, d)))
    for L in [64 * 3 + 17, 64 * 5]:
        k = np.repeat(x, L, axis=0)
        off = np.array([0, L], np.int64)
        out = oracle.encode(k, k, k, off, rope_theta=theta)
        xv = f64(x[0, 0])
        for q in range(math.ceil(L / 64)):
            p0 = 64 * q
            n = min(64, L - p0)
            want = np.empty(d)
            for i in range(d // 2):
                w = theta ** (-2.0 * i / d)
                g = 1.0 if abs(math.sin(w / 2)) < 1e-300 else math.sin(n * w / 2) / (n * math.sin(w / 2))
                ang = (p0 + (n - 1) / 2.0) * w
                a, b = xv[i], xv[i + d // 2]
                want[i] = g * (a * math.cos(ang) - b * math.sin(ang))
                want[i + d // 2] = g * (a * math.sin(ang) + b * math.cos(ang))
            got = f64(out["kbar"][q, 0])
            # one bfloat16 rounding of the result: within half an ulp (+ fp64 noise)
            ulp = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7), 2.0 ** -133)
            assert np.all(np.abs(got - want) <= 0.5 * ulp + 1e-12), q


def test_encode_pool_then_rotate_reading():
    # rope_mode 1: the pooled chunk q of a document is rotated at position q.
    # Identical tokens x: K-bar = bf16(R(q w) x) exactly up to one rounding.
    d, theta = 128, 1e4
    x = bf(RNG.standard_normal((1, 1, d)))
    L = 64 * 3 + 5
    k = np.repeat(x, L, axis=0)
    out = oracle.encode(k, k, k, np.array([0, L], np.int64), rope_theta=theta, rope_mode=1)
    for q in range(4):
        want = oracle.rope(f64(x[0, 0]), float(q), theta)
        got = f64(out["kbar"][q, 0])
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 1e-30))) - 7)
        assert np.all(np.abs(got - want) <= 0.5 * ulp + 1e-12), q
    # the two readings agree on a document's first chunk only at position 0 for a single token
    one = oracle.encode(k[:1], k[:1], k[:1], np.array([0, 1], np.int64), rope_mode=1)
    np.testing.assert_array_equal(one["kbar"][0], x[0])
    # and the pooled values and routing keys do not depend on the reading
    np.testing.assert_array_equal(out["vbar"], oracle.encode(k, k, k, np.array([0, L], np.int64))["vbar"])
    # chunk indices restart in every document: two identical documents pool identically
    kk = np.concatenate([k, k])
    two = oracle.encode(kk, kk, kk, np.array([0, L, 2 * L], np.int64), rope_theta=theta, rope_mode=1)
    n = math.ceil(L / 64)
    np.testing.assert_array_equal(two["kbar"][:n], two["kbar"][n:])


def test_encode_inverse_norms():
    lens = [64, 64]
    off = np.array([0, 64, 128], np.int64)
    k, v = _rand_tokens(128, 1, 8), _rand_tokens(128, 1, 8)
    kr = _rand_tokens(128, 2, 8)
    kr[64:, 1] = 0  # second chunk, second head: zero vector -> clamped norm
    out = oracle.encode(k, v, kr, off, eps=1e-8)
    inv = out["kr_inv_norm"]
    for c in range(2):
        for h in range(2):
            x = f64(out["kbar_r"][c, h])
            if c == 1 and h == 1:
                assert inv[c, h] == pytest.approx(1e8)
            else:
                assert inv[c, h] * math.sqrt(float(x @ x)) == pytest.approx(1.0, rel=1e-14)


# ------------------------------------------------------------------- route

def _bank(n_docs, chunks_per_doc, hr, d, scale=1.0):
    nch = np.asarray(chunks_per_doc if np.ndim(chunks_per_doc) else [chunks_per_doc] * n_docs)
    dco = np.concatenate([[0], np.cumsum(nch)]).astype(np.int64)
    kr = _rand_tokens(int(dco[-1]), hr, d, scale)
    return kr, dco


def test_route_reduces_to_cosine_knn():
    # One head, one chunk per document, one query row: the score is the cosine
    # similarity, so the ranking is a cosine nearest-neighbour search.
    from sklearn.neighbors import NearestNeighbors
    kr, dco = _bank(300, 1, 1, 32)
    qr = _rand_tokens(1, 1, 32)
    ids, sc, ds = oracle.route(kr, dco, qr, [0, 1], top_k=10)
    nn = NearestNeighbors(n_neighbors=10, metric="cosine", algorithm="brute").fit(f64(kr[:, 0]))
    dist, idx = nn.kneighbors(f64(qr[:, 0]))
    np.testing.assert_array_equal(ids[0], idx[0])
    np.testing.assert_allclose(sc[0], 1.0 - dist[0], atol=1e-12)


def test_route_scores_are_cosines_in_range_and_scale_invariant():
    kr, dco = _bank(64, 3, 4, 32)
    qr = _rand_tokens(5, 4, 32)
    _, _, ds = oracle.route(kr, dco, qr, [0, 2, 5], top_k=4)
    assert np.all(ds <= 1.0 + 1e-12) and np.all(ds >= -1.0 - 1e-12)
    kr2 = oracle.f64_to_bf16(2.0 * f64(kr))  # exact in bfloat16
    qr2 = oracle.f64_to_bf16(4.0 * f64(qr))
    _, _, ds2 = oracle.route(kr2, dco, qr2, [0, 2, 5], top_k=4)
    np.testing.assert_allclose(ds2, ds, atol=1e-14)


def test_route_each_norm_is_clamped_at_eps():
    # With eps = 0.5 a vector shorter than eps counts as if it had length eps:
    # for parallel q and k the score is |q| |k| / (max(|q|, eps) max(|k|, eps)),
    # exactly 1 when both are longer than eps and proportionally less when not.
    hr, d = 4, 32
    e = np.zeros((hr, d))
    e[np.arange(hr), 3 * np.arange(hr)] = 1.0  # one unit direction per head
    kbar = np.stack([2.0 * e, 0.25 * e, np.roll(e, 1, axis=1)])  # docs: long, short, orthogonal
    qr = np.stack([0.25 * e, 2.0 * e])  # sequence 0: a short row, sequence 1: a long row
    _, _, ds = oracle.route(bf(kbar), [0, 1, 2, 3], bf(qr), [0, 1, 2], top_k=3, eps=0.5)
    np.testing.assert_allclose(ds, [[0.5, 0.25, 0.0], [1.0, 0.5, 0.0]], atol=1e-15)


def test_route_mean_over_heads():
    # Two heads; the second query head is the zero vector, so it contributes
    # nothing and every score is half the first head's cosine.
    kr, dco = _bank(50, 1, 2, 16)
    qr = _rand_tokens(1, 2, 16)
    qr[0, 1] = 0
    _, _, ds = oracle.route(kr, dco, qr, [0, 1], top_k=3)
    _, _, ds1 = oracle.route(np.ascontiguousarray(kr[:, :1]), dco,
                             np.ascontiguousarray(qr[:, :1]), [0, 1], top_k=3)
    np.testing.assert_allclose(ds, ds1 / 2.0, atol=1e-14)


def test_route_max_over_rows_and_chunks():
    # Documents of 4 chunks; row 0 equals chunk 2 of doc 7 and row 1 equals
    # chunk 0 of doc 11: both documents score exactly 1 (max, not mean).
    kr, dco = _bank(20, 4, 2, 16)
    qr = np.stack([kr[dco[7] + 2], kr[dco[11]]])
    ids, sc, ds = oracle.route(kr, dco, qr, [0, 2], top_k=2)
    assert sorted(ids[0].tolist()) == [7, 11]
    np.testing.assert_allclose(sc[0], [1.0, 1.0], atol=1e-12)
    if sc[0][0] == sc[0][1]:
        assert ids[0].tolist() == [7, 11]  # equal scores: lower id first
    # splitting the rows into two sequences separates the two documents
    ids2, _, _ = oracle.route(kr, dco, qr, [0, 1, 2], top_k=1)
    assert ids2[:, 0].tolist() == [7, 11]


def test_route_topk_order_ties_and_k_equals_d():
    kr, dco = _bank(10, 2, 2, 8)
    kr[dco[6]:dco[7]] = kr[dco[3]:dco[4]]  # doc 6 duplicates doc 3: an exact tie
    qr = np.ascontiguousarray(kr[dco[3]][None])
    ids, sc, ds = oracle.route(kr, dco, qr, [0, 1], top_k=50)  # k > D clamps to D
    assert ids.shape == (1, 10)
    assert sorted(ids[0].tolist()) == list(range(10))
    assert ids[0, 0] == 3 and ids[0, 1] == 6 and sc[0, 0] == sc[0, 1]
    assert np.all(np.diff(sc[0]) <= 0)
    # brute force over the permutations' defining order: (score desc, id asc)
    order = sorted(range(10), key=lambda j: (-ds[0, j], j))
    assert ids[0].tolist() == order


def test_route_permuting_documents_permutes_ids():
    kr, dco = _bank(40, 2, 2, 16)
    qr = _rand_tokens(3, 2, 16)
    ids, sc, _ = oracle.route(kr, dco, qr, [0, 3], top_k=5)
    perm = RNG.permutation(40)  # new doc j is old doc perm[j]
    new_kr = np.concatenate([kr[dco[p]:dco[p + 1]] for p in perm])
    ids2, sc2, _ = oracle.route(new_kr, dco, qr, [0, 3], top_k=5)
    inv = np.argsort(perm)
    np.testing.assert_array_equal(inv[ids[0]], ids2[0])
    np.testing.assert_allclose(sc2, sc, atol=1e-14)


def test_route_empty_document_ranks_last():
    nch = [2, 0, 3, 1]
    kr, dco = _bank(4, nch, 2, 8)
    qr = _rand_tokens(1, 2, 8)
    ids, sc, ds = oracle.route(kr, dco, qr, [0, 1], top_k=4)
    assert ds[0, 1] == -np.inf
    assert ids[0, -1] == 1


def test_route_rejects_empty_sequence():
    kr, dco = _bank(4, 1, 1, 8)
    qr = _rand_tokens(2, 1, 8)
    with pytest.raises(ValueError):
        oracle.route(kr, dco, qr, [0, 0, 2], top_k=1)


def test_route_planted_needles_retrieved():
    w = synth.workload("tiny")
    dco, _ = w.index()
    C = int(dco[-1])
    kr = synth.normal_bf16_host(C * w.hr * w.d, synth.tid("kbar_r", 0)).reshape(C, w.hr, w.d)
    qr, qso, plan = synth.make_routing_queries(lambda c: f64(kr[c]), dco, [w.route_rows],
                                               w.top_k, w.n_needles, w.hr, w.d, 0)
    ids, sc, ds = oracle.route(kr, dco, qr, qso, w.top_k)
    assert set(ids[0].tolist()) == set(plan.docs[0])
    assert set(ids[0, :3].tolist()) == set(plan.docs[0][:3])  # needles on top
    np.testing.assert_allclose(sorted(sc[0]), sorted(plan.cos[0]), atol=3e-3)
    srt = np.sort(ds[0])[::-1]
    assert srt[w.top_k - 1] - srt[w.top_k] >= 1e-2


# ------------------------------------------------------------------ gather

def test_gather_concatenates_selected_documents_in_rank_order():
    dco = np.array([0, 3, 3, 5, 9, 10], np.int64)
    ids = np.array([[3, 0], [1, 4]], np.int32)
    so, sel = oracle.gather(ids, dco)
    assert so.tolist() == [0, 7, 8]
    assert sel.tolist() == [5, 6, 7, 8, 0, 1, 2, 9]


# ------------------------------------------------------------------ attend

def _attn_case(n_seq=2, rows=(3, 2), n_loc=(5, 4), n_mem=(6, 0), hq=8, hkv=2, d=16, C=12,
               q_start=(2, 3)):
    q = _rand_tokens(sum(rows), hq, d)
    kl = _rand_tokens(sum(n_loc), hkv, d)
    vl = _rand_tokens(sum(n_loc), hkv, d)
    mk = _rand_tokens(C, hkv, d)
    mv = _rand_tokens(C, hkv, d)
    sel = np.concatenate([RNG.choice(C, m, replace=False) for m in n_mem]).astype(np.int64)
    return dict(q=q, q_seq_off=np.concatenate([[0], np.cumsum(rows)]).astype(np.int32),
                q_start=np.array(q_start, np.int32), k_loc=kl, v_loc=vl,
                loc_off=np.concatenate([[0], np.cumsum(n_loc)]).astype(np.int32),
                mem_k=mk, mem_v=mv,
                sel_off=np.concatenate([[0], np.cumsum(n_mem)]).astype(np.int64), sel_chunk=sel)


def test_attend_matches_sdpa_dense_reference():
    # Rotate with the (separately pinned) RoPE, then the rest is standard GQA
    # softmax attention with a mask: torch's scaled_dot_product_attention.
    c = _attn_case()
    pos_off, theta, d = 16.0, 1e4, 16
    out, lse = oracle.attend(**c, pos_offset=pos_off, rope_theta=theta)
    hq, hkv = 8, 2
    for s in range(2):
        r0, r1 = c["q_seq_off"][s], c["q_seq_off"][s + 1]
        l0, l1 = c["loc_off"][s], c["loc_off"][s + 1]
        sel = c["sel_chunk"][c["sel_off"][s]:c["sel_off"][s + 1]]
        g = c["q_start"][s] + np.arange(r1 - r0)
        qr = np.stack([[oracle.rope(f64(c["q"][r, h]), pos_off + g[i], theta) for h in range(hq)]
                       for i, r in enumerate(range(r0, r1))])
        kl = np.stack([[oracle.rope(f64(c["k_loc"][l0 + j, h]), pos_off + j, theta) for h in range(hkv)]
                       for j in range(l1 - l0)])
        K = np.concatenate([f64(c["mem_k"][sel]), kl])
        V = np.concatenate([f64(c["mem_v"][sel]), f64(c["v_loc"][l0:l1])])
        n_mem = sel.size
        mask = np.ones((r1 - r0, K.shape[0]), bool)
        for i in range(r1 - r0):
            mask[i, n_mem:] = np.arange(l1 - l0) <= g[i]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr.transpose(1, 0, 2))[None], torch.from_numpy(K.transpose(1, 0, 2))[None],
            torch.from_numpy(V.transpose(1, 0, 2))[None], attn_mask=torch.from_numpy(mask),
            scale=1.0 / math.sqrt(d), enable_gqa=True)[0].numpy().transpose(1, 0, 2)
        np.testing.assert_allclose(out[r0:r1], ref, atol=1e-12)


def test_attend_lse_closed_form_without_rotation():
    # pos_offset = 0 and one query row at active index 0 with no local keys
    # visible beyond j = 0: memory logits are plain scaled dot products.
    c = _attn_case(n_seq=1, rows=(1,), n_loc=(1,), n_mem=(7,), q_start=(0,))
    out, lse = oracle.attend(**c, pos_offset=0.0, rope_theta=1e6)
    from scipy.special import logsumexp
    d, hq, hkv = 16, 8, 2
    sel = c["sel_chunk"]
    for h in range(hq):
        kh = h // (hq // hkv)
        qv = f64(c["q"][0, h])
        keys = np.concatenate([f64(c["mem_k"][sel, kh]), f64(c["k_loc"][0:1, kh])])
        vals = np.concatenate([f64(c["mem_v"][sel, kh]), f64(c["v_loc"][0:1, kh])])
        lg = keys @ qv / math.sqrt(d)
        assert lse[0, h] == pytest.approx(logsumexp(lg), abs=1e-12)
        w = np.exp(lg - logsumexp(lg))
        np.testing.assert_allclose(out[0, h], w @ vals, atol=1e-12)


def test_attend_invariants():
    c = _attn_case()
    base, lse = oracle.attend(**c, pos_offset=16.0)
    # constant values: weights sum to one, so the output is that constant
    c1 = dict(c)
    c1["v_loc"] = bf(np.full(c["v_loc"].shape, 0.75))
    c1["mem_v"] = bf(np.full(c["mem_v"].shape, 0.75))
    o1, _ = oracle.attend(**c1, pos_offset=16.0)
    np.testing.assert_allclose(o1, 0.75, atol=1e-14)
    # zero query: uniform weights -> mean of the visible values, lse = log(count)
    c2 = dict(c)
    c2["q"] = np.zeros_like(c["q"])
    o2, l2 = oracle.attend(**c2, pos_offset=16.0)
    s, r = 0, 1  # sequence 0, its second row: g = 3 -> local 0..3 plus 6 memory keys
    vis = np.concatenate([f64(c["mem_v"][c["sel_chunk"][:6], 0]), f64(c["v_loc"][0:4, 0])])
    np.testing.assert_allclose(o2[r, 0], vis.mean(axis=0), atol=1e-14)
    assert l2[r, 0] == pytest.approx(math.log(10.0), abs=1e-14)
    # order of the selected chunks does not matter
    c3 = dict(c)
    c3["sel_chunk"] = c["sel_chunk"].copy()
    c3["sel_chunk"][:6] = c["sel_chunk"][:6][::-1]
    o3, _ = oracle.attend(**c3, pos_offset=16.0)
    np.testing.assert_allclose(o3, base, atol=1e-13)
    # causality: future local values do not reach an earlier row
    c4 = dict(c)
    c4["v_loc"] = c["v_loc"].copy()
    c4["v_loc"][4] = bf(RNG.standard_normal(c["v_loc"][4].shape))  # seq 0, j = 4 > g of rows 0,1
    o4, _ = oracle.attend(**c4, pos_offset=16.0)
    np.testing.assert_array_equal(o4[0:2], base[0:2])
    assert not np.allclose(o4[2], base[2])


def test_attend_single_key_and_position_offset():
    # one local key, no memory: output is that value whatever the query
    c = _attn_case(n_seq=1, rows=(1,), n_loc=(1,), n_mem=(0,), q_start=(0,))
    out, lse = oracle.attend(**c, pos_offset=5.0)
    for h in range(8):
        np.testing.assert_array_equal(out[0, h], f64(c["v_loc"][0, h // 4]))
    # with local keys only, a global shift of positions changes nothing (RoPE is relative) ...
    c = _attn_case(n_seq=1, rows=(3,), n_loc=(6,), n_mem=(0,), q_start=(3,))
    a, _ = oracle.attend(**c, pos_offset=0.0)
    b, _ = oracle.attend(**c, pos_offset=37.0)
    np.testing.assert_allclose(a, b, atol=1e-12)
    # ... but with memory keys (rotated at document-local positions) it does
    c = _attn_case(n_seq=1, rows=(3,), n_loc=(6,), n_mem=(5,), q_start=(3,))
    a, _ = oracle.attend(**c, pos_offset=0.0)
    b, _ = oracle.attend(**c, pos_offset=37.0)
    assert np.abs(a - b).max() > 1e-3


def test_attend_k_equals_all_documents_is_dense_attention():
    # Selecting every document reproduces dense attention over all pooled KV
    # plus the local keys; order of the chunk list is irrelevant.
    c = _attn_case(n_seq=1, rows=(2,), n_loc=(3,), n_mem=(12,), q_start=(1,))
    dense, _ = oracle.attend(**c, pos_offset=4.0)
    c2 = dict(c)
    c2["sel_chunk"] = np.arange(12, dtype=np.int64)
    o2, _ = oracle.attend(**c2, pos_offset=4.0)
    np.testing.assert_allclose(o2, dense, atol=1e-13)


# --------------------------------------------------------- sizing figure

def test_routing_key_bytes_match_pages_100m_figure():
    # The pages quote about 56 GB of GPU-resident routing keys for 100M tokens
    # ("MSA-arXiv26", 核心方法, Memory Parallel inference). 18 routing layers x
    # 8 heads x 128 dims x bfloat16 per 64-token chunk reproduces it.
    import json
    fig = json.load(open(os.path.join(GOLDEN, "page_figures.json")))
    w = synth.workload("100m")
    dco, _ = w.index()
    kr_bytes = int(dco[-1]) * w.hr * w.d * 2 * w.n_layers
    assert w.memory_tokens == fig["memory_tokens"]
    assert abs(kr_bytes / 1e9 - fig["routing_key_gb"]) / fig["routing_key_gb"] < 0.05
