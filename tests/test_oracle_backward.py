"""Pins for the oracle's gradients (no GPU): the fp64-input forwards equal the
pinned bfloat16 forwards on bfloat16-valued inputs, and the analytic
gradients equal central finite differences of those forwards."""
import numpy as np
import pytest

import oracle
import synth

RNG = np.random.default_rng(77)


def bf(x):
    return synth.bf16_bits(np.asarray(x, np.float64))


def f64(b):
    return oracle.bf16_to_f64(b)


def _attn_inputs(rows=(2, 1), n_loc=(4, 3), n_mem=(5, 2), q_start=(2, 2), hq=8, hkv=2, d=16, C=9):
    T, L = sum(rows), sum(n_loc)
    return dict(q=bf(RNG.standard_normal((T, hq, d))), q_seq_off=np.concatenate([[0], np.cumsum(rows)]),
                q_start=np.array(q_start), k_loc=bf(RNG.standard_normal((L, hkv, d))),
                v_loc=bf(RNG.standard_normal((L, hkv, d))), loc_off=np.concatenate([[0], np.cumsum(n_loc)]),
                mem_k=bf(RNG.standard_normal((C, hkv, d))), mem_v=bf(RNG.standard_normal((C, hkv, d))),
                sel_off=np.concatenate([[0], np.cumsum(n_mem)]),
                sel_chunk=np.concatenate([RNG.choice(C, m, replace=False) for m in n_mem]).astype(np.int64))


def test_fp64_forwards_equal_bf16_forwards():
    c = _attn_inputs()
    a, la = oracle.attend(**c, pos_offset=5.0, rope_theta=1e4)
    b, lb = oracle.attend_f64(**c, pos_offset=5.0, rope_theta=1e4)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)
    kr = bf(RNG.standard_normal((30, 4, 16)))
    dco = np.array([0, 5, 5, 12, 30])
    qr = bf(RNG.standard_normal((3, 4, 16)))
    _, _, ds = oracle.route(kr, dco, qr, [0, 1, 3], 2)
    np.testing.assert_array_equal(oracle.route_scores_f64(kr, dco, qr, [0, 1, 3]), ds)


def _fd(f, x, h=1e-6):
    g = np.empty_like(x)
    flat, gf = x.reshape(-1), g.reshape(-1)
    for i in range(flat.size):
        v = flat[i]
        flat[i] = v + h
        fp = f()
        flat[i] = v - h
        fm = f()
        flat[i] = v
        gf[i] = (fp - fm) / (2 * h)
    return g


def test_attend_gradients_match_finite_differences():
    c = _attn_inputs()
    x = {k: (f64(v) if v.dtype == np.uint16 else v) for k, v in c.items()}
    W = RNG.standard_normal((sum((2, 1)), 8, 16))
    pos, theta = 7.0, 1e4

    def loss():
        out, _ = oracle.attend_f64(**x, pos_offset=pos, rope_theta=theta)
        return float(np.sum(out * W))

    out, lse, dq, dkl, dvl, dmk, dmv = oracle.attend_f64(**x, pos_offset=pos, rope_theta=theta, dout=W)
    np.testing.assert_allclose(dq, _fd(loss, x["q"]), atol=1e-7)
    np.testing.assert_allclose(dkl, _fd(loss, x["k_loc"]), atol=1e-7)
    np.testing.assert_allclose(dvl, _fd(loss, x["v_loc"]), atol=1e-7)
    # memory rows: gradient per selected row; a chunk selected by two sequences sums both
    fd_mk, fd_mv = _fd(loss, x["mem_k"]), _fd(loss, x["mem_v"])
    got_mk, got_mv = np.zeros_like(x["mem_k"]), np.zeros_like(x["mem_v"])
    for pos_in_sel, chunk in enumerate(c["sel_chunk"]):
        got_mk[chunk] += dmk[pos_in_sel]
        got_mv[chunk] += dmv[pos_in_sel]
    np.testing.assert_allclose(got_mk, fd_mk, atol=1e-7)
    np.testing.assert_allclose(got_mv, fd_mv, atol=1e-7)


def test_route_gradients_match_finite_differences():
    # documents of 3 chunks; each planted row makes one (row, chunk) pair the
    # clear argmax of its document, so the score is smooth around the input
    hr, d = 4, 16
    kr = RNG.standard_normal((24, hr, d))
    dco = np.array([0, 3, 6, 9, 12, 15, 18, 21, 24])
    qr = RNG.standard_normal((5, hr, d))
    qr[1] = kr[4] + 0.05 * RNG.standard_normal((hr, d))   # sequence 0 -> doc 1, chunk 4
    qr[3] = kr[20] + 0.05 * RNG.standard_normal((hr, d))  # sequence 1 -> doc 6, chunk 20
    qso = [0, 2, 5]
    pairs_s, pairs_d, dsc = [0, 1, 1], [1, 6, 2], [0.7, -1.3, 0.4]

    def loss():
        ds = oracle.route_scores_f64(kr, dco, qr, qso)
        return float(sum(g * ds[s, j] for s, j, g in zip(pairs_s, pairs_d, dsc)))

    dq, dk, ac, ar = oracle.route_backward(kr, dco, qr, qso, pairs_s, pairs_d, dsc)
    assert ac[0] == 4 and ar[0] == 1 and ac[1] == 20 and ar[1] == 3
    np.testing.assert_allclose(dq, _fd(loss, qr), atol=1e-7)
    fd_k = _fd(loss, kr)
    got_k = np.zeros_like(kr)
    for p, c in enumerate(ac):
        got_k[c] += dk[p]
    np.testing.assert_allclose(got_k, fd_k, atol=1e-7)


def test_route_gradient_of_a_zero_query_head_uses_the_clamp():
    # |q_h| below eps: the inverse norm is the constant 1/eps, so the gradient
    # is k * invq * invk / hr with no normalisation term
    kr = RNG.standard_normal((2, 2, 8))
    qr = np.zeros((1, 2, 8))
    qr[0, 0] = kr[1, 0]
    dq, dk, ac, ar = oracle.route_backward(kr, [0, 2], qr, [0, 1], [0], [0], [1.0], eps=1e-8)
    assert ac[0] == 1
    np.testing.assert_allclose(dq[0, 1], kr[1, 1] * 1e8 / np.linalg.norm(kr[1, 1]) / 2, rtol=1e-12)


def test_route_gradient_goes_to_the_first_of_tied_maxima():
    # two identical chunks tie exactly; the gradient follows the forward's
    # order (chunk-major, row-minor): the first chunk, the first row
    kr = RNG.standard_normal((3, 2, 8))
    kr[2] = kr[1]
    qr = np.stack([kr[1], kr[1]])
    dq, dk, ac, ar = oracle.route_backward(kr, [0, 3], qr, [0, 2], [0], [0], [1.0])
    assert ac[0] == 1 and ar[0] == 0
    assert np.all(dq[1] == 0.0)
