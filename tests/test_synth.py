"""The seeded input generator (no GPU): determinism, slicing and moments."""
import numpy as np

import synth


def test_slices_regenerate_bit_identically():
    full = synth.normal_bf16_host(10000, synth.tid("kbar_r", 3))
    part = synth.normal_bf16_host(1000, synth.tid("kbar_r", 3), index0=4321)
    np.testing.assert_array_equal(full[4321:5321], part)
    other = synth.normal_bf16_host(1000, synth.tid("kbar_r", 4), index0=4321)
    assert np.count_nonzero(other != part) > 990


def test_normal_moments():
    x = synth.bits_to_f64(synth.normal_bf16_host(1 << 20, synth.tid("kbar", 0)))
    assert abs(x.mean()) < 5e-3
    assert abs(x.std() - 1.0) < 5e-3
    # Irwin-Hall of four 16-bit uniforms: support within +-sqrt(12) standard deviations
    assert np.abs(x).max() <= np.sqrt(12.0) + 1e-2
    sig = synth.bits_to_f64(synth.normal_bf16_host(1 << 16, synth.tid("kbar", 0), sigma=0.5))
    np.testing.assert_allclose(sig, synth.bits_to_f64(synth.bf16_bits(0.5 * x[: 1 << 16])), rtol=0)


def test_workload_shapes():
    w = synth.workload("10m")
    assert w.memory_tokens == 10_000_000
    lens = np.diff(w.doc_tok_off)
    assert lens[:-1].min() >= 64 and lens.max() <= 8192
    assert 700 < lens.mean() < 1300
    dco, cdoc = w.index()
    assert dco[-1] == cdoc.size and 150_000 < dco[-1] < 170_000
    w = synth.workload("100m")
    dco, _ = w.index()
    assert dco[-1] == 1_562_500 and np.all(np.diff(w.doc_tok_off) % 64 == 0)
    w = synth.workload("encode")
    assert w.memory_tokens == 10_000_000 and w.n_docs == 2442
