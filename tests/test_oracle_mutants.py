"""The oracle pins must catch plausible mistakes.

Each case below plants one mistake in a copy of the oracle's C source (on the
CPU, in a temporary directory), builds it, points the oracle binding at it and
runs the pin tests: at least one pin must fail for every mutant.
"""
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle as pins
from tests import test_oracle_backward as grad_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "msa_oracle.c")

MUTANTS = {
    "rope_sign": ("x[i] = x0 * c - x1 * s;", "x[i] = x0 * c + x1 * s;"),
    "rope_frequency": ("pow(theta, -2.0 * (double)i / (double)d)", "pow(theta, -1.0 * (double)i / (double)d)"),
    "rope_pairing": ("double x0 = x[i], x1 = x[i + h];", "double x0 = x[i], x1 = x[(i + h + 1) % d];"),
    "encode_global_position": ("int64_t p = q * chunk + u; /* document-local position */",
                               "int64_t p = t0 + q * chunk + u;"),
    "encode_chunk_rotation_global": ("orc_rope(sk + (size_t)h * d, d, (double)q, rope_theta);",
                                     "orc_rope(sk + (size_t)h * d, d, (double)c, rope_theta);"),
    "encode_full_chunk_divisor": ("kbar[(size_t)c * hkv * d + i] = orc_double_to_bf16(sk[i] / (double)n);",
                                  "kbar[(size_t)c * hkv * d + i] = orc_double_to_bf16(sk[i] / (double)chunk);"),
    "encode_norm_unrounded": ("double x = orc_bf16_to_double(b);", "double x = sr[(size_t)h * d + i] / (double)n + 1e-3;"),
    "route_no_head_mean": ("return cos_sum / (double)hr; /* mean over heads */", "return cos_sum;"),
    "route_mean_not_max": ("if (sc > best) best = sc; /* max over rows and chunks */",
                           "best = (best == -INFINITY ? 0.0 : best) + sc;"),
    "route_missing_knorm": ("cos_sum += dot * inv_q[h] * inv_k[h];", "cos_sum += dot * inv_q[h];"),
    "route_ties_high_id": ("return (x->id > y->id) - (x->id < y->id);", "return (x->id < y->id) - (x->id > y->id);"),
    "route_transposed_head": ("kr, ((size_t)c * hr + h) * d, d);", "kr, ((size_t)c * hr + (hr - 1 - h)) * d, d);"),
    "attend_gqa_modulo": ("int kh = h / group;", "int kh = h % hkv;"),
    "attend_causal_strict": ("for (int64_t j = 0; j < n_loc && j <= gq; ++j) {",
                             "for (int64_t j = 0; j < n_loc && j < gq; ++j) {"),
    "attend_no_query_offset": ("orc_rope(qv, d, pos_offset + (double)gq, rope_theta);",
                               "orc_rope(qv, d, (double)gq, rope_theta);"),
    "backward_no_softmax_term": ("double ds = p * (dp - D);", "double ds = p * dp;"),
    "backward_q_not_rotated_back": ("orc_rope(g, d, -(pos_offset + (double)gq), rope_theta);", "(void)0;"),
    "backward_local_k_not_rotated_back": ("orc_rope(kv, d, -(pos_offset + (double)gidx[j]), rope_theta);", "(void)0;"),
    "backward_dv_unweighted": ("for (int i = 0; i < d; ++i) dv[i] += p * go[i];", "for (int i = 0; i < d; ++i) dv[i] += go[i];"),
    "route_backward_no_norm_term": ("double gq = kv[i] * iq * ik - (nq > eps ? dot * ik * iq * iq * iq * qv[i] : 0.0);",
                                    "double gq = kv[i] * iq * ik;"),
    "route_backward_wrong_argmax": ("if (sc > best) { best = sc; cb = c; tb = t; }", "if (sc >= best) { best = sc; cb = c; tb = t; }"),
    "attend_lse_no_max": ("lse[(size_t)r * hq + h] = mx + log(den);", "lse[(size_t)r * hq + h] = log(den);"),
    "bf16_truncate": ("double r = nearbyint(ldexp(ax, -q));", "double r = floor(ldexp(ax, -q));"),
    "gather_skips_last_chunk": ("for (int64_t c = doc_chunk_off[doc]; c < doc_chunk_off[doc + 1]; ++c) {",
                                "for (int64_t c = doc_chunk_off[doc]; c + 1 < doc_chunk_off[doc + 1]; ++c) {"),
    "gather_reverse_rank": ("int32_t doc = top_ids[(size_t)s * top_k + i];",
                            "int32_t doc = top_ids[(size_t)s * top_k + (top_k - 1 - i)];"),
    "encode_rotates_v": ("for (int i = 0; i < d; ++i) sv[(size_t)h * d + i] += orc_bf16_to_double(vs[i]);",
                         "{ double w[1024]; for (int i = 0; i < d; ++i) w[i] = orc_bf16_to_double(vs[i]); "
                         "orc_rope(w, d, (double)p, rope_theta); for (int i = 0; i < d; ++i) sv[(size_t)h * d + i] += w[i]; }"),
    "encode_rotates_kr": ("for (int i = 0; i < d; ++i) sr[(size_t)h * d + i] += orc_bf16_to_double(rs[i]);",
                          "{ double w[1024]; for (int i = 0; i < d; ++i) w[i] = orc_bf16_to_double(rs[i]); "
                          "orc_rope(w, d, (double)p, rope_theta); for (int i = 0; i < d; ++i) sr[(size_t)h * d + i] += w[i]; }"),
    "encode_v_full_chunk_divisor": ("vbar[(size_t)c * hkv * d + i] = orc_double_to_bf16(sv[i] / (double)n);",
                                    "vbar[(size_t)c * hkv * d + i] = orc_double_to_bf16(sv[i] / (double)chunk);"),
    "route_missing_qnorm": ("cos_sum += dot * inv_q[h] * inv_k[h];", "cos_sum += dot * inv_k[h];"),
    "route_norm_eps_added": ("inv[(size_t)r * hr + h] = 1.0 / (nrm > eps ? nrm : eps);",
                             "inv[(size_t)r * hr + h] = 1.0 / (nrm + eps);"),
    "route_first_row_only": ("for (int64_t t = q_seq_off[s]; t < q_seq_off[s + 1]; ++t) {",
                             "for (int64_t t = q_seq_off[s]; t < q_seq_off[s] + 1; ++t) {"),
    "attend_memory_keys_rotated": ("gidx[n++] = sel_off[s] + m;",
                                   "{ orc_rope(keys + (size_t)n * d, d, pos_offset, rope_theta); double t2 = 0.0; "
                                   "for (int i = 0; i < d; ++i) t2 += qv[i] * keys[(size_t)n * d + i]; "
                                   "logit[n] = t2 * scale; } gidx[n++] = sel_off[s] + m;"),
    "attend_local_keys_no_offset": ("orc_rope(kv, d, pos_offset + (double)j, rope_theta);",
                                    "orc_rope(kv, d, (double)j, rope_theta);"),
    "attend_values_from_keys": ("for (int i = 0; i < d; ++i) o[i] += p * orc_ld(vv, voff[j] + i);",
                                "for (int i = 0; i < d; ++i) o[i] += p * orc_ld(vsrc[j] ? k_loc : mem_k, voff[j] + i);"),
    "attend_q_start_ignored": ("int64_t gq = (int64_t)q_start[s] + (r - q_seq_off[s]);",
                               "int64_t gq = (int64_t)(r - q_seq_off[s]);"),
    "bf16_ties_away": ("double r = nearbyint(ldexp(ax, -q));", "double r = round(ldexp(ax, -q));"),
    "backward_memory_key_rotated_back": ("for (int i = 0; i < d; ++i) dk[i] += scale * ds * qv[i];\n          }",
                                         "double w[1024]; for (int i = 0; i < d; ++i) w[i] = scale * ds * qv[i]; "
                                         "orc_rope(w, d, -pos_offset, rope_theta); for (int i = 0; i < d; ++i) dk[i] += w[i];\n          }"),
}

PIN_TESTS = ([getattr(pins, n) for n in dir(pins) if n.startswith("test_")] +
             [getattr(grad_pins, n) for n in dir(grad_pins) if n.startswith("test_")])


def _build(src_text, workdir, name):
    c = os.path.join(workdir, name + ".c")
    so = os.path.join(workdir, name + ".so")
    with open(c, "w") as f:
        f.write(src_text)
    shutil.copy(os.path.join(os.path.dirname(SRC), "msa_oracle.h"), workdir)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-o", so, c,
                    "-lm"], check=True)
    return so


def _failing_pins():
    failed = []
    for t in PIN_TESTS:
        try:
            t()
        except Exception:  # any assertion or error counts as caught
            failed.append(t.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    before, after = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(before) >= 1, f"mutation site for {name} not found"
    with tempfile.TemporaryDirectory() as tmp:
        so = _build(text.replace(before, after, 1), tmp, name)
        oracle.use_library(so)
        try:
            failed = _failing_pins()
        finally:
            oracle.use_library(None)
    assert failed, f"no pin caught the planted mistake {name}"
