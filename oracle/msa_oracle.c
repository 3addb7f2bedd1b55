/* CPU oracle for the MSA routing + sparse attention step.
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, benchmark CPU baseline).
 * See msa_oracle.h for the definitions and the pages each function follows.
 *
 * Deliberately plain: one thread, loops in definition order, fp64 sums, no
 * blocking or fusion. Build without -ffast-math and with -ffp-contract=off. */
#include "msa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- bfloat16 */

double orc_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bfloat16 (8 significant bits), ties to even.
 * bfloat16 has fp32's exponent range: normal numbers down to 2^-126, then
 * subnormals with a fixed quantum of 2^-133; the largest finite value is
 * (2 - 2^-7) * 2^127, and anything that rounds above it is infinite. */
uint16_t orc_double_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double ax = fabs(x);
  if (ax == 0.0) return sign;
  if (isinf(ax)) return sign | 0x7F80;
  int e;
  frexp(ax, &e); /* ax = m * 2^e with m in [0.5, 1) */
  int q = e - 8; /* exponent of the last kept bit */
  if (q < -133) q = -133;
  double r = nearbyint(ldexp(ax, -q)); /* default rounding mode: ties to even */
  double v = ldexp(r, q);
  if (v > 3.3895313892515355e38) return sign | 0x7F80;
  float f = (float)v; /* exact: v has at most 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return sign | (uint16_t)(u >> 16);
}

void orc_bf16_array_to_double(const uint16_t* in, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_to_double(in[i]);
}

void orc_double_array_to_bf16(const double* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_double_to_bf16(in[i]);
}

/* An input array of either bfloat16 bit patterns or doubles. The bfloat16
 * entry points read their inputs through it; the fp64 entry points (used to
 * take finite differences) pass doubles. Either way every value is widened
 * to double before any arithmetic. */
typedef struct {
  const void* p;
  int f64;
} orc_arr;

static inline double orc_ld(orc_arr a, size_t i) {
  return a.f64 ? ((const double*)a.p)[i] : orc_bf16_to_double(((const uint16_t*)a.p)[i]);
}

/* -------------------------------------------------------------------- RoPE */

/* Rotary embedding with half-split pairing. The pages name RoPE without its
 * layout or base; the pairing (i, i + d/2) and the frequency theta^(-2i/d)
 * are the common rotary convention, and theta is a parameter. */
int orc_rope(double* x, int d, double pos, double theta) {
  if (d <= 0 || (d & 1)) return -1;
  int h = d / 2;
  for (int i = 0; i < h; ++i) {
    double w = pow(theta, -2.0 * (double)i / (double)d);
    double a = pos * w;
    double c = cos(a), s = sin(a);
    double x0 = x[i], x1 = x[i + h];
    x[i] = x0 * c - x1 * s;
    x[i + h] = x0 * s + x1 * c;
  }
  return 0;
}

/* ------------------------------------------------------------------ encode */

/* [P1] 核心方法: each document's K/V/K^R come from its own forward pass, then
 * are compressed by chunk-wise mean pooling. [P2] Architecture: document-wise
 * RoPE restarts positions at 0 in every document. Readings:
 *  - RoPE is applied to K per token at its document-local position, before
 *    pooling; V and the routing keys K^R are not rotated.
 *  - A chunk never spans two documents; a document's last chunk may hold fewer
 *    than `chunk` tokens and is the mean over the tokens it holds.
 *  - The pooled values are stored as bfloat16; the inverse norm of each pooled
 *    routing key is taken from the stored (rounded) values, clamped at eps. */
int orc_encode(const uint16_t* k_tok, const uint16_t* v_tok, const uint16_t* kr_tok,
               const int64_t* doc_tok_off, int64_t n_docs, int hkv, int hr, int d, int chunk,
               double rope_theta, double eps, int rope_mode,
               uint16_t* kbar, uint16_t* vbar, uint16_t* kbar_r, double* kr_inv_norm,
               int64_t* doc_chunk_off, int32_t* chunk_doc, int64_t n_chunks) {
  if (n_docs < 0 || hkv <= 0 || hr <= 0 || d <= 0 || (d & 1) || chunk <= 0) return -1;
  if (rope_mode != 0 && rope_mode != 1) return -1;
  int64_t total = 0;
  for (int64_t j = 0; j < n_docs; ++j) {
    int64_t len = doc_tok_off[j + 1] - doc_tok_off[j];
    if (len < 0) return -2;
    total += (len + chunk - 1) / chunk;
  }
  if (total != n_chunks) return -3;

  double* sk = (double*)malloc(sizeof(double) * (size_t)hkv * d);
  double* sv = (double*)malloc(sizeof(double) * (size_t)hkv * d);
  double* sr = (double*)malloc(sizeof(double) * (size_t)hr * d);
  double* row = (double*)malloc(sizeof(double) * (size_t)d);
  if (!sk || !sv || !sr || !row) {
    free(sk); free(sv); free(sr); free(row);
    return -4;
  }

  int64_t c = 0;
  doc_chunk_off[0] = 0;
  for (int64_t j = 0; j < n_docs; ++j) {
    int64_t t0 = doc_tok_off[j];
    int64_t len = doc_tok_off[j + 1] - t0;
    int64_t nch = (len + chunk - 1) / chunk;
    for (int64_t q = 0; q < nch; ++q, ++c) {
      int64_t n = len - q * chunk;
      if (n > chunk) n = chunk;
      memset(sk, 0, sizeof(double) * (size_t)hkv * d);
      memset(sv, 0, sizeof(double) * (size_t)hkv * d);
      memset(sr, 0, sizeof(double) * (size_t)hr * d);
      for (int64_t u = 0; u < n; ++u) {
        int64_t p = q * chunk + u; /* document-local position */
        int64_t t = t0 + p;
        for (int h = 0; h < hkv; ++h) {
          const uint16_t* src = k_tok + ((size_t)t * hkv + h) * d;
          for (int i = 0; i < d; ++i) row[i] = orc_bf16_to_double(src[i]);
          if (rope_mode == 0) orc_rope(row, d, (double)p, rope_theta);
          for (int i = 0; i < d; ++i) sk[(size_t)h * d + i] += row[i];
          const uint16_t* vs = v_tok + ((size_t)t * hkv + h) * d;
          for (int i = 0; i < d; ++i) sv[(size_t)h * d + i] += orc_bf16_to_double(vs[i]);
        }
        for (int h = 0; h < hr; ++h) {
          const uint16_t* rs = kr_tok + ((size_t)t * hr + h) * d;
          for (int i = 0; i < d; ++i) sr[(size_t)h * d + i] += orc_bf16_to_double(rs[i]);
        }
      }
      if (rope_mode == 1) /* pooled chunk rotated at its chunk index */
        for (int h = 0; h < hkv; ++h) orc_rope(sk + (size_t)h * d, d, (double)q, rope_theta);
      for (int64_t i = 0; i < (int64_t)hkv * d; ++i) {
        kbar[(size_t)c * hkv * d + i] = orc_double_to_bf16(sk[i] / (double)n);
        vbar[(size_t)c * hkv * d + i] = orc_double_to_bf16(sv[i] / (double)n);
      }
      for (int h = 0; h < hr; ++h) {
        double ss = 0.0;
        for (int i = 0; i < d; ++i) {
          uint16_t b = orc_double_to_bf16(sr[(size_t)h * d + i] / (double)n);
          kbar_r[((size_t)c * hr + h) * d + i] = b;
          double x = orc_bf16_to_double(b);
          ss += x * x;
        }
        double nrm = sqrt(ss);
        kr_inv_norm[(size_t)c * hr + h] = 1.0 / (nrm > eps ? nrm : eps);
      }
      chunk_doc[c] = (int32_t)j;
    }
    doc_chunk_off[j + 1] = c;
  }
  free(sk); free(sv); free(sr); free(row);
  return 0;
}

/* ------------------------------------------------------------------- route */

typedef struct {
  double score;
  int32_t id;
} orc_ranked;

/* Score descending, then document id ascending: a total order. */
static int orc_rank_cmp(const void* a, const void* b) {
  const orc_ranked* x = (const orc_ranked*)a;
  const orc_ranked* y = (const orc_ranked*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->id > y->id) - (x->id < y->id);
}

static double orc_dot(orc_arr a, size_t ia, orc_arr b, size_t ib, int d) {
  double s = 0.0;
  for (int i = 0; i < d; ++i) s += orc_ld(a, ia + i) * orc_ld(b, ib + i);
  return s;
}

/* 1 / max(|x|, eps) for each of the `rows` x `hr` vectors of a [rows, hr, d] array. */
static void orc_inv_norms(orc_arr x, int64_t rows, int hr, int d, double eps, double* inv) {
  for (int64_t r = 0; r < rows; ++r)
    for (int h = 0; h < hr; ++h) {
      size_t o = ((size_t)r * hr + h) * d;
      double nrm = sqrt(orc_dot(x, o, x, o, d));
      inv[(size_t)r * hr + h] = 1.0 / (nrm > eps ? nrm : eps);
    }
}

/* The routing score of query row t against pooled chunk c: the mean over
 * heads of cos = q.k / (max(|q|, eps) max(|k|, eps)); inv_q and inv_k hold
 * the row's and the chunk's inverse norms per head. */
static double orc_chunk_score(orc_arr kr, int64_t c, orc_arr q, int64_t t, int hr, int d, const double* inv_q,
                              const double* inv_k) {
  double cos_sum = 0.0;
  for (int h = 0; h < hr; ++h) {
    double dot = orc_dot(q, ((size_t)t * hr + h) * d, kr, ((size_t)c * hr + h) * d, d);
    cos_sum += dot * inv_q[h] * inv_k[h];
  }
  return cos_sum / (double)hr; /* mean over heads */
}

/* [P2] Architecture: relevance is a cosine similarity averaged over the heads
 * and then maximised over query tokens; the top-k documents are selected. [P1] 核心方法: the
 * query is compared with every document's pooled routing keys.
 * Readings: the max runs over the sequence's query rows and the document's
 * chunks; each norm is clamped separately at eps; ties go to the lower id. */
static int orc_route_core(orc_arr kbar_r, const int64_t* doc_chunk_off, int64_t n_docs,
                          int hr, int d, orc_arr qr, const int32_t* q_seq_off, int n_seq,
                          double eps, int top_k, double* doc_scores, int32_t* top_ids, double* top_scores) {
  if (n_docs <= 0 || hr <= 0 || d <= 0 || n_seq <= 0 || top_k <= 0) return -1;
  for (int s = 0; s < n_seq; ++s)
    if (q_seq_off[s + 1] <= q_seq_off[s]) return -2; /* every sequence needs a row */
  int k = top_k < n_docs ? top_k : (int)n_docs;
  int64_t n_chunks = doc_chunk_off[n_docs], n_rows = q_seq_off[n_seq];
  orc_ranked* rank = (orc_ranked*)malloc(sizeof(orc_ranked) * (size_t)n_docs);
  double* inv_k = (double*)malloc(sizeof(double) * (size_t)(n_chunks > 0 ? n_chunks : 1) * hr);
  double* inv_q = (double*)malloc(sizeof(double) * (size_t)n_rows * hr);
  if (!rank || !inv_k || !inv_q) {
    free(rank); free(inv_k); free(inv_q);
    return -4;
  }
  orc_inv_norms(kbar_r, n_chunks, hr, d, eps, inv_k);
  orc_inv_norms(qr, n_rows, hr, d, eps, inv_q);
  for (int s = 0; s < n_seq; ++s) {
    for (int64_t j = 0; j < n_docs; ++j) {
      double best = -INFINITY;
      for (int64_t c = doc_chunk_off[j]; c < doc_chunk_off[j + 1]; ++c) {
        for (int64_t t = q_seq_off[s]; t < q_seq_off[s + 1]; ++t) {
          double sc = orc_chunk_score(kbar_r, c, qr, t, hr, d, inv_q + (size_t)t * hr, inv_k + (size_t)c * hr);
          if (sc > best) best = sc; /* max over rows and chunks */
        }
      }
      rank[j].score = best;
      rank[j].id = (int32_t)j;
      if (doc_scores) doc_scores[(size_t)s * n_docs + j] = best;
    }
    qsort(rank, (size_t)n_docs, sizeof(orc_ranked), orc_rank_cmp);
    for (int i = 0; i < k; ++i) {
      top_ids[(size_t)s * k + i] = rank[i].id;
      top_scores[(size_t)s * k + i] = rank[i].score;
    }
  }
  free(rank); free(inv_k); free(inv_q);
  return 0;
}

int orc_route(const uint16_t* kbar_r, const int64_t* doc_chunk_off, int64_t n_docs,
              int hr, int d, const uint16_t* qr, const int32_t* q_seq_off, int n_seq,
              double eps, int top_k, double* doc_scores, int32_t* top_ids, double* top_scores) {
  orc_arr k = {kbar_r, 0}, q = {qr, 0};
  return orc_route_core(k, doc_chunk_off, n_docs, hr, d, q, q_seq_off, n_seq, eps, top_k, doc_scores, top_ids,
                        top_scores);
}

int orc_route_f64(const double* kbar_r, const int64_t* doc_chunk_off, int64_t n_docs,
                  int hr, int d, const double* qr, const int32_t* q_seq_off, int n_seq,
                  double eps, int top_k, double* doc_scores, int32_t* top_ids, double* top_scores) {
  orc_arr k = {kbar_r, 1}, q = {qr, 1};
  return orc_route_core(k, doc_chunk_off, n_docs, hr, d, q, q_seq_off, n_seq, eps, top_k, doc_scores, top_ids,
                        top_scores);
}

/* Gradient of the routing scores (the contrastive routing loss needs it).
 * For each (sequence, document, dL/dscore) triple, the score is the head mean
 * of cosines at the (row, chunk) pair that attains the max (the first one in
 * chunk-major, row-minor order, as in the forward); its gradient flows there:
 *   d cos/dq = k invq invk - [|q| > eps] (q.k) invk invq^3 q, symmetric in k.
 * dqr [n_rows, hr, d] accumulates over triples (the caller zeroes it); dkr
 * [n_pairs, hr, d] is each triple's gradient for its argmax chunk, whose
 * index goes to argmax_chunk (-1 for a document without chunks). */
int orc_route_backward(const double* kbar_r, const int64_t* doc_chunk_off, int64_t n_docs, int hr, int d,
                       const double* qr, const int32_t* q_seq_off, int n_seq, double eps,
                       const int32_t* pair_seq, const int32_t* pair_doc, const double* pair_dscore, int n_pairs,
                       double* dqr, double* dkr, int64_t* argmax_chunk, int32_t* argmax_row) {
  if (n_docs <= 0 || hr <= 0 || d <= 0 || n_seq <= 0 || n_pairs < 0) return -1;
  orc_arr K = {kbar_r, 1}, Q = {qr, 1};
  double* iq_row = (double*)malloc(sizeof(double) * (size_t)hr);
  double* ik_row = (double*)malloc(sizeof(double) * (size_t)hr);
  if (!iq_row || !ik_row) {
    free(iq_row); free(ik_row);
    return -4;
  }
  for (int p = 0; p < n_pairs; ++p) {
    int s = pair_seq[p];
    int32_t j = pair_doc[p];
    if (s < 0 || s >= n_seq || j < 0 || j >= n_docs) {
      free(iq_row); free(ik_row);
      return -2;
    }
    double best = -INFINITY;
    int64_t cb = -1, tb = -1;
    for (int64_t c = doc_chunk_off[j]; c < doc_chunk_off[j + 1]; ++c)
      for (int64_t t = q_seq_off[s]; t < q_seq_off[s + 1]; ++t) {
        orc_inv_norms((orc_arr){(const double*)qr + (size_t)t * hr * d, 1}, 1, hr, d, eps, iq_row);
        orc_inv_norms((orc_arr){(const double*)kbar_r + (size_t)c * hr * d, 1}, 1, hr, d, eps, ik_row);
        double sc = orc_chunk_score(K, c, Q, t, hr, d, iq_row, ik_row);
        if (sc > best) { best = sc; cb = c; tb = t; }
      }
    argmax_chunk[p] = cb;
    argmax_row[p] = (int32_t)tb;
    double* gk = dkr + (size_t)p * hr * d;
    for (size_t i = 0; i < (size_t)hr * d; ++i) gk[i] = 0.0;
    if (cb < 0) continue;
    double g = pair_dscore[p] / (double)hr;
    for (int h = 0; h < hr; ++h) {
      const double* qv = qr + ((size_t)tb * hr + h) * d;
      const double* kv = kbar_r + ((size_t)cb * hr + h) * d;
      double nq = 0.0, nk = 0.0, dot = 0.0;
      for (int i = 0; i < d; ++i) { nq += qv[i] * qv[i]; nk += kv[i] * kv[i]; dot += qv[i] * kv[i]; }
      nq = sqrt(nq);
      nk = sqrt(nk);
      double iq = 1.0 / (nq > eps ? nq : eps), ik = 1.0 / (nk > eps ? nk : eps);
      double* dq = dqr + ((size_t)tb * hr + h) * d;
      for (int i = 0; i < d; ++i) {
        double gq = kv[i] * iq * ik - (nq > eps ? dot * ik * iq * iq * iq * qv[i] : 0.0);
        double gkk = qv[i] * iq * ik - (nk > eps ? dot * iq * ik * ik * ik * kv[i] : 0.0);
        dq[i] += g * gq;
        gk[(size_t)h * d + i] = g * gkk;
      }
    }
  }
  free(iq_row); free(ik_row);
  return 0;
}

/* ------------------------------------------------------------------ gather */

int64_t orc_gather(const int32_t* top_ids, int n_seq, int top_k, const int64_t* doc_chunk_off,
                   int64_t* sel_off, int64_t* sel_chunk, int64_t cap) {
  if (n_seq <= 0 || top_k <= 0) return -1;
  int64_t n = 0;
  sel_off[0] = 0;
  for (int s = 0; s < n_seq; ++s) {
    for (int i = 0; i < top_k; ++i) {
      int32_t doc = top_ids[(size_t)s * top_k + i];
      for (int64_t c = doc_chunk_off[doc]; c < doc_chunk_off[doc + 1]; ++c) {
        if (n >= cap) return -2;
        sel_chunk[n++] = c;
      }
    }
    sel_off[s + 1] = n;
  }
  return n;
}

/* ------------------------------------------------------------------ attend */

/* [P2] Architecture: the selected documents' pooled K/V are joined to the
 * K/V of the query's own recent context; global RoPE shifts the query by k,
 * keeping the order background -> query -> generation. Readings: every query
 * row sees every selected pooled key; local keys are causal (row g sees local
 * j <= g); q head h uses kv head h / (hq / hkv); logits are scaled by `scale`.
 *
 * With dout != NULL the same pass also computes the gradients (the chain rule
 * of the forward): D = dout.out; for every key j, ds_j = p_j (dout.v_j - D);
 * dq' = scale sum_j ds_j k'_j, dk'_j = scale ds_j q', dv_j = p_j dout, where
 * primes are rotated vectors; dq and dk_loc are rotated back (by the negative
 * angle), pooled memory keys are used as stored so dmem_k = dk'. */
static int orc_attend_core(orc_arr q, const int32_t* q_seq_off, const int32_t* q_start, int n_seq,
                           int hq, int hkv, int d, orc_arr k_loc, orc_arr v_loc, const int32_t* loc_off,
                           orc_arr mem_k, orc_arr mem_v, const int64_t* sel_off, const int64_t* sel_chunk,
                           double pos_offset, double rope_theta, double scale, double* out, double* lse,
                           const double* dout, double* dq, double* dk_loc, double* dv_loc, double* dmem_k,
                           double* dmem_v) {
  if (n_seq <= 0 || hq <= 0 || hkv <= 0 || hq % hkv || d <= 0 || (d & 1)) return -1;
  int group = hq / hkv;
  int64_t max_keys = 0;
  for (int s = 0; s < n_seq; ++s) {
    int64_t nk = (sel_off[s + 1] - sel_off[s]) + (loc_off[s + 1] - loc_off[s]);
    if (nk > max_keys) max_keys = nk;
  }
  size_t mk = (size_t)(max_keys > 0 ? max_keys : 1);
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  double* keys = (double*)malloc(sizeof(double) * mk * d); /* rotated keys of the row */
  double* logit = (double*)malloc(sizeof(double) * mk);
  int* vsrc = (int*)malloc(sizeof(int) * mk);               /* 0: memory row, 1: local row */
  size_t* voff = (size_t*)malloc(sizeof(size_t) * mk);      /* element offset of the value row */
  int64_t* gidx = (int64_t*)malloc(sizeof(int64_t) * mk);   /* sel position or local index */
  double* g = (double*)malloc(sizeof(double) * (size_t)d);
  if (!qv || !keys || !logit || !vsrc || !voff || !gidx || !g) {
    free(qv); free(keys); free(logit); free(vsrc); free(voff); free(gidx); free(g);
    return -4;
  }
  for (int s = 0; s < n_seq; ++s) {
    int64_t n_mem = sel_off[s + 1] - sel_off[s];
    int64_t n_loc = loc_off[s + 1] - loc_off[s];
    for (int32_t r = q_seq_off[s]; r < q_seq_off[s + 1]; ++r) {
      int64_t gq = (int64_t)q_start[s] + (r - q_seq_off[s]); /* active-context index */
      for (int h = 0; h < hq; ++h) {
        int kh = h / group;
        for (int i = 0; i < d; ++i) qv[i] = orc_ld(q, ((size_t)r * hq + h) * d + i);
        orc_rope(qv, d, pos_offset + (double)gq, rope_theta);
        int64_t n = 0;
        for (int64_t m = 0; m < n_mem; ++m) {
          int64_t c = sel_chunk[sel_off[s] + m];
          size_t ko = ((size_t)c * hkv + kh) * d;
          double dot = 0.0;
          for (int i = 0; i < d; ++i) {
            keys[(size_t)n * d + i] = orc_ld(mem_k, ko + i);
            dot += qv[i] * keys[(size_t)n * d + i];
          }
          logit[n] = dot * scale;
          vsrc[n] = 0;
          voff[n] = ko;
          gidx[n++] = sel_off[s] + m;
        }
        for (int64_t j = 0; j < n_loc && j <= gq; ++j) {
          size_t ko = ((size_t)(loc_off[s] + j) * hkv + kh) * d;
          double* kv = keys + (size_t)n * d;
          for (int i = 0; i < d; ++i) kv[i] = orc_ld(k_loc, ko + i);
          orc_rope(kv, d, pos_offset + (double)j, rope_theta);
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += qv[i] * kv[i];
          logit[n] = dot * scale;
          vsrc[n] = 1;
          voff[n] = ko;
          gidx[n++] = j;
        }
        double* o = out + ((size_t)r * hq + h) * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (n == 0) {
          lse[(size_t)r * hq + h] = -INFINITY;
          continue;
        }
        double mx = -INFINITY;
        for (int64_t j = 0; j < n; ++j)
          if (logit[j] > mx) mx = logit[j];
        double den = 0.0;
        for (int64_t j = 0; j < n; ++j) {
          double p = exp(logit[j] - mx);
          den += p;
          orc_arr vv = vsrc[j] ? v_loc : mem_v;
          for (int i = 0; i < d; ++i) o[i] += p * orc_ld(vv, voff[j] + i);
        }
        for (int i = 0; i < d; ++i) o[i] /= den;
        lse[(size_t)r * hq + h] = mx + log(den);
        if (!dout) continue;
        /* ---- gradients of this (row, head) */
        const double* go = dout + ((size_t)r * hq + h) * d;
        double D = 0.0;
        for (int i = 0; i < d; ++i) D += go[i] * o[i];
        for (int i = 0; i < d; ++i) g[i] = 0.0; /* dq' */
        for (int64_t j = 0; j < n; ++j) {
          double p = exp(logit[j] - mx) / den;
          orc_arr vv = vsrc[j] ? v_loc : mem_v;
          double dp = 0.0;
          for (int i = 0; i < d; ++i) dp += go[i] * orc_ld(vv, voff[j] + i);
          double ds = p * (dp - D);
          for (int i = 0; i < d; ++i) g[i] += scale * ds * keys[(size_t)j * d + i];
          double* dk = vsrc[j] ? dk_loc + ((size_t)(loc_off[s] + gidx[j]) * hkv + kh) * d
                                : dmem_k + ((size_t)gidx[j] * hkv + kh) * d;
          double* dv = vsrc[j] ? dv_loc + ((size_t)(loc_off[s] + gidx[j]) * hkv + kh) * d
                                : dmem_v + ((size_t)gidx[j] * hkv + kh) * d;
          if (vsrc[j]) {
            /* local key: the gradient w.r.t. the rotated key, rotated back */
            double* kv = keys + (size_t)j * d; /* reuse as scratch: it is no longer needed */
            for (int i = 0; i < d; ++i) kv[i] = scale * ds * qv[i];
            orc_rope(kv, d, -(pos_offset + (double)gidx[j]), rope_theta);
            for (int i = 0; i < d; ++i) dk[i] += kv[i];
          } else {
            for (int i = 0; i < d; ++i) dk[i] += scale * ds * qv[i];
          }
          for (int i = 0; i < d; ++i) dv[i] += p * go[i];
        }
        orc_rope(g, d, -(pos_offset + (double)gq), rope_theta);
        double* dqo = dq + ((size_t)r * hq + h) * d;
        for (int i = 0; i < d; ++i) dqo[i] = g[i];
      }
    }
  }
  free(qv); free(keys); free(logit); free(vsrc); free(voff); free(gidx); free(g);
  return 0;
}

int orc_attend(const uint16_t* q, const int32_t* q_seq_off, const int32_t* q_start, int n_seq,
               int hq, int hkv, int d,
               const uint16_t* k_loc, const uint16_t* v_loc, const int32_t* loc_off,
               const uint16_t* mem_k, const uint16_t* mem_v,
               const int64_t* sel_off, const int64_t* sel_chunk,
               double pos_offset, double rope_theta, double scale,
               double* out, double* lse) {
  orc_arr Q = {q, 0}, KL = {k_loc, 0}, VL = {v_loc, 0}, MK = {mem_k, 0}, MV = {mem_v, 0};
  return orc_attend_core(Q, q_seq_off, q_start, n_seq, hq, hkv, d, KL, VL, loc_off, MK, MV, sel_off, sel_chunk,
                         pos_offset, rope_theta, scale, out, lse, NULL, NULL, NULL, NULL, NULL, NULL);
}

/* fp64 inputs; with dout != NULL also the gradients (the caller zeroes
 * dk_loc, dv_loc, dmem_k, dmem_v; dmem rows are in selection order). */
int orc_attend_f64(const double* q, const int32_t* q_seq_off, const int32_t* q_start, int n_seq,
                   int hq, int hkv, int d,
                   const double* k_loc, const double* v_loc, const int32_t* loc_off,
                   const double* mem_k, const double* mem_v,
                   const int64_t* sel_off, const int64_t* sel_chunk,
                   double pos_offset, double rope_theta, double scale,
                   double* out, double* lse, const double* dout, double* dq, double* dk_loc, double* dv_loc,
                   double* dmem_k, double* dmem_v) {
  orc_arr Q = {q, 1}, KL = {k_loc, 1}, VL = {v_loc, 1}, MK = {mem_k, 1}, MV = {mem_v, 1};
  return orc_attend_core(Q, q_seq_off, q_start, n_seq, hq, hkv, d, KL, VL, loc_off, MK, MV, sel_off, sel_chunk,
                         pos_offset, rope_theta, scale, out, lse, dout, dq, dk_loc, dv_loc, dmem_k, dmem_v);
}
