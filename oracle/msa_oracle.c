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

static double orc_dot_bf16(const uint16_t* a, const uint16_t* b, int d) {
  double s = 0.0;
  for (int i = 0; i < d; ++i) s += orc_bf16_to_double(a[i]) * orc_bf16_to_double(b[i]);
  return s;
}

/* [P2] Architecture: relevance by cosine similarity, mean-pooled over heads,
 * then token-wise max; the top-k documents are selected. [P1] 核心方法: the
 * query is compared with every document's pooled routing keys.
 * Readings: the max runs over the sequence's query rows and the document's
 * chunks; each norm is clamped separately at eps; ties go to the lower id. */
int orc_route(const uint16_t* kbar_r, const int64_t* doc_chunk_off, int64_t n_docs,
              int hr, int d, const uint16_t* qr, const int32_t* q_seq_off, int n_seq,
              double eps, int top_k, double* doc_scores, int32_t* top_ids, double* top_scores) {
  if (n_docs <= 0 || hr <= 0 || d <= 0 || n_seq <= 0 || top_k <= 0) return -1;
  for (int s = 0; s < n_seq; ++s)
    if (q_seq_off[s + 1] <= q_seq_off[s]) return -2; /* every sequence needs a row */
  int64_t n_chunks = doc_chunk_off[n_docs];
  int64_t n_rows = q_seq_off[n_seq];
  int k = top_k < n_docs ? top_k : (int)n_docs;

  double* inv_k = (double*)malloc(sizeof(double) * (size_t)(n_chunks > 0 ? n_chunks : 1) * hr);
  double* inv_q = (double*)malloc(sizeof(double) * (size_t)n_rows * hr);
  orc_ranked* rank = (orc_ranked*)malloc(sizeof(orc_ranked) * (size_t)n_docs);
  if (!inv_k || !inv_q || !rank) {
    free(inv_k); free(inv_q); free(rank);
    return -4;
  }
  for (int64_t c = 0; c < n_chunks; ++c)
    for (int h = 0; h < hr; ++h) {
      const uint16_t* kv = kbar_r + ((size_t)c * hr + h) * d;
      double nrm = sqrt(orc_dot_bf16(kv, kv, d));
      inv_k[(size_t)c * hr + h] = 1.0 / (nrm > eps ? nrm : eps);
    }
  for (int64_t t = 0; t < n_rows; ++t)
    for (int h = 0; h < hr; ++h) {
      const uint16_t* qv = qr + ((size_t)t * hr + h) * d;
      double nrm = sqrt(orc_dot_bf16(qv, qv, d));
      inv_q[(size_t)t * hr + h] = 1.0 / (nrm > eps ? nrm : eps);
    }

  for (int s = 0; s < n_seq; ++s) {
    for (int64_t j = 0; j < n_docs; ++j) {
      double best = -INFINITY;
      for (int64_t c = doc_chunk_off[j]; c < doc_chunk_off[j + 1]; ++c) {
        for (int64_t t = q_seq_off[s]; t < q_seq_off[s + 1]; ++t) {
          double cos_sum = 0.0;
          for (int h = 0; h < hr; ++h) {
            double dot = orc_dot_bf16(qr + ((size_t)t * hr + h) * d,
                                      kbar_r + ((size_t)c * hr + h) * d, d);
            cos_sum += dot * inv_q[(size_t)t * hr + h] * inv_k[(size_t)c * hr + h];
          }
          double sc = cos_sum / (double)hr; /* mean over heads */
          if (sc > best) best = sc;         /* max over rows and chunks */
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
  free(inv_k); free(inv_q); free(rank);
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

/* [P2] Architecture: the selected documents' compressed K/V are concatenated
 * with the query's local K/V; global RoPE offsets the query's start index by k,
 * keeping the order background -> query -> generation. Readings: every query
 * row sees every selected pooled key; local keys are causal (row g sees local
 * j <= g); q head h uses kv head h / (hq / hkv); logits are scaled by `scale`. */
int orc_attend(const uint16_t* q, const int32_t* q_seq_off, const int32_t* q_start, int n_seq,
               int hq, int hkv, int d,
               const uint16_t* k_loc, const uint16_t* v_loc, const int32_t* loc_off,
               const uint16_t* mem_k, const uint16_t* mem_v,
               const int64_t* sel_off, const int64_t* sel_chunk,
               double pos_offset, double rope_theta, double scale,
               double* out, double* lse) {
  if (n_seq <= 0 || hq <= 0 || hkv <= 0 || hq % hkv || d <= 0 || (d & 1)) return -1;
  int group = hq / hkv;
  int64_t max_keys = 0;
  for (int s = 0; s < n_seq; ++s) {
    int64_t nk = (sel_off[s + 1] - sel_off[s]) + (loc_off[s + 1] - loc_off[s]);
    if (nk > max_keys) max_keys = nk;
  }
  double* qv = (double*)malloc(sizeof(double) * (size_t)d);
  double* kv = (double*)malloc(sizeof(double) * (size_t)d);
  double* logit = (double*)malloc(sizeof(double) * (size_t)(max_keys > 0 ? max_keys : 1));
  const uint16_t** vrow = (const uint16_t**)malloc(sizeof(uint16_t*) * (size_t)(max_keys > 0 ? max_keys : 1));
  if (!qv || !kv || !logit || !vrow) {
    free(qv); free(kv); free(logit); free(vrow);
    return -4;
  }
  for (int s = 0; s < n_seq; ++s) {
    int64_t n_mem = sel_off[s + 1] - sel_off[s];
    int64_t n_loc = loc_off[s + 1] - loc_off[s];
    for (int32_t r = q_seq_off[s]; r < q_seq_off[s + 1]; ++r) {
      int64_t g = (int64_t)q_start[s] + (r - q_seq_off[s]); /* active-context index */
      for (int h = 0; h < hq; ++h) {
        int kh = h / group;
        const uint16_t* qs = q + ((size_t)r * hq + h) * d;
        for (int i = 0; i < d; ++i) qv[i] = orc_bf16_to_double(qs[i]);
        orc_rope(qv, d, pos_offset + (double)g, rope_theta);
        int64_t n = 0;
        for (int64_t m = 0; m < n_mem; ++m) {
          int64_t c = sel_chunk[sel_off[s] + m];
          const uint16_t* ks = mem_k + ((size_t)c * hkv + kh) * d;
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += qv[i] * orc_bf16_to_double(ks[i]);
          logit[n] = dot * scale;
          vrow[n++] = mem_v + ((size_t)c * hkv + kh) * d;
        }
        for (int64_t j = 0; j < n_loc && j <= g; ++j) {
          const uint16_t* ks = k_loc + ((size_t)(loc_off[s] + j) * hkv + kh) * d;
          for (int i = 0; i < d; ++i) kv[i] = orc_bf16_to_double(ks[i]);
          orc_rope(kv, d, pos_offset + (double)j, rope_theta);
          double dot = 0.0;
          for (int i = 0; i < d; ++i) dot += qv[i] * kv[i];
          logit[n] = dot * scale;
          vrow[n++] = v_loc + ((size_t)(loc_off[s] + j) * hkv + kh) * d;
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
          for (int i = 0; i < d; ++i) o[i] += p * orc_bf16_to_double(vrow[j][i]);
        }
        for (int i = 0; i < d; ++i) o[i] /= den;
        lse[(size_t)r * hq + h] = mx + log(den);
      }
    }
  }
  free(qv); free(kv); free(logit); free(vrow);
  return 0;
}
