/* CPU oracle for the Memory Sparse Attention (MSA) routing + sparse attention
 * step. TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; the library's own path never does.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Plain C, one thread, loops in the order of the definitions, every sum in
 * fp64. bfloat16 values travel as their 16-bit patterns (uint16_t).
 *
 * Sources (page title, section):
 *   [P1] "MSA-arXiv26" (paper digest), 核心方法 (architecture, Document-wise
 *        RoPE, Memory Parallel inference).
 *   [P2] "MSA: Memory Sparse Attention" (project README), Overall Design:
 *        Architecture and Figure 2; Inference Pipeline and Figure 3.
 * Readings of passages that leave a step open are listed beside each function.
 *
 * Every function returns 0 on success and a negative value on a bad argument.
 */
#ifndef MSA_ORACLE_H
#define MSA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* bfloat16 <-> double. The conversion to bfloat16 rounds to nearest, ties to
 * even, directly from the double (one rounding). */
double orc_bf16_to_double(uint16_t b);
uint16_t orc_double_to_bf16(double x);
void orc_bf16_array_to_double(const uint16_t* in, int64_t n, double* out);
void orc_double_array_to_bf16(const double* in, int64_t n, uint16_t* out);

/* Rotary position embedding of one d-vector (in place), half-split pairing:
 * the pair (x[i], x[i + d/2]) is rotated by the angle pos * theta^(-2i/d). */
int orc_rope(double* x, int d, double pos, double theta);

/* Offline encode of one routing layer ([P2] Inference Pipeline, stage 1;
 * [P1] 核心方法: chunk-wise mean pooling; [P2] Architecture: parallel RoPE).
 * Inputs per token t: k_tok/v_tok [n_tok, hkv, d], kr_tok [n_tok, hr, d];
 * documents are the token ranges doc_tok_off[j] .. doc_tok_off[j+1].
 * Outputs per pooled chunk c: kbar, vbar [C, hkv, d], kbar_r [C, hr, d]
 * (bfloat16), kr_inv_norm [C, hr], doc_chunk_off [n_docs + 1], chunk_doc [C].
 * C must equal sum_j ceil(len_j / chunk). */
int orc_encode(const uint16_t* k_tok, const uint16_t* v_tok, const uint16_t* kr_tok,
               const int64_t* doc_tok_off, int64_t n_docs, int hkv, int hr, int d, int chunk,
               double rope_theta, double eps, int rope_mode,
               uint16_t* kbar, uint16_t* vbar, uint16_t* kbar_r, double* kr_inv_norm,
               int64_t* doc_chunk_off, int32_t* chunk_doc, int64_t n_chunks);
/* rope_mode 0: each token of K rotated at its document-local position, then
 * pooled (the reading the library uses by default). rope_mode 1: K pooled
 * first, the pooled chunk rotated at its chunk index within the document (an
 * alternative reading of the same passage). */

/* Online routing of one layer ([P2] Architecture; [P1] 核心方法):
 * cosine similarity of every query routing vector with every pooled routing
 * key, mean over heads, max over the sequence's query rows and over the
 * document's chunks; then the top_k documents per sequence ordered by score
 * (descending), ties to the lower document id. top_k is clamped to n_docs.
 * qr [n_rows, hr, d]; q_seq_off [n_seq + 1] partitions the rows.
 * Outputs: doc_scores [n_seq, n_docs] (may be NULL), top_ids/top_scores
 * [n_seq, top_k]. A document with no chunks scores -infinity. */
int orc_route(const uint16_t* kbar_r, const int64_t* doc_chunk_off, int64_t n_docs,
              int hr, int d, const uint16_t* qr, const int32_t* q_seq_off, int n_seq,
              double eps, int top_k, double* doc_scores, int32_t* top_ids, double* top_scores);

/* Context assembly ([P2] Inference Pipeline, stage 2: load only the selected
 * pooled K/V): the chunks of each sequence's selected documents, in rank order.
 * sel_off [n_seq + 1]; sel_chunk [cap]. Returns the total count, or < 0. */
int64_t orc_gather(const int32_t* top_ids, int n_seq, int top_k, const int64_t* doc_chunk_off,
                   int64_t* sel_off, int64_t* sel_chunk, int64_t cap);

/* Sparse attention ([P2] Architecture and Figure 2; [P1] 核心方法): each query
 * row attends over its sequence's selected pooled keys concatenated with its
 * local keys up to and including its own position. The query row with
 * active-context index g is rotated at position pos_offset + g (global RoPE,
 * offset by k); local key j at pos_offset + j; pooled keys keep the
 * document-local rotation they got at encode time.
 * q [n_q, hq, d]; q_seq_off [n_seq + 1]; q_start [n_seq] = active index of each
 * sequence's first query row; k_loc/v_loc [n_loc, hkv, d] with loc_off
 * [n_seq + 1]; mem_k/mem_v [*, hkv, d] indexed by sel_chunk.
 * Outputs out [n_q, hq, d] and lse [n_q, hq] (natural log), fp64. */
int orc_attend(const uint16_t* q, const int32_t* q_seq_off, const int32_t* q_start, int n_seq,
               int hq, int hkv, int d,
               const uint16_t* k_loc, const uint16_t* v_loc, const int32_t* loc_off,
               const uint16_t* mem_k, const uint16_t* mem_v,
               const int64_t* sel_off, const int64_t* sel_chunk,
               double pos_offset, double rope_theta, double scale,
               double* out, double* lse);

/* fp64-input twins of orc_route and orc_attend (same arithmetic; used for
 * finite differences), and the gradients. orc_attend_f64 with dout != NULL
 * computes dq [n_q, hq, d], dk_loc/dv_loc [n_loc, hkv, d] and dmem_k/dmem_v
 * [n_sel, hkv, d] (selection order); the caller zeroes the accumulated ones.
 * orc_route_backward: for (sequence, document, dL/dscore) triples, the
 * gradient through the max's argmax (row, chunk) to dqr [n_rows, hr, d]
 * (accumulated; caller zeroes) and dkr [n_pairs, hr, d]. */
int orc_route_f64(const double* kbar_r, const int64_t* doc_chunk_off, int64_t n_docs,
                  int hr, int d, const double* qr, const int32_t* q_seq_off, int n_seq,
                  double eps, int top_k, double* doc_scores, int32_t* top_ids, double* top_scores);
int orc_route_backward(const double* kbar_r, const int64_t* doc_chunk_off, int64_t n_docs, int hr, int d,
                       const double* qr, const int32_t* q_seq_off, int n_seq, double eps,
                       const int32_t* pair_seq, const int32_t* pair_doc, const double* pair_dscore, int n_pairs,
                       double* dqr, double* dkr, int64_t* argmax_chunk, int32_t* argmax_row);
int orc_attend_f64(const double* q, const int32_t* q_seq_off, const int32_t* q_start, int n_seq,
                   int hq, int hkv, int d,
                   const double* k_loc, const double* v_loc, const int32_t* loc_off,
                   const double* mem_k, const double* mem_v,
                   const int64_t* sel_off, const int64_t* sel_chunk,
                   double pos_offset, double rope_theta, double scale,
                   double* out, double* lse, const double* dout, double* dq, double* dk_loc, double* dv_loc,
                   double* dmem_k, double* dmem_v);

#ifdef __cplusplus
}
#endif
#endif
