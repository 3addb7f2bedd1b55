/* msa.h — C ABI of the Memory Sparse Attention (MSA) routing + sparse
 * attention library for NVIDIA B200 (sm_100a).
 *
 * The library implements the per-layer hot path that the pages describe:
 *   msa_encode  offline: chunk-mean pooling of per-token K/V/K_r with
 *               document-wise RoPE on K, inverse norms of the pooled routing
 *               keys, the document -> chunk index.
 *               ["MSA: Memory Sparse Attention", Overall Design: Architecture,
 *               Inference Pipeline stage 1 (Global Memory Encoding);
 *               "MSA-arXiv26", 核心方法 (chunk-wise mean pool, Document-wise RoPE)]
 *   msa_route   online: cosine similarity of the query routing vectors with
 *               every pooled routing key, mean over heads, max over the
 *               sequence's rows and the document's chunks, top-k documents.
 *               ["MSA: Memory Sparse Attention", Overall Design: Architecture
 *               (head mean first, then the max over query tokens; Top-k);
 *               "MSA-arXiv26", 核心方法 (cosine similarity, top-k documents)]
 *   msa_gather  context assembly: the chunk list of the selected documents,
 *               and their pooled K/V fetched from pinned host memory when the
 *               content tier lives there.
 *               ["MSA: Memory Sparse Attention", Inference Pipeline stage 2
 *               (only the selected documents' pooled K/V are loaded) and the Memory Parallel
 *               paragraph (content K/V in host DRAM, fetched asynchronously);
 *               "MSA-arXiv26", 核心方法 / Memory Parallel inference (tiered storage)]
 *   msa_attend  sparse attention of every query row over the selected pooled
 *               K/V concatenated with its local K/V; query and local keys under
 *               global RoPE offset by k; GQA.
 *               ["MSA: Memory Sparse Attention", Overall Design: Architecture
 *               (concatenation with local K/V; Parallel and Global RoPE), Figure 2]
 *
 * Conventions
 *  - bfloat16 tensors are passed as uint16_t bit patterns. Row-major, the last
 *    dimension contiguous. d (head dimension) must be 128.
 *  - "device" pointers are CUDA device memory of the current device;
 *    "host" pointers are ordinary host memory; "pinned host" pointers come
 *    from cudaHostAlloc / cudaHostRegister (mapped).
 *  - `stream` arguments are cudaStream_t values passed as void*; NULL is the
 *    legacy default stream. All work is enqueued on that stream and the call
 *    returns without waiting, except where a function says otherwise.
 *  - The caller owns every buffer. The library allocates no device memory:
 *    functions that need scratch space report its size (msa_*_workspace) and
 *    take a caller-provided device buffer of at least that size.
 *  - Every function returns MSA_OK or an error code; on error nothing has
 *    been enqueued unless the code is MSA_ERR_CUDA. msa_last_error() returns
 *    a message for the calling thread's last failure. Errors raised by kernels
 *    after launch surface at the next CUDA synchronisation (msa_sync_check).
 *  - No C++ exception crosses this interface.
 *  - Several GPUs in one process are supported: every call works on the
 *    device current on the calling thread, and per-device kernel settings
 *    (shared-memory limits, msa_route_static's scratch address) are set up
 *    once per device on first use.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MSA_VERSION 1

typedef enum msa_status {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,  /* a pointer, size or shape is invalid */
  MSA_ERR_WORKSPACE = 2,    /* workspace missing or smaller than required */
  MSA_ERR_UNSUPPORTED = 3,  /* valid but not implemented (e.g. d != 128) */
  MSA_ERR_CUDA = 4,         /* a CUDA call failed; see msa_last_error() */
  MSA_ERR_TIMEOUT = 5,      /* a bounded host wait ran out */
  MSA_ERR_CAPACITY = 6      /* an output buffer is too small */
} msa_status;

/* Static string naming a status code. */
const char* msa_status_string(msa_status s);
/* Message of the calling thread's most recent failure ("" if none). */
const char* msa_last_error(void);
/* MSA_VERSION of the built library. */
int msa_version(void);

/* ------------------------------------------------------------------------
 * Memory bank of one routing layer.
 *
 * A bank holds n_docs documents split into n_chunks pooled chunks; document j
 * owns chunks doc_chunk_off[j] .. doc_chunk_off[j+1]-1 (a contiguous range;
 * documents with no tokens own none). Routing keys live in HBM; the content
 * K-bar/V-bar lives in HBM or, if content_on_host != 0, in pinned host memory.
 * ---------------------------------------------------------------------- */
typedef struct msa_bank_layer {
  int64_t n_docs;
  int64_t n_chunks;
  int32_t hr;              /* routing heads (query and key, one to one) */
  int32_t hkv;             /* key/value heads of the content */
  int32_t d;               /* head dimension; 128 */
  int32_t max_doc_chunks;  /* largest chunk count of any document (host-known) */
  const int64_t* doc_chunk_off;  /* device [n_docs + 1] */
  const int32_t* chunk_doc;      /* device [n_chunks]: owning document of each chunk */
  const uint16_t* kbar_r;        /* device [n_chunks, hr, d] bf16 pooled routing keys */
  const float* kr_inv_norm;      /* device [n_chunks, hr]: 1 / max(||kbar_r||, eps) */
  const uint16_t* kbar;          /* [n_chunks, hkv, d] bf16 pooled keys (RoPE'd at doc-local positions) */
  const uint16_t* vbar;          /* [n_chunks, hkv, d] bf16 pooled values */
  int32_t content_on_host;       /* 0: kbar/vbar are device memory; 1: pinned host memory */
  int32_t reserved;
} msa_bank_layer;

/* ------------------------------------------------------------------------
 * Encode (offline).
 *
 * Document j is tokens doc_tok_off[j] .. doc_tok_off[j+1]-1 of the per-token
 * arrays. For every token at document-local position p, K is rotated by RoPE
 * at position p (half-split pairs (i, i + d/2), angle p * rope_theta^(-2i/d));
 * with rope_mode = 1 the rotation is instead applied to each pooled chunk at
 * its chunk index within the document (the pages leave the order open).
 * Each document is cut into chunks of `chunk` tokens (the last may be
 * shorter; chunks never cross documents) and K, V, K_r are averaged over the
 * tokens of each chunk, in fp32, rounded to bf16 (nearest even). The inverse
 * norm of every pooled routing-key head is computed from the rounded values:
 * 1 / max(sqrt(sum x^2), eps). doc_chunk_off and chunk_doc are written.
 * ---------------------------------------------------------------------- */
typedef struct msa_encode_args {
  const uint16_t* k_tok;        /* device [n_tok, hkv, d] bf16 */
  const uint16_t* v_tok;        /* device [n_tok, hkv, d] bf16 */
  const uint16_t* kr_tok;       /* device [n_tok, hr, d] bf16 */
  const int64_t* doc_tok_off;   /* device [n_docs + 1], non-decreasing, [0] = 0, [n_docs] = n_tok */
  int64_t n_docs;
  int64_t n_tok;
  int64_t n_chunks;             /* from msa_encode_plan */
  int32_t hkv, hr, d, chunk;    /* d = 128; chunk in 1..1024 */
  float rope_theta;             /* RoPE base, > 1 */
  float eps;                    /* norm clamp, > 0 */
  uint16_t* kbar;               /* device out [n_chunks, hkv, d] */
  uint16_t* vbar;               /* device out [n_chunks, hkv, d] */
  uint16_t* kbar_r;             /* device out [n_chunks, hr, d] */
  float* kr_inv_norm;           /* device out [n_chunks, hr] */
  int64_t* doc_chunk_off;       /* device out [n_docs + 1] */
  int32_t* chunk_doc;           /* device out [n_chunks] */
  int32_t rope_mode;            /* 0: rotate each token at its document-local position, then pool
                                   (default reading); 1: pool, then rotate each pooled chunk at its
                                   chunk index within the document (alternative reading) */
  int32_t reserved;
} msa_encode_args;

/* Host-side planning: n_chunks = sum_j ceil(len_j / chunk) from a HOST copy
 * of the token offsets; optionally (doc_chunk_off_host != NULL) the document
 * -> chunk offsets [n_docs + 1] and (max_doc_chunks != NULL) the largest
 * per-document chunk count. Synchronous; touches no device. */
msa_status msa_encode_plan(const int64_t* doc_tok_off_host, int64_t n_docs, int32_t chunk,
                           int64_t* n_chunks_out, int64_t* doc_chunk_off_host,
                           int32_t* max_doc_chunks);

/* Enqueues the encode of one layer on `stream`. */
msa_status msa_encode(const msa_encode_args* args, void* stream);

/* Inverse norms 1 / max(||kbar_r[c, h]||, eps) of pooled routing keys that
 * were produced elsewhere (e.g. loaded from storage). kbar_r device
 * [n_chunks, hr, d] bf16 -> kr_inv_norm device [n_chunks, hr] fp32. */
msa_status msa_bank_norms(const uint16_t* kbar_r, int64_t n_chunks, int32_t hr, int32_t d,
                          float eps, float* kr_inv_norm, void* stream);

/* ------------------------------------------------------------------------
 * Route.
 *
 * Query routing rows qr [n_rows, hr, d] (device, bf16) are split into n_seq
 * sequences by the HOST array q_seq_off [n_seq + 1] (q_seq_off[0] = 0,
 * strictly increasing: every sequence has at least one row,
 * q_seq_off[n_seq] = n_rows). For sequence s and document j:
 *   score(s, j) = max over rows t of s and chunks c of j of
 *                 (1/hr) * sum_h cos(qr[t, h], kbar_r[c, h]),
 *   cos(a, b)   = a.b / (max(||a||, eps) * max(||b||, eps)),
 * and a document with no chunks scores -infinity. The top_k documents of each
 * sequence (top_k clamped to n_docs; call the clamped value k) are written in
 * order of decreasing score, equal scores by increasing document id:
 * top_ids [n_seq, k] int32 and top_scores [n_seq, k] fp32 (device).
 * all_doc_scores (device [n_seq, n_docs] fp32, or NULL) receives every score.
 * Limits: d = 128, top_k <= 4096. More than 256 sequences run as successive
 * groups of 256 on `stream` (each group streams the bank once); the
 * workspace is sized for one group.
 * How it runs (not part of the contract): with hr = 8 and up to 64 rows in a
 * call the scorer streams the bank once with all heads' accumulators in
 * tensor memory (bound by HBM bandwidth); above 64 rows it contracts the
 * heads in turn on the tensor cores (bound by tensor throughput); other head
 * counts use CUDA cores. All compute the same fp32 scores.
 * ---------------------------------------------------------------------- */
msa_status msa_route_workspace(const msa_bank_layer* bank, int32_t n_seq, int32_t n_rows,
                               int32_t top_k, size_t* bytes);

msa_status msa_route(const msa_bank_layer* bank, const uint16_t* qr, const int32_t* q_seq_off,
                     int32_t n_seq, int32_t n_rows, int32_t top_k, float eps,
                     int32_t* top_ids, float* top_scores, float* all_doc_scores,
                     void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Merge of per-shard top-k lists (Memory Parallel).
 *
 * ["MSA: Memory Sparse Attention", Inference Pipeline: Memory Parallel splits
 * the routing keys over GPUs, each scores the query against its part and the
 * results are combined; "MSA-arXiv26", 核心方法 / Memory Parallel inference]
 *
 * When the documents are split into n_shards contiguous ranges, each routed
 * by msa_route on its own bank (local document ids), shard g's lists
 * ids[g, s, :] / scores[g, s, :] (device, [n_shards, n_seq, k]) hold its
 * best k documents of sequence s; id_offset[g] (HOST) is the global id of its
 * first document. The merge writes the best k_out of all shards' candidates
 * (k_out <= n_shards * k) in the same order as msa_route on the whole bank
 * (score descending, then global id ascending), so the result is identical
 * to routing the unsharded bank. Entries with id < 0 are ignored.
 * Limits: n_shards <= 64, n_shards * k <= 4096.
 * ---------------------------------------------------------------------- */
msa_status msa_topk_merge(const int32_t* ids, const float* scores, const int64_t* id_offset,
                          int32_t n_shards, int32_t n_seq, int32_t k, int32_t k_out,
                          int32_t* top_ids, float* top_scores, void* stream);

/* ------------------------------------------------------------------------
 * Route without a workspace. The pages have no counterpart: this is an
 * interface addition of the library.
 *
 * For callers that cannot allocate device memory, such as a serving process
 * whose framework reserves all of HBM for its own pool and forbids further
 * cudaMalloc, or a latency-critical loop that cannot accept cudaMalloc's
 * implicit device-wide synchronisation. msa_route_static computes exactly what
 * msa_route computes, with the same arguments minus the workspace, and
 * allocates nothing. Its scratch is one fixed array of
 * MSA_ROUTE_STATIC_SCRATCH_BYTES in the library's device memory, which every
 * GPU that loads the library holds until the process exits.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current). Make that first call before any
 *    stream capture. The address is kept for the life of the process, so
 *    cudaDeviceReset between calls is not supported.
 *  - A call whose scratch need (msa_route_workspace) exceeds the array
 *    returns MSA_ERR_CAPACITY and enqueues nothing.
 *  - All calls on a device share the one array; it keeps the last call's
 *    contents, and every call first clears the part that must start at zero.
 *    Calls that overlap on the GPU (different streams, or different threads
 *    without ordering between them) race on the array and give wrong
 *    results; order them on one stream.
 * ---------------------------------------------------------------------- */
#define MSA_ROUTE_STATIC_SCRATCH_BYTES ((size_t)4 << 20) /* 4 MiB */

msa_status msa_route_static(const msa_bank_layer* bank, const uint16_t* qr, const int32_t* q_seq_off,
                            int32_t n_seq, int32_t n_rows, int32_t top_k, float eps,
                            int32_t* top_ids, float* top_scores, float* all_doc_scores, void* stream);

/* ------------------------------------------------------------------------
 * Gather (context assembly).
 *
 * For each sequence s, the chunks of its selected documents top_ids[s, :] are
 * listed in rank order: sel_chunk[sel_off[s] .. sel_off[s+1]) (device, int64
 * chunk ids). When the bank's content is in pinned host memory the pooled
 * K-bar/V-bar rows of those chunks are also copied, in the same order, into
 * stage_k/stage_v [cap, hkv, d] (device), so that msa_attend can read them
 * with sel_chunk = NULL.
 *
 * Modes for the host tier:
 *   MSA_GATHER_COPY_ENGINE: the call waits (bounded by timeout_us) for the
 *     selected ids on `stream`, copies them to top_ids_host, and issues one
 *     cudaMemcpyAsync per selected document for K-bar and for V-bar on
 *     copy_stream; it records done_event on copy_stream and makes `stream`
 *     wait for it. Needs doc_chunk_off_host and pinned top_ids_host.
 *   MSA_GATHER_DEVICE_PULL: a kernel on `stream` reads the rows straight from
 *     the mapped pinned host memory; nothing waits on the host.
 * cap must be >= n_seq * min(top_k, n_docs) * bank->max_doc_chunks.
 * Exception to the no-enqueue-on-error rule, copy-engine mode only: the ids
 * are known only after the wait, so MSA_ERR_TIMEOUT and an out-of-range id
 * (MSA_ERR_INVALID_ARG) leave the chunk listing and the copy of the ids
 * enqueued on `stream`; no K-bar/V-bar copy has been issued.
 * ---------------------------------------------------------------------- */
typedef enum msa_gather_mode {
  MSA_GATHER_COPY_ENGINE = 0,
  MSA_GATHER_DEVICE_PULL = 1
} msa_gather_mode;

typedef struct msa_gather_args {
  const msa_bank_layer* bank;
  const int32_t* top_ids;            /* device [n_seq, k] (k = min(top_k, n_docs)) */
  int32_t n_seq;
  int32_t top_k;
  int64_t* sel_off;                  /* device out [n_seq + 1] */
  int64_t* sel_chunk;                /* device out [cap] */
  int64_t cap;
  /* used only when bank->content_on_host */
  uint16_t* stage_k;                 /* device out [cap, hkv, d] */
  uint16_t* stage_v;                 /* device out [cap, hkv, d] */
  int32_t mode;                      /* msa_gather_mode */
  int32_t reserved;
  const int64_t* doc_chunk_off_host; /* host [n_docs + 1] (copy-engine mode) */
  int32_t* top_ids_host;             /* pinned host [n_seq * k] (copy-engine mode) */
  void* copy_stream;                 /* cudaStream_t for the copies (copy-engine mode) */
  void* done_event;                  /* cudaEvent_t recorded after the copies (copy-engine mode) */
  int64_t timeout_us;                /* bound on the host wait for the ids; <= 0: 10 s */
} msa_gather_args;

msa_status msa_gather(const msa_gather_args* args, void* stream);

/* ------------------------------------------------------------------------
 * Attend.
 *
 * Sequence s has query rows q_seq_off[s] .. q_seq_off[s+1]-1 (HOST offsets),
 * local keys/values loc_off[s] .. loc_off[s+1]-1 (HOST offsets) and memory
 * rows sel_off[s] .. sel_off[s+1]-1 (DEVICE offsets). Query row r of s has
 * active-context index g = q_start[s] + (r - q_seq_off[s]) (HOST q_start).
 * For q head h (kv head h / (hq / hkv)):
 *   q'   = RoPE(q[r, h], pos_offset + g)
 *   keys = memory rows (as stored: already rotated at their document-local
 *          positions)  followed by  RoPE(k_loc[j], pos_offset + j) for local
 *          j <= g
 *   out[r, h] = softmax(scale * q' . keys) @ values, lse[r, h] = log-sum-exp.
 * Memory row m of s is mem_k[sel_chunk[sel_off[s] + m]] (or, if sel_chunk is
 * NULL, mem_k[sel_off[s] + m], e.g. the staging buffer of msa_gather).
 * Routed form (sel_off = sel_chunk = NULL, top_ids set): the call lists the
 * memory rows itself, exactly as msa_gather would for device-resident content.
 * The memory rows of s are the chunks of documents top_ids[s * top_k + j],
 * j = 0 .. top_k - 1 in that order, each from doc_chunk_off[id] to
 * doc_chunk_off[id + 1] - 1 (rows of mem_k/mem_v: a bank's kbar/vbar in device
 * memory). top_ids is msa_route's output and doc_chunk_off the bank's, both on
 * the device. An id outside [0, n_docs) lists nothing. max_sel must be at
 * least every sequence's memory row count (top_k x the bank's max_doc_chunks
 * always is); with less, the call stays inside its buffers but its result is
 * unspecified. This form saves the msa_gather launch on the path route ->
 * attend; msa_attend_backward does not take it (MSA_ERR_UNSUPPORTED).
 * out is bf16 (nearest even of the fp32 result); out_f32 and lse are optional.
 * max_sel >= sel_off[s+1] - sel_off[s] for every s sizes the split-K grid.
 * Limits: d = 128, hq % hkv == 0, hq / hkv <= 16. More than 256 sequences
 * run as successive groups of 256 on `stream` with one workspace (sized for
 * the largest group); msa_attend_backward takes at most 256. q, k_loc,
 * v_loc, mem_k, mem_v, out and out_f32 must be 16-byte aligned and the
 * workspace 256-byte aligned (MSA_ERR_INVALID_ARG / MSA_ERR_WORKSPACE).
 * How it runs (not part of the contract): when a sequence's query vectors
 * (rows x hq / hkv) fill at least 64, the logits and P.V run on the tensor
 * cores (the logits at fp32 accuracy, P rounded to bf16) after a kernel that
 * rotates the queries and local keys; otherwise one decoding kernel rotates
 * its own rows, streams the key rows by cp.async and runs the logits and P.V
 * as warp-level MMAs, its key splits merged by log-sum-exp inside a
 * thread-block cluster.
 * ---------------------------------------------------------------------- */
typedef struct msa_attend_args {
  const uint16_t* q;          /* device [n_q, hq, d] bf16, not rotated */
  const int32_t* q_seq_off;   /* HOST [n_seq + 1] */
  const int32_t* q_start;     /* HOST [n_seq] */
  int32_t n_seq, n_q, hq, hkv, d;
  int32_t reserved;
  const uint16_t* k_loc;      /* device [n_loc, hkv, d] bf16, not rotated */
  const uint16_t* v_loc;      /* device [n_loc, hkv, d] bf16 */
  const int32_t* loc_off;     /* HOST [n_seq + 1] */
  const uint16_t* mem_k;      /* device (or mapped pinned host) [*, hkv, d] bf16 */
  const uint16_t* mem_v;
  const int64_t* sel_off;     /* device [n_seq + 1], or NULL for the routed form */
  const int64_t* sel_chunk;   /* device [*] or NULL */
  int64_t max_sel;
  float pos_offset;           /* global RoPE offset of the active context (the pages: k) */
  float rope_theta;
  float scale;                /* logit scale; <= 0 means 1/sqrt(d) */
  uint16_t* out;              /* device out [n_q, hq, d] bf16 */
  float* out_f32;             /* device out [n_q, hq, d] or NULL */
  float* lse;                 /* device out [n_q, hq] or NULL */
  /* routed form (used when top_ids != NULL; sel_off and sel_chunk must be NULL) */
  const int32_t* top_ids;     /* device [n_seq, top_k]: msa_route's top_ids */
  const int64_t* doc_chunk_off; /* device [n_docs + 1]: the bank's */
  int64_t n_docs;
  int32_t top_k;              /* 1 .. 4096 */
  int32_t reserved2;
} msa_attend_args;

msa_status msa_attend_workspace(const msa_attend_args* args, size_t* bytes);
msa_status msa_attend(const msa_attend_args* args, void* workspace, size_t workspace_bytes,
                      void* stream);

/* ------------------------------------------------------------------------
 * Gradients (training). The pages present top-k routing plus sparse attention
 * as one end-to-end differentiable operation trained with a generation loss
 * and a contrastive routing loss ["MSA: Memory Sparse Attention", Abstract,
 * Key Contributions; "MSA-arXiv26", 核心方法 (training)].
 *
 * msa_route_backward: for n_pairs (sequence, document, dL/dscore) triples
 * (device arrays pair_seq, pair_doc, pair_dscore), the gradient of
 * sum dscore * score(sequence, document). The score is a max over the
 * sequence's rows and the document's chunks, so the gradient flows through its
 * first argmax (row t*, chunk c*) in chunk-major, row-minor order:
 *   d/dq_h = (k invq invk - [|q| > eps] (q.k) invk invq^3 q) / hr, symmetric in k.
 * dqr [n_rows, hr, d] fp32 is ACCUMULATED (the caller zeroes it); dkr
 * [n_pairs, hr, d] fp32 receives each triple's gradient for its argmax chunk,
 * whose index goes to argmax_chunk [n_pairs] (-1 for a document without
 * chunks) and whose row to argmax_row [n_pairs]. q_seq_off is HOST memory.
 *
 * msa_attend_backward: gradients of msa_attend for dout [n_q, hq, d] fp32.
 * args is the forward's argument block with out_f32 and lse holding the
 * forward's results (both required). Outputs (fp32, device): dq [n_q, hq, d]
 * (w.r.t. the un-rotated queries), dk_loc and dv_loc [n_loc, hkv, d] (w.r.t.
 * the un-rotated local keys and values; zero for local keys no row sees),
 * dmem_k and dmem_v [sel_off[n_seq], hkv, d]: one row per selected memory
 * row in selection order (a chunk selected by several sequences gets one row
 * per selection; sum them to get the bank's gradient).
 * ---------------------------------------------------------------------- */
msa_status msa_route_backward(const msa_bank_layer* bank, const uint16_t* qr, const int32_t* q_seq_off,
                              int32_t n_seq, int32_t n_rows, float eps, const int32_t* pair_seq,
                              const int32_t* pair_doc, const float* pair_dscore, int32_t n_pairs,
                              float* dqr, float* dkr, int64_t* argmax_chunk, int32_t* argmax_row,
                              void* stream);

msa_status msa_attend_backward_workspace(const msa_attend_args* args, size_t* bytes);
msa_status msa_attend_backward(const msa_attend_args* args, const float* dout, float* dq, float* dk_loc,
                               float* dv_loc, float* dmem_k, float* dmem_v, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Waits for `stream` and reports any pending CUDA error as MSA_ERR_CUDA. */
msa_status msa_sync_check(void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H */
