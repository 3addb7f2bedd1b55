// The C ABI: argument validation, workspace layout, launches.
// Declarations and the meaning of every argument: include/msa.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <chrono>
#include <thread>

#include "msa_internal.cuh"
#include "attend_params.cuh"

namespace msa {

namespace {
thread_local char g_err[512] = "";
int g_score_kernel = 0;  // 0 auto, 1 CUDA cores, 2 tensor cores, 3 tensor cores (many rows)
constexpr int kManyRows = 64;  // above this many query rows the many-row scorer is chosen
thread_local cudaEvent_t g_score_ev[2] = {nullptr, nullptr};
}  // namespace

std::atomic<long long> g_launches{0};

msa_status fail(msa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

msa_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_err, sizeof g_err, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
  return MSA_ERR_CUDA;
}

void record_debug_event(int which, cudaStream_t st) {
  cudaEvent_t ev = g_score_ev[which];
  if (!ev) return;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(st, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, st);
  if (which == 1) g_score_ev[0] = g_score_ev[1] = nullptr;
}

msa_status launch_check(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MSA_OK : cuda_fail(e, what);
}

namespace {

msa_status check_bank(const msa_bank_layer* b, bool need_content) {
  if (!b) return fail(MSA_ERR_INVALID_ARG, "bank is NULL");
  if (b->n_docs <= 0 || b->n_docs > 0x7FFFFFFE) return fail(MSA_ERR_INVALID_ARG, "bank: n_docs = %lld out of range", (long long)b->n_docs);
  if (b->n_chunks < 0) return fail(MSA_ERR_INVALID_ARG, "bank: n_chunks < 0");
  if (b->d != kHeadDim) return fail(MSA_ERR_UNSUPPORTED, "bank: d = %d (only 128 is supported)", b->d);
  if (b->hr <= 0 || b->hr > 16 || (b->hr & 1)) return fail(MSA_ERR_UNSUPPORTED, "bank: hr = %d (even, <= 16)", b->hr);
  if (!b->doc_chunk_off || !b->chunk_doc || !b->kbar_r || !b->kr_inv_norm)
    return fail(MSA_ERR_INVALID_ARG, "bank: routing arrays must be non-NULL");
  if (need_content) {
    if (b->hkv <= 0 || b->hkv > 16) return fail(MSA_ERR_UNSUPPORTED, "bank: hkv = %d", b->hkv);
    if (!b->kbar || !b->vbar) return fail(MSA_ERR_INVALID_ARG, "bank: content arrays must be non-NULL");
    if (b->max_doc_chunks < 0) return fail(MSA_ERR_INVALID_ARG, "bank: max_doc_chunks < 0");
  }
  return MSA_OK;
}

struct RouteLayout {
  size_t invq, invq_t, col_code, doc_key, topk, total;
  int n_rows_pad;
};

// Workspace of one route call: query scales (row-major and head-major), the
// per-row sequence codes, then (cleared before scoring) document keys and
// top-k state.
RouteLayout route_layout(const msa_bank_layer* b, int n_seq, int n_rows, int top_k) {
  RouteLayout L;
  int k = top_k < b->n_docs ? top_k : (int)b->n_docs;
  L.n_rows_pad = (n_rows + 3) & ~3;
  L.invq = 0;
  L.invq_t = align_up((size_t)n_rows * b->hr * sizeof(float), 256);
  L.col_code = L.invq_t + align_up((size_t)L.n_rows_pad * b->hr * sizeof(float), 256);
  L.doc_key = L.col_code + align_up((size_t)n_rows * sizeof(int32_t), 256);
  L.topk = L.doc_key + align_up((size_t)n_seq * b->n_docs * sizeof(uint32_t), 256);
  L.total = L.topk + topk_workspace(n_seq, b->n_docs, k);
  return L;
}

bool timed_out(std::chrono::steady_clock::time_point t0, int64_t limit_us) {
  return std::chrono::duration_cast<std::chrono::microseconds>(std::chrono::steady_clock::now() - t0).count() > limit_us;
}

}  // namespace
}  // namespace msa

using namespace msa;

extern "C" {

const char* msa_status_string(msa_status s) {
  switch (s) {
    case MSA_OK: return "MSA_OK";
    case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
    case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE";
    case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
    case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
    case MSA_ERR_TIMEOUT: return "MSA_ERR_TIMEOUT";
    case MSA_ERR_CAPACITY: return "MSA_ERR_CAPACITY";
  }
  return "MSA_ERR_UNKNOWN";
}

const char* msa_last_error(void) { return g_err; }

int msa_version(void) { return MSA_VERSION; }

// Selects the routing score kernel for later msa_route calls in this process:
// 0 = automatic, 1 = CUDA-core kernel, 2 = tensor-core kernel (per-head
// accumulators), 3 = tensor-core kernel for many rows. A testing and
// benchmarking control; not declared in msa.h.
int msa_debug_set_score_kernel(int which) {
  int old = g_score_kernel;
  if (which >= 0 && which <= 3) g_score_kernel = which;
  return old;
}

// Number of kernels this library has launched in the process (every launch
// goes through launch_check). Benchmark instrumentation.
long long msa_debug_launch_count(void) { return g_launches.load(); }

// The calling thread's next msa_route (or msa_encode) records `begin` and
// `end` (cudaEvent_t) on its stream immediately around its main kernel (the
// scoring kernel, or the pooling kernel), then forgets them. Under stream
// capture the records become external event nodes, so they fire on every
// replay. Benchmark instrumentation: it times that kernel inside a real step.
void msa_debug_score_events(void* begin, void* end) {
  g_score_ev[0] = (cudaEvent_t)begin;
  g_score_ev[1] = (cudaEvent_t)end;
}

// 1 if the tensor-core scoring kernel is compiled in. Testing control.
int msa_debug_tc_available(void) { return score_tc_built() ? 1 : 0; }

// ------------------------------------------------------------------ encode

msa_status msa_encode_plan(const int64_t* off, int64_t n_docs, int32_t chunk, int64_t* n_chunks_out,
                           int64_t* doc_chunk_off_host, int32_t* max_doc_chunks) {
  if (!off || n_docs <= 0 || !n_chunks_out) return fail(MSA_ERR_INVALID_ARG, "encode_plan: NULL or empty input");
  if (chunk <= 0 || chunk > 1024) return fail(MSA_ERR_INVALID_ARG, "encode_plan: chunk = %d", chunk);
  if (off[0] != 0) return fail(MSA_ERR_INVALID_ARG, "encode_plan: doc_tok_off[0] must be 0");
  int64_t total = 0, mx = 0;
  if (doc_chunk_off_host) doc_chunk_off_host[0] = 0;
  for (int64_t j = 0; j < n_docs; ++j) {
    int64_t len = off[j + 1] - off[j];
    if (len < 0) return fail(MSA_ERR_INVALID_ARG, "encode_plan: doc_tok_off decreases at %lld", (long long)j);
    int64_t c = (len + chunk - 1) / chunk;
    total += c;
    if (c > mx) mx = c;
    if (doc_chunk_off_host) doc_chunk_off_host[j + 1] = total;
  }
  *n_chunks_out = total;
  if (max_doc_chunks) *max_doc_chunks = (int32_t)mx;
  return MSA_OK;
}

msa_status msa_encode(const msa_encode_args* a, void* stream) {
  if (!a) return fail(MSA_ERR_INVALID_ARG, "encode: args is NULL");
  if (a->d != kHeadDim) return fail(MSA_ERR_UNSUPPORTED, "encode: d = %d (only 128)", a->d);
  if (a->hkv <= 0 || a->hkv > 16 || a->hr <= 0 || a->hr > 16)
    return fail(MSA_ERR_UNSUPPORTED, "encode: hkv = %d, hr = %d (1..16)", a->hkv, a->hr);
  if (a->chunk <= 0 || a->chunk > 1024) return fail(MSA_ERR_INVALID_ARG, "encode: chunk = %d", a->chunk);
  if (a->n_docs <= 0 || a->n_tok < 0 || a->n_chunks < 0) return fail(MSA_ERR_INVALID_ARG, "encode: bad sizes");
  if (!(a->rope_theta > 1.0f) || !(a->eps > 0.0f)) return fail(MSA_ERR_INVALID_ARG, "encode: rope_theta > 1 and eps > 0 required");
  if (!a->doc_tok_off || !a->doc_chunk_off) return fail(MSA_ERR_INVALID_ARG, "encode: NULL offsets");
  if (a->rope_mode != 0 && a->rope_mode != 1) return fail(MSA_ERR_INVALID_ARG, "encode: rope_mode = %d", a->rope_mode);
  if (a->n_chunks > 0 && (!a->k_tok || !a->v_tok || !a->kr_tok || !a->kbar || !a->vbar || !a->kbar_r ||
                          !a->kr_inv_norm || !a->chunk_doc))
    return fail(MSA_ERR_INVALID_ARG, "encode: NULL tensor");
  return launch_encode(*a, (cudaStream_t)stream);
}

msa_status msa_bank_norms(const uint16_t* kbar_r, int64_t n_chunks, int32_t hr, int32_t d, float eps,
                          float* inv_norm, void* stream) {
  if (d != kHeadDim) return fail(MSA_ERR_UNSUPPORTED, "bank_norms: d = %d", d);
  if (hr <= 0 || hr > 16 || n_chunks < 0 || !(eps > 0.f)) return fail(MSA_ERR_INVALID_ARG, "bank_norms: bad sizes");
  if (n_chunks > 0 && (!kbar_r || !inv_norm)) return fail(MSA_ERR_INVALID_ARG, "bank_norms: NULL tensor");
  return launch_bank_norms(kbar_r, n_chunks, hr, eps, inv_norm, (cudaStream_t)stream);
}

// ------------------------------------------------------------------- route

msa_status msa_route_workspace(const msa_bank_layer* b, int32_t n_seq, int32_t n_rows, int32_t top_k,
                               size_t* bytes) {
  msa_status s = check_bank(b, false);
  if (s != MSA_OK) return s;
  if (!bytes || n_seq <= 0 || n_rows < n_seq || top_k <= 0)
    return fail(MSA_ERR_INVALID_ARG, "route_workspace: bad sizes");
  if ((top_k < b->n_docs ? top_k : b->n_docs) > 4096)
    return fail(MSA_ERR_UNSUPPORTED, "route_workspace: min(top_k, n_docs) > 4096");
  *bytes = route_layout(b, n_seq < kMaxSeq ? n_seq : kMaxSeq, n_rows, top_k).total;
  return MSA_OK;
}

namespace msa {
namespace {

// The routing kernels over one group of at most kMaxSeq sequences: q_seq_off
// rebased to the group's first row, outputs already offset to its first
// sequence; the workspace is laid out for kMaxSeq sequences (or fewer) and
// the call's whole row count, so every group fits it.
msa_status route_group(const msa_bank_layer* b, const uint16_t* qr, const int32_t* q_seq_off, int n_seq, int n_rows,
                       int top_k, float eps, int32_t* top_ids, float* top_scores, float* all_doc_scores, char* w,
                       const RouteLayout& L, cudaStream_t st) {
  RoutePlan p;
  p.qr = qr; p.kr_inv_norm = b->kr_inv_norm; p.chunk_doc = b->chunk_doc; p.kbar_r = b->kbar_r;
  p.n_chunks = b->n_chunks; p.n_docs = b->n_docs; p.hr = b->hr; p.n_rows = n_rows; p.n_seq = n_seq;
  for (int i = 0; i <= n_seq; ++i) p.q_seq_off[i] = q_seq_off[i];
  p.invq = reinterpret_cast<float*>(w + L.invq);
  p.invq_t = reinterpret_cast<float*>(w + L.invq_t);
  p.col_code = reinterpret_cast<int32_t*>(w + L.col_code);
  p.n_rows_pad = L.n_rows_pad;
  p.doc_key = reinterpret_cast<uint32_t*>(w + L.doc_key);
  p.zero = w + L.doc_key;
  p.zero_bytes = L.total - L.doc_key;  // a multiple of 256
  // automatic: many rows -> heads in turn with the scales in the epilogue
  // (score_pf.cu), a few -> all heads' accumulators at once (score_tc.cu),
  // other head counts -> CUDA cores
  int which = g_score_kernel;
  if (which == 0)
    which = score_pf_supported(p) && n_rows > kManyRows ? 3 : score_tc_supported(p) ? 2 : 1;
  msa_status s = launch_qprep(p, eps, st);
  if (s != MSA_OK) return s;
  if (b->n_chunks > 0) {
    record_debug_event(0, st);
    s = which == 3 ? launch_score_pf(p, st) : which == 2 ? launch_score_tc(p, st) : launch_score_simt(p, st);
    record_debug_event(1, st);
    if (s != MSA_OK) return s;
  }
  int k = top_k < b->n_docs ? top_k : (int)b->n_docs;
  return launch_topk(p.doc_key, n_seq, b->n_docs, k, top_ids, top_scores, all_doc_scores, w + L.topk, st);
}

}  // namespace
}  // namespace msa

msa_status msa_route(const msa_bank_layer* b, const uint16_t* qr, const int32_t* q_seq_off, int32_t n_seq,
                     int32_t n_rows, int32_t top_k, float eps, int32_t* top_ids, float* top_scores,
                     float* all_doc_scores, void* ws, size_t ws_bytes, void* stream) {
  msa_status s = check_bank(b, false);
  if (s != MSA_OK) return s;
  if (n_seq <= 0) return fail(MSA_ERR_UNSUPPORTED, "route: n_seq = %d (1..)", n_seq);
  if (top_k <= 0) return fail(MSA_ERR_INVALID_ARG, "route: top_k = %d", top_k);
  if ((top_k < b->n_docs ? top_k : b->n_docs) > 4096)
    return fail(MSA_ERR_UNSUPPORTED, "route: min(top_k, n_docs) = %lld > 4096",
                (long long)(top_k < b->n_docs ? top_k : b->n_docs));
  if (!qr || !q_seq_off || !top_ids || !top_scores) return fail(MSA_ERR_INVALID_ARG, "route: NULL pointer");
  if (!(eps > 0.f)) return fail(MSA_ERR_INVALID_ARG, "route: eps must be > 0");
  if (q_seq_off[0] != 0 || q_seq_off[n_seq] != n_rows)
    return fail(MSA_ERR_INVALID_ARG, "route: q_seq_off must start at 0 and end at n_rows");
  for (int i = 0; i < n_seq; ++i)
    if (q_seq_off[i + 1] <= q_seq_off[i])
      return fail(MSA_ERR_INVALID_ARG, "route: sequence %d has no query rows", i);
  const int group = n_seq < kMaxSeq ? n_seq : kMaxSeq;
  RouteLayout L = route_layout(b, group, n_rows, top_k);
  if (!ws || ws_bytes < L.total)
    return fail(MSA_ERR_WORKSPACE, "route: workspace %zu B, need %zu B", ws_bytes, L.total);
  {
    RoutePlan probe;
    probe.qr = qr; probe.kbar_r = b->kbar_r; probe.hr = b->hr; probe.n_chunks = b->n_chunks;
    const int which = g_score_kernel;
    if (b->n_chunks > 0 && ((which == 2 && !score_tc_supported(probe)) || (which == 3 && !score_pf_supported(probe))))
      return fail(MSA_ERR_UNSUPPORTED, "route: tensor-core scoring needs hr = 8");
  }
  cudaStream_t st = (cudaStream_t)stream;
  char* w = reinterpret_cast<char*>(ws);
  const int k = top_k < b->n_docs ? top_k : (int)b->n_docs;
  // more than kMaxSeq sequences: one pass of the kernels per group of kMaxSeq, in order on the
  // stream (each group streams the bank once)
  int32_t qso[kMaxSeq + 1];
  for (int s0 = 0; s0 < n_seq; s0 += kMaxSeq) {
    const int gs = n_seq - s0 < kMaxSeq ? n_seq - s0 : kMaxSeq;
    for (int i = 0; i <= gs; ++i) qso[i] = q_seq_off[s0 + i] - q_seq_off[s0];
    s = route_group(b, qr + (size_t)q_seq_off[s0] * b->hr * kHeadDim, qso, gs, qso[gs], top_k, eps,
                    top_ids + (size_t)s0 * k, top_scores + (size_t)s0 * k,
                    all_doc_scores ? all_doc_scores + (size_t)s0 * b->n_docs : nullptr, w, L, st);
    if (s != MSA_OK) return s;
  }
  return MSA_OK;
}

msa_status msa_topk_merge(const int32_t* ids, const float* scores, const int64_t* id_offset, int32_t n_shards,
                          int32_t n_seq, int32_t k, int32_t k_out, int32_t* top_ids, float* top_scores,
                          void* stream) {
  if (!ids || !scores || !id_offset || !top_ids || !top_scores) return fail(MSA_ERR_INVALID_ARG, "topk_merge: NULL pointer");
  if (n_seq <= 0 || n_seq > 65535 || k <= 0 || k_out <= 0 || k_out > n_shards * k)
    return fail(MSA_ERR_INVALID_ARG, "topk_merge: bad sizes");
  if ((int64_t)n_shards * k > 4096) return fail(MSA_ERR_UNSUPPORTED, "topk_merge: n_shards * k > 4096");
  for (int g = 0; g < n_shards && g < 64; ++g)
    if (id_offset[g] < 0 || id_offset[g] > 0x7FFFFFFF) return fail(MSA_ERR_INVALID_ARG, "topk_merge: id_offset[%d]", g);
  return launch_topk_merge(ids, scores, id_offset, n_shards, n_seq, k, k_out, top_ids, top_scores,
                           (cudaStream_t)stream);
}

// ------------------------------------------------------------------ gather

msa_status msa_gather(const msa_gather_args* a, void* stream) {
  if (!a) return fail(MSA_ERR_INVALID_ARG, "gather: args is NULL");
  msa_status s = check_bank(a->bank, true);
  if (s != MSA_OK) return s;
  const msa_bank_layer& b = *a->bank;
  if (a->n_seq <= 0 || a->top_k <= 0) return fail(MSA_ERR_INVALID_ARG, "gather: bad sizes");
  if (!a->top_ids || !a->sel_off || !a->sel_chunk) return fail(MSA_ERR_INVALID_ARG, "gather: NULL pointer");
  const int k = a->top_k < b.n_docs ? a->top_k : (int)b.n_docs;
  const int64_t need = (int64_t)a->n_seq * k * b.max_doc_chunks;
  if (a->cap < need)
    return fail(MSA_ERR_CAPACITY, "gather: cap = %lld < n_seq * k * max_doc_chunks = %lld", (long long)a->cap,
                (long long)need);
  if (b.content_on_host) {  // checked before anything is enqueued
    if (!a->stage_k || !a->stage_v) return fail(MSA_ERR_INVALID_ARG, "gather: staging buffers required for host content");
    if (a->mode != MSA_GATHER_DEVICE_PULL && a->mode != MSA_GATHER_COPY_ENGINE)
      return fail(MSA_ERR_INVALID_ARG, "gather: unknown mode %d", a->mode);
    if (a->mode == MSA_GATHER_COPY_ENGINE &&
        (!a->doc_chunk_off_host || !a->top_ids_host || !a->copy_stream || !a->done_event))
      return fail(MSA_ERR_INVALID_ARG, "gather: copy-engine mode needs doc_chunk_off_host, top_ids_host, copy_stream, done_event");
  }
  cudaStream_t st = (cudaStream_t)stream;
  s = launch_gather_index(b.doc_chunk_off, b.n_docs, a->top_ids, a->n_seq, k, a->sel_off, a->sel_chunk, a->cap, st);
  if (s != MSA_OK || !b.content_on_host) return s;
  if (a->mode == MSA_GATHER_DEVICE_PULL) {
    // The kernel reads the pinned host rows through their device-side mapping.
    msa_bank_layer mapped = b;
    void* dk = nullptr;
    void* dv = nullptr;
    cudaError_t e = cudaHostGetDevicePointer(&dk, const_cast<uint16_t*>(b.kbar), 0);
    if (e == cudaSuccess) e = cudaHostGetDevicePointer(&dv, const_cast<uint16_t*>(b.vbar), 0);
    if (e != cudaSuccess) return cuda_fail(e, "gather: host content is not mapped pinned memory");
    mapped.kbar = static_cast<const uint16_t*>(dk);
    mapped.vbar = static_cast<const uint16_t*>(dv);
    return launch_gather_pull(mapped, a->sel_off + a->n_seq, a->sel_chunk, a->cap, a->stage_k, a->stage_v, st);
  }
  const size_t ids_bytes = (size_t)a->n_seq * k * sizeof(int32_t);
  cudaError_t e = cudaMemcpyAsync(a->top_ids_host, a->top_ids, ids_bytes, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "gather: copy ids to host");
  // Bounded wait for the ids (and everything before them on `stream`).
  const int64_t limit = a->timeout_us > 0 ? a->timeout_us : 10000000;
  auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    e = cudaStreamQuery(st);
    if (e == cudaSuccess) break;
    if (e != cudaErrorNotReady) return cuda_fail(e, "gather: wait for ids");
    if (timed_out(t0, limit)) return fail(MSA_ERR_TIMEOUT, "gather: ids not ready after %lld us", (long long)limit);
    std::this_thread::yield();
  }
  for (int i = 0; i < a->n_seq * k; ++i)  // every id checked before the first copy is issued
    if (a->top_ids_host[i] < 0 || a->top_ids_host[i] >= b.n_docs)
      return fail(MSA_ERR_INVALID_ARG, "gather: document id %d out of range", a->top_ids_host[i]);
  cudaStream_t cs = (cudaStream_t)a->copy_stream;
  const size_t row = (size_t)b.hkv * kHeadDim;
  int64_t dst = 0;
  for (int i = 0; i < a->n_seq * k; ++i) {
    const int32_t doc = a->top_ids_host[i];
    int64_t c0 = a->doc_chunk_off_host[doc], c1 = a->doc_chunk_off_host[doc + 1];
    // merge with following ranks whose chunks continue this range
    while (i + 1 < a->n_seq * k && c1 == a->doc_chunk_off_host[a->top_ids_host[i + 1]] &&
           (i + 1) % k != 0) {
      ++i;
      c1 = a->doc_chunk_off_host[a->top_ids_host[i] + 1];
    }
    const int64_t n = c1 - c0;
    if (n <= 0) continue;
    e = cudaMemcpyAsync(a->stage_k + dst * row, b.kbar + c0 * row, n * row * 2, cudaMemcpyHostToDevice, cs);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(a->stage_v + dst * row, b.vbar + c0 * row, n * row * 2, cudaMemcpyHostToDevice, cs);
    if (e != cudaSuccess) return cuda_fail(e, "gather: host-to-device copy");
    dst += n;
  }
  e = cudaEventRecord((cudaEvent_t)a->done_event, cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, (cudaEvent_t)a->done_event, 0);
  if (e != cudaSuccess) return cuda_fail(e, "gather: copy completion event");
  return MSA_OK;
}

// ------------------------------------------------------------------ attend

static msa_status check_attend(const msa_attend_args* a) {
  if (!a) return fail(MSA_ERR_INVALID_ARG, "attend: args is NULL");
  if (a->d != kHeadDim) return fail(MSA_ERR_UNSUPPORTED, "attend: d = %d (only 128)", a->d);
  if (a->hkv <= 0 || a->hq <= 0 || a->hq % a->hkv) return fail(MSA_ERR_INVALID_ARG, "attend: hq must be a multiple of hkv");
  const int g = a->hq / a->hkv;
  if (g > 16 || (g & (g - 1))) return fail(MSA_ERR_UNSUPPORTED, "attend: hq / hkv = %d (1, 2, 4, 8 or 16)", g);
  if (a->n_seq <= 0) return fail(MSA_ERR_UNSUPPORTED, "attend: n_seq = %d (1..)", a->n_seq);
  if (!a->q || !a->q_seq_off || !a->q_start || !a->loc_off || !a->out)
    return fail(MSA_ERR_INVALID_ARG, "attend: NULL pointer");
  if (!a->sel_off == !a->top_ids)
    return fail(MSA_ERR_INVALID_ARG, "attend: give exactly one of sel_off (a gather listing) and top_ids (routed)");
  if (a->top_ids) {
    if (a->sel_chunk) return fail(MSA_ERR_INVALID_ARG, "attend: routed form takes no sel_chunk");
    if (!a->doc_chunk_off) return fail(MSA_ERR_INVALID_ARG, "attend: routed form needs doc_chunk_off");
    if (a->top_k <= 0 || a->top_k > 4096) return fail(MSA_ERR_INVALID_ARG, "attend: top_k = %d (1..4096)", a->top_k);
    if (a->n_docs < 0) return fail(MSA_ERR_INVALID_ARG, "attend: n_docs < 0");
  }
  if (a->q_seq_off[0] != 0 || a->q_seq_off[a->n_seq] != a->n_q)
    return fail(MSA_ERR_INVALID_ARG, "attend: q_seq_off must start at 0 and end at n_q");
  if (a->loc_off[0] != 0) return fail(MSA_ERR_INVALID_ARG, "attend: loc_off[0] must be 0");
  for (int s = 0; s < a->n_seq; ++s) {
    if (a->q_seq_off[s + 1] < a->q_seq_off[s] || a->loc_off[s + 1] < a->loc_off[s])
      return fail(MSA_ERR_INVALID_ARG, "attend: offsets decrease at sequence %d", s);
    if (a->q_start[s] < 0) return fail(MSA_ERR_INVALID_ARG, "attend: q_start[%d] < 0", s);
  }
  if (a->loc_off[a->n_seq] > 0 && (!a->k_loc || !a->v_loc)) return fail(MSA_ERR_INVALID_ARG, "attend: NULL local K/V");
  if (a->max_sel < 0) return fail(MSA_ERR_INVALID_ARG, "attend: max_sel < 0");
  if (a->max_sel > 0 && (!a->mem_k || !a->mem_v)) return fail(MSA_ERR_INVALID_ARG, "attend: NULL memory K/V");
  if (!(a->rope_theta > 1.0f)) return fail(MSA_ERR_INVALID_ARG, "attend: rope_theta must be > 1");
  // the kernels move rows in 16-byte pieces
  const void* rows[] = {a->q, a->k_loc, a->v_loc, a->mem_k, a->mem_v, a->out, a->out_f32};
  for (const void* r : rows)
    if (reinterpret_cast<uintptr_t>(r) & 15) return fail(MSA_ERR_INVALID_ARG, "attend: row arrays must be 16-byte aligned");
  return MSA_OK;
}

namespace {

// The sequences s0 .. s1 - 1 of an attention call (at most kMaxSeq) as a call
// of their own: host offsets rebased, device row arrays and outputs offset to
// the group's first row, local key and sequence.
struct AttendGroup {
  msa_attend_args a;
  int32_t qso[kMaxSeq + 1], qst[kMaxSeq], lo[kMaxSeq + 1];
};

void attend_group(const msa_attend_args& a, int s0, int s1, AttendGroup& g) {
  g.a = a;
  const int row0 = a.q_seq_off[s0], loc0 = a.loc_off[s0], n = s1 - s0;
  for (int i = 0; i <= n; ++i) {
    g.qso[i] = a.q_seq_off[s0 + i] - row0;
    g.lo[i] = a.loc_off[s0 + i] - loc0;
    if (i < n) g.qst[i] = a.q_start[s0 + i];
  }
  const size_t qrow = (size_t)a.hq * kHeadDim, krow = (size_t)a.hkv * kHeadDim;
  g.a.n_seq = n;
  g.a.n_q = g.qso[n];
  g.a.q_seq_off = g.qso;
  g.a.q_start = g.qst;
  g.a.loc_off = g.lo;
  g.a.q = a.q + row0 * qrow;
  g.a.out = a.out + row0 * qrow;
  if (a.out_f32) g.a.out_f32 = a.out_f32 + row0 * qrow;
  if (a.lse) g.a.lse = a.lse + (size_t)row0 * a.hq;
  if (a.k_loc) g.a.k_loc = a.k_loc + loc0 * krow;
  if (a.v_loc) g.a.v_loc = a.v_loc + loc0 * krow;
  if (a.sel_off) g.a.sel_off = a.sel_off + s0;  // absolute positions in sel_chunk: unchanged
  if (a.top_ids) g.a.top_ids = a.top_ids + (size_t)s0 * a.top_k;
}

// More than kMaxSeq sequences: groups of kMaxSeq, run in order on the stream
// with one workspace, sized for the largest group's need.
size_t attend_workspace_all(const msa_attend_args& a) {
  if (a.n_seq <= kMaxSeq) return attend_workspace(a, nullptr);
  size_t need = 0;
  AttendGroup g;
  for (int s0 = 0; s0 < a.n_seq; s0 += kMaxSeq) {
    attend_group(a, s0, std::min(a.n_seq, s0 + kMaxSeq), g);
    need = std::max(need, attend_workspace(g.a, nullptr));
  }
  return need;
}

}  // namespace

msa_status msa_attend_workspace(const msa_attend_args* a, size_t* bytes) {
  msa_status s = check_attend(a);
  if (s != MSA_OK) return s;
  if (!bytes) return fail(MSA_ERR_INVALID_ARG, "attend_workspace: bytes is NULL");
  *bytes = attend_workspace_all(*a);
  return MSA_OK;
}

msa_status msa_attend(const msa_attend_args* a, void* ws, size_t ws_bytes, void* stream) {
  msa_status s = check_attend(a);
  if (s != MSA_OK) return s;
  size_t need = attend_workspace_all(*a);
  if (!ws || ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "attend: workspace %zu B, need %zu B", ws_bytes, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(MSA_ERR_WORKSPACE, "attend: workspace must be 256-byte aligned");
  if (a->n_q == 0) return MSA_OK;
  if (a->n_seq <= kMaxSeq) return launch_attend(*a, ws, (cudaStream_t)stream);
  AttendGroup g;
  for (int s0 = 0; s0 < a->n_seq; s0 += kMaxSeq) {
    attend_group(*a, s0, std::min(a->n_seq, s0 + kMaxSeq), g);
    if (g.a.n_q == 0) continue;
    s = launch_attend(g.a, ws, (cudaStream_t)stream);
    if (s != MSA_OK) return s;
  }
  return MSA_OK;
}

// ---------------------------------------------------------------- backward

msa_status msa_route_backward(const msa_bank_layer* b, const uint16_t* qr, const int32_t* q_seq_off, int32_t n_seq,
                              int32_t n_rows, float eps, const int32_t* pair_seq, const int32_t* pair_doc,
                              const float* pair_dscore, int32_t n_pairs, float* dqr, float* dkr,
                              int64_t* argmax_chunk, int32_t* argmax_row, void* stream) {
  msa_status s = check_bank(b, false);
  if (s != MSA_OK) return s;
  if (n_seq <= 0 || n_seq > kMaxSeq || n_pairs < 0) return fail(MSA_ERR_INVALID_ARG, "route_backward: bad sizes");
  if (!(eps > 0.f)) return fail(MSA_ERR_INVALID_ARG, "route_backward: eps must be > 0");
  if (!q_seq_off || q_seq_off[0] != 0 || q_seq_off[n_seq] != n_rows)
    return fail(MSA_ERR_INVALID_ARG, "route_backward: q_seq_off must start at 0 and end at n_rows");
  for (int i = 0; i < n_seq; ++i)
    if (q_seq_off[i + 1] <= q_seq_off[i]) return fail(MSA_ERR_INVALID_ARG, "route_backward: sequence %d has no rows", i);
  if (n_pairs > 0 && (!qr || !pair_seq || !pair_doc || !pair_dscore || !dqr || !dkr || !argmax_chunk || !argmax_row))
    return fail(MSA_ERR_INVALID_ARG, "route_backward: NULL pointer");
  return launch_route_backward(*b, qr, q_seq_off, n_seq, eps, pair_seq, pair_doc, pair_dscore, n_pairs, dqr, dkr,
                               argmax_chunk, argmax_row, (cudaStream_t)stream);
}

msa_status msa_attend_backward_workspace(const msa_attend_args* a, size_t* bytes) {
  msa_status s = check_attend(a);
  if (s != MSA_OK) return s;
  if (a->top_ids) return fail(MSA_ERR_UNSUPPORTED, "attend_backward: needs a gather listing (sel_off), not the routed form");
  if (a->n_seq > kMaxSeq) return fail(MSA_ERR_UNSUPPORTED, "attend_backward: n_seq = %d (1..%d)", a->n_seq, kMaxSeq);
  if (!bytes) return fail(MSA_ERR_INVALID_ARG, "attend_backward_workspace: bytes is NULL");
  *bytes = attend_backward_workspace(*a);
  return MSA_OK;
}

msa_status msa_attend_backward(const msa_attend_args* a, const float* dout, float* dq, float* dk_loc, float* dv_loc,
                               float* dmem_k, float* dmem_v, void* ws, size_t ws_bytes, void* stream) {
  msa_status s = check_attend(a);
  if (s != MSA_OK) return s;
  if (a->top_ids) return fail(MSA_ERR_UNSUPPORTED, "attend_backward: needs a gather listing (sel_off), not the routed form");
  if (a->n_seq > kMaxSeq) return fail(MSA_ERR_UNSUPPORTED, "attend_backward: n_seq = %d (1..%d)", a->n_seq, kMaxSeq);
  if (!a->out_f32 || !a->lse) return fail(MSA_ERR_INVALID_ARG, "attend_backward: the forward's out_f32 and lse are required");
  if (!dout || !dq) return fail(MSA_ERR_INVALID_ARG, "attend_backward: NULL dout or dq");
  if (a->loc_off[a->n_seq] > 0 && (!dk_loc || !dv_loc)) return fail(MSA_ERR_INVALID_ARG, "attend_backward: NULL dk_loc/dv_loc");
  if (a->max_sel > 0 && (!dmem_k || !dmem_v)) return fail(MSA_ERR_INVALID_ARG, "attend_backward: NULL dmem_k/dmem_v");
  const size_t need = attend_backward_workspace(*a);
  if (!ws || ws_bytes < need) return fail(MSA_ERR_WORKSPACE, "attend_backward: workspace %zu B, need %zu B", ws_bytes, need);
  if (a->n_q == 0) return MSA_OK;
  return launch_attend_backward(*a, dout, dq, dk_loc, dv_loc, dmem_k, dmem_v, ws, (cudaStream_t)stream);
}

// Launches a kernel whose bounded mbarrier wait runs out (nothing arrives),
// so that the failure path can be tested without faulting the GPU: the next
// msa_sync_check reports MSA_ERR_TIMEOUT and the context stays usable. A
// testing control; not declared in msa.h.
msa_status msa_debug_wait_probe(void* stream) { return launch_wait_probe((cudaStream_t)stream); }

msa_status msa_sync_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "sync_check");
  const int e_tc = tc_error_take(), e_pf = pf_error_take(), e_pr = probe_error_take();
  const int e_at = attend_tc_error_take() | attend_dec_tc_error_take() | attend_dec_error_take();
  if (e_tc || e_pf) return fail(MSA_ERR_TIMEOUT, "sync_check: a tensor-core scoring kernel gave up on a wait");
  if (e_pr) return fail(MSA_ERR_TIMEOUT, "sync_check: the wait probe's wait ran out");
  if (e_at) return fail(MSA_ERR_TIMEOUT, "sync_check: the tensor-core attention kernel gave up on a wait");
  return MSA_OK;
}

}  // extern "C"
