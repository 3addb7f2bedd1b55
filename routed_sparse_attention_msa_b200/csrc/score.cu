// Routing scores on CUDA cores, and the query preparation shared by both
// scoring kernels.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — relevance by
// cosine similarity, averaged over heads, then maximised over query tokens; "MSA-arXiv26",
// 核心方法 — the query is compared with every document's pooled routing key]
//
// score(s, j) = max over rows t of s, chunks c of j, of
//               sum_h invq[t,h] * invk[c,h] * (qr[t,h] . kbar_r[c,h])
// with invq already holding 1 / (hr * max(||q||, eps)).
//
// This kernel is the GEMV form for one or two query rows per pass: every
// chunk row (hr x 256 B) is read once with 16-byte loads, the query rows sit
// in registers, and a warp folds its chunks' scores into a running
// per-document maximum that is flushed with one atomicMax (on an
// order-preserving integer encoding) when the document changes. Scores never
// leave the chip. Larger row counts go to the tensor-core kernel.
#include "msa_internal.cuh"

namespace msa {
namespace {

struct QprepArgs {
  const uint16_t* qr;
  int n_rows, hr, n_rows_pad, n_seq;
  float eps;
  float* invq;       // [T, hr]
  float* invq_t;     // [hr, Tp]
  int32_t* col_code; // [T]
  uint4* zero;
  int64_t zero_vecs;
  int32_t q_seq_off[kMaxSeq + 1];
};

// One warp per (row, head): invq = 1 / (hr * max(||q||, eps)), stored row-major
// and head-major; per row, its sequence and whether it is the sequence's last
// row (the column metadata of the many-row scorer). The whole grid also clears
// the scoring workspace (document keys and top-k state).
__global__ void qprep_kernel(const __grid_constant__ QprepArgs a) {
  pdl_wait();
  pdl_trigger();
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (int64_t i = tid; i < a.zero_vecs; i += (int64_t)gridDim.x * blockDim.x) a.zero[i] = make_uint4(0, 0, 0, 0);
  const int lane = threadIdx.x & 31;
  const int w = (int)(tid >> 5);
  if (w >= a.n_rows * a.hr) return;
  uint2 v = __ldg(reinterpret_cast<const uint2*>(a.qr + (size_t)w * kHeadDim + 4 * lane));
  float x0 = bf_lo(v.x), x1 = bf_hi(v.x), x2 = bf_lo(v.y), x3 = bf_hi(v.y);
  float ss = x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) {
    const float iq = 1.0f / ((float)a.hr * fmaxf(sqrtf(ss), a.eps));
    const int t = w / a.hr, h = w % a.hr;
    a.invq[w] = iq;
    a.invq_t[(size_t)h * a.n_rows_pad + t] = iq;
    if (h == 0) {
      int lo = 0, hi = a.n_seq - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a.q_seq_off[mid] <= t) lo = mid; else hi = mid - 1;
      }
      a.col_code[t] = lo | (t + 1 == a.q_seq_off[lo + 1] ? 256 : 0);
    }
  }
}

struct SimtArgs {
  const uint16_t* kbar_r;
  const float* invk;
  const int32_t* chunk_doc;
  const uint16_t* qr;
  const float* invq;
  uint32_t* doc_key;
  int64_t n_chunks, n_docs;
  int hr;
  int row0;        // first row of this pass
  int seq[2];      // sequence of each row of the pass
  int n_rows_pass; // 1 or 2
};

constexpr int kChunksPerWarpTask = 64;

template <int TP>
__global__ void __launch_bounds__(256) score_simt_kernel(SimtArgs a) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int pairs = a.hr >> 1;  // 16-byte loads per lane per chunk
  const int e0 = 8 * (lane & 15);
  const int hsel = lane >> 4;

  // Query rows of this pass in registers, pre-scaled by invq: q[r][i][e].
  float q[TP][8][8];
#pragma unroll
  for (int r = 0; r < TP; ++r) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int h = 2 * i + hsel;
      if (i < pairs && r < a.n_rows_pass) {
        int row = a.row0 + r;
        float sc = a.invq[row * a.hr + h];
        uint4 w = __ldg(reinterpret_cast<const uint4*>(a.qr + ((size_t)row * a.hr + h) * kHeadDim + e0));
        q[r][i][0] = bf_lo(w.x) * sc; q[r][i][1] = bf_hi(w.x) * sc;
        q[r][i][2] = bf_lo(w.y) * sc; q[r][i][3] = bf_hi(w.y) * sc;
        q[r][i][4] = bf_lo(w.z) * sc; q[r][i][5] = bf_hi(w.z) * sc;
        q[r][i][6] = bf_lo(w.w) * sc; q[r][i][7] = bf_hi(w.w) * sc;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) q[r][i][e] = 0.f;
      }
    }
  }

  const int64_t n_tasks = (a.n_chunks + kChunksPerWarpTask - 1) / kChunksPerWarpTask;
  for (int64_t task = gw; task < n_tasks; task += nw) {
    const int64_t c_begin = task * kChunksPerWarpTask;
    const int64_t c_end = min(c_begin + kChunksPerWarpTask, a.n_chunks);
    int cur_doc = -1;
    float best[TP];
#pragma unroll
    for (int r = 0; r < TP; ++r) best[r] = -INFINITY;
    for (int64_t c = c_begin; c < c_end; ++c) {
      const int doc = __ldg(a.chunk_doc + c);
      if (doc != cur_doc) {
        if (cur_doc >= 0 && lane == 0) {
#pragma unroll
          for (int r = 0; r < TP; ++r)
            if (r < a.n_rows_pass)
              atomicMax(a.doc_key + (size_t)a.seq[r] * a.n_docs + cur_doc, ord_f32(best[r]));
        }
        cur_doc = doc;
#pragma unroll
        for (int r = 0; r < TP; ++r) best[r] = -INFINITY;
      }
      const uint16_t* row = a.kbar_r + (size_t)c * a.hr * kHeadDim;
      float part[TP];
#pragma unroll
      for (int r = 0; r < TP; ++r) part[r] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (i < pairs) {
          int h = 2 * i + hsel;
          uint4 w = __ldg(reinterpret_cast<const uint4*>(row + h * kHeadDim + e0));
          float kk = __ldg(a.invk + (size_t)c * a.hr + h);
          float x[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                        bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
#pragma unroll
          for (int r = 0; r < TP; ++r) {
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) dot += x[e] * q[r][i][e];
            part[r] += dot * kk;
          }
        }
      }
#pragma unroll
      for (int r = 0; r < TP; ++r) {
        float v = part[r];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        best[r] = fmaxf(best[r], v);
      }
    }
    if (cur_doc >= 0 && lane == 0) {
#pragma unroll
      for (int r = 0; r < TP; ++r)
        if (r < a.n_rows_pass)
          atomicMax(a.doc_key + (size_t)a.seq[r] * a.n_docs + cur_doc, ord_f32(best[r]));
    }
  }
}

}  // namespace

msa_status launch_qprep(const RoutePlan& p, float eps, cudaStream_t st) {
  const int64_t warps = (int64_t)p.n_rows * p.hr;
  int64_t blocks = (warps * 32 + 255) / 256;
  const int64_t zvecs = (int64_t)(p.zero_bytes / 16);
  const int64_t zblocks = (zvecs + 255) / 256;
  if (blocks < zblocks) blocks = zblocks < 148 * 4 ? zblocks : 148 * 4;
  QprepArgs a{};
  a.qr = p.qr;
  a.n_rows = p.n_rows;
  a.hr = p.hr;
  a.n_rows_pad = p.n_rows_pad;
  a.n_seq = p.n_seq;
  a.eps = eps;
  a.invq = p.invq;
  a.invq_t = p.invq_t;
  a.col_code = p.col_code;
  a.zero = reinterpret_cast<uint4*>(p.zero);
  a.zero_vecs = zvecs;
  for (int i = 0; i <= p.n_seq; ++i) a.q_seq_off[i] = p.q_seq_off[i];
  cudaError_t e = launch_pdl(qprep_kernel, dim3((unsigned)blocks), dim3(256), 0, st, a);
  if (e != cudaSuccess) return cuda_fail(e, "route: query norms");
  return launch_check("route: query norms");
}

msa_status launch_score_simt(const RoutePlan& p, cudaStream_t st) {
  SimtArgs a;
  a.kbar_r = p.kbar_r; a.invk = p.kr_inv_norm; a.chunk_doc = p.chunk_doc;
  a.qr = p.qr; a.invq = p.invq; a.doc_key = p.doc_key;
  a.n_chunks = p.n_chunks; a.n_docs = p.n_docs; a.hr = p.hr;
  int64_t tasks = (p.n_chunks + kChunksPerWarpTask - 1) / kChunksPerWarpTask;
  int64_t blocks = (tasks * 32 + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  int seq = 0;
  for (int row0 = 0; row0 < p.n_rows; row0 += 2) {
    a.row0 = row0;
    a.n_rows_pass = (p.n_rows - row0) >= 2 ? 2 : 1;
    for (int r = 0; r < a.n_rows_pass; ++r) {
      while (p.q_seq_off[seq + 1] <= row0 + r) ++seq;
      a.seq[r] = seq;
    }
    if (a.n_rows_pass == 2) {
      score_simt_kernel<2><<<(unsigned)blocks, 256, 0, st>>>(a);
    } else {
      a.seq[1] = a.seq[0];
      score_simt_kernel<1><<<(unsigned)blocks, 256, 0, st>>>(a);
    }
    msa_status s = launch_check("route: score (CUDA cores)");
    if (s != MSA_OK) return s;
  }
  return MSA_OK;
}

}  // namespace msa
