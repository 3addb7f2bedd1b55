// Gradient of the routing scores, for the contrastive routing loss that
// trains the routing projectors end to end.
//
// ["MSA: Memory Sparse Attention", Abstract and Key Contributions — sparse
// attention whose document selection is trained jointly with the model; "MSA-arXiv26", 核心方法 — generation loss plus a contrastive
// routing loss]
//
// score(s, j) = max over rows t of s and chunks c of j of
//               f(t, c) = (1/hr) sum_h q.k invq invk,  inv = 1 / max(|x|, eps).
// Its gradient flows through the first (chunk-major, row-minor) argmax
// (t*, c*), as in the forward:
//   df/dq_h = (k invq invk - [|q| > eps] (q.k) invk invq^3 q) / hr,
// symmetric in k. One CTA per (sequence, document, dL/dscore) triple: the
// (row, chunk) scores are recomputed on CUDA cores, the argmax is a block-wide
// max on a 64-bit key (score, then the lower chunk, then the lower row), and
// the gradient is added to dqr[t*] (atomics: several triples may share a row)
// and written to dkr[triple].
#include "msa_internal.cuh"

namespace msa {
namespace {

struct RouteBwdArgs {
  const uint16_t* qr;          // [T, hr, d]
  const uint16_t* kbar_r;      // [C, hr, d]
  const float* invk;           // [C, hr]
  const int64_t* doc_chunk_off;
  const int32_t* pair_seq;
  const int32_t* pair_doc;
  const float* pair_dscore;
  float* dqr;                  // [T, hr, d], accumulated
  float* dkr;                  // [P, hr, d]
  int64_t* argmax_chunk;       // [P]
  int32_t* argmax_row;         // [P]
  int hr, n_pairs, n_seq;
  float eps;
  int32_t q_seq_off[kMaxSeq + 1];
};

__device__ __forceinline__ float dot_bf16_row(const uint16_t* a, const uint16_t* b) {
  float s = 0.f;
  for (int i = 0; i < kHeadDim; i += 8) {
    const uint4 x = *reinterpret_cast<const uint4*>(a + i);
    const uint4 y = *reinterpret_cast<const uint4*>(b + i);
    s += bf_lo(x.x) * bf_lo(y.x) + bf_hi(x.x) * bf_hi(y.x) + bf_lo(x.y) * bf_lo(y.y) + bf_hi(x.y) * bf_hi(y.y) +
         bf_lo(x.z) * bf_lo(y.z) + bf_hi(x.z) * bf_hi(y.z) + bf_lo(x.w) * bf_lo(y.w) + bf_hi(x.w) * bf_hi(y.w);
  }
  return s;
}

__global__ void __launch_bounds__(256) route_backward_kernel(const __grid_constant__ RouteBwdArgs a) {
  __shared__ unsigned long long s_best;
  __shared__ float s_stat[3][16];  // per head: |q|, |k|, q.k at the argmax
  pdl_wait();
  pdl_trigger();
  const int p = blockIdx.x;
  const int s = a.pair_seq[p];
  const int32_t j = a.pair_doc[p];
  const int64_t c0 = a.doc_chunk_off[j], c1 = a.doc_chunk_off[j + 1];
  const int t0 = a.q_seq_off[s], t1 = a.q_seq_off[s + 1];
  const int nt = t1 - t0;
  const int64_t n = (c1 - c0) * nt;
  const size_t row = (size_t)a.hr * kHeadDim;
  if (threadIdx.x == 0) s_best = 0ull;
  __syncthreads();
  // every (chunk, row) pair: f(t, c), keyed for the forward's tie order
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const int64_t c = c0 + i / nt;
    const int t = t0 + (int)(i % nt);
    float f = 0.f;
    for (int h = 0; h < a.hr; ++h) {
      const uint16_t* qv = a.qr + (size_t)t * row + (size_t)h * kHeadDim;
      const uint16_t* kv = a.kbar_r + (size_t)c * row + (size_t)h * kHeadDim;
      const float invq = 1.0f / fmaxf(sqrtf(dot_bf16_row(qv, qv)), a.eps);
      f += dot_bf16_row(qv, kv) * invq * a.invk[(size_t)c * a.hr + h];
    }
    f /= (float)a.hr;
    const unsigned long long key = ((unsigned long long)ord_f32(f) << 32) | (0xFFFFFFFFull - (unsigned long long)i);
    atomicMax(&s_best, key);
  }
  __syncthreads();
  float* gk = a.dkr + (size_t)p * row;
  if (n == 0) {  // a document without chunks: no gradient
    for (size_t e = threadIdx.x; e < row; e += blockDim.x) gk[e] = 0.f;
    if (threadIdx.x == 0) {
      a.argmax_chunk[p] = -1;
      a.argmax_row[p] = -1;
    }
    return;
  }
  const int64_t ib = (int64_t)(0xFFFFFFFFull - (s_best & 0xFFFFFFFFull));
  const int64_t cb = c0 + ib / nt;
  const int tb = t0 + (int)(ib % nt);
  if (threadIdx.x == 0) {
    a.argmax_chunk[p] = cb;
    a.argmax_row[p] = tb;
  }
  if (threadIdx.x < a.hr) {
    const int h = threadIdx.x;
    const uint16_t* qv = a.qr + (size_t)tb * row + (size_t)h * kHeadDim;
    const uint16_t* kv = a.kbar_r + (size_t)cb * row + (size_t)h * kHeadDim;
    s_stat[0][h] = sqrtf(dot_bf16_row(qv, qv));
    s_stat[1][h] = sqrtf(dot_bf16_row(kv, kv));
    s_stat[2][h] = dot_bf16_row(qv, kv);
  }
  __syncthreads();
  const float g = a.pair_dscore[p] / (float)a.hr;
  for (size_t e = threadIdx.x; e < row; e += blockDim.x) {
    const int h = (int)(e / kHeadDim);
    const float nq = s_stat[0][h], nk = s_stat[1][h], dot = s_stat[2][h];
    const float iq = 1.0f / fmaxf(nq, a.eps), ik = 1.0f / fmaxf(nk, a.eps);
    const float q = bf1(a.qr[(size_t)tb * row + e]);
    const float k = bf1(a.kbar_r[(size_t)cb * row + e]);
    const float gq = k * iq * ik - (nq > a.eps ? dot * ik * iq * iq * iq * q : 0.f);
    const float gkk = q * iq * ik - (nk > a.eps ? dot * iq * ik * ik * ik * k : 0.f);
    atomicAdd(a.dqr + (size_t)tb * row + e, g * gq);
    gk[e] = g * gkk;
  }
}

}  // namespace

msa_status launch_route_backward(const msa_bank_layer& b, const uint16_t* qr, const int32_t* q_seq_off, int n_seq,
                                 float eps, const int32_t* pair_seq, const int32_t* pair_doc,
                                 const float* pair_dscore, int n_pairs, float* dqr, float* dkr,
                                 int64_t* argmax_chunk, int32_t* argmax_row, cudaStream_t st) {
  if (n_pairs == 0) return MSA_OK;
  RouteBwdArgs a{};
  a.qr = qr; a.kbar_r = b.kbar_r; a.invk = b.kr_inv_norm; a.doc_chunk_off = b.doc_chunk_off;
  a.pair_seq = pair_seq; a.pair_doc = pair_doc; a.pair_dscore = pair_dscore;
  a.dqr = dqr; a.dkr = dkr; a.argmax_chunk = argmax_chunk; a.argmax_row = argmax_row;
  a.hr = b.hr; a.n_pairs = n_pairs; a.n_seq = n_seq; a.eps = eps;
  for (int i = 0; i <= n_seq; ++i) a.q_seq_off[i] = q_seq_off[i];
  cudaError_t e = launch_pdl(route_backward_kernel, dim3(n_pairs), dim3(256), 0, st, a);
  if (e != cudaSuccess) return cuda_fail(e, "route backward");
  return launch_check("route backward");
}

}  // namespace msa
