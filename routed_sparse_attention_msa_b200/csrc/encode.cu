// Offline encode of one routing layer: document -> chunk index, RoPE on K at
// document-local positions, chunk-mean pooling of K, V and K_r, inverse norms
// of the pooled routing keys.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture (chunk-mean
// pooled K/V/K_r; Parallel RoPE resets positions in every document) and
// Inference Pipeline stage 1; "MSA-arXiv26", 核心方法 (chunk-wise mean pool,
// Document-wise RoPE)]
//
// The pooling kernel streams 3 x hkv|hr x 256 B per token from HBM and writes
// one pooled row per chunk: it is HBM-bound. One CTA of 16 threads per head
// handles one chunk at a time; a thread owns 4 RoPE pairs (8 elements) of K,
// and 8 consecutive elements of V and of K_r, so every load is 8 or 16 B and
// every warp reads whole 128-byte segments.
//
// RoPE is applied through the identity sum_u R((p0+u)w) x_u = R(p0 w) sum_u
// R(u w) x_u: per token the thread rotates by u*w (a two-term recurrence in
// fp32 started from cos/sin of w computed in double), and the chunk start
// angle p0*w is applied once per chunk in double.
#include <math.h>

#include "msa_internal.cuh"

namespace msa {
namespace {

__global__ void doc_chunk_scan_kernel(const int64_t* __restrict__ doc_tok_off, int64_t n_docs,
                                      int chunk, int64_t* __restrict__ doc_chunk_off) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t carry;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) {
    carry = 0;
    doc_chunk_off[0] = 0;
  }
  __syncthreads();
  for (int64_t base = 0; base < n_docs; base += blockDim.x) {
    int64_t j = base + tid;
    int64_t v = 0;
    if (j < n_docs) {
      int64_t len = doc_tok_off[j + 1] - doc_tok_off[j];
      v = (len + chunk - 1) / chunk;
    }
    // inclusive warp scan
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int64_t w = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int64_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sums[lane] = w;  // inclusive prefix of warp totals
    }
    __syncthreads();
    int64_t before = carry + (wid > 0 ? warp_sums[wid - 1] : 0);
    if (j < n_docs) doc_chunk_off[j + 1] = before + x;
    __syncthreads();
    if (tid == blockDim.x - 1) carry = before + x;
    __syncthreads();
  }
}

struct PoolArgs {
  const uint16_t* k_tok;
  const uint16_t* v_tok;
  const uint16_t* kr_tok;
  const int64_t* doc_tok_off;
  const int64_t* doc_chunk_off;
  int64_t n_docs, n_chunks;
  int hkv, hr, chunk, rope_mode;
  double log2_theta;
  float eps;
  uint16_t* kbar;
  uint16_t* vbar;
  uint16_t* kbar_r;
  float* inv_norm;
  int32_t* chunk_doc;
};

__device__ __forceinline__ void acc8(float* s, uint4 w) {
  s[0] += bf_lo(w.x); s[1] += bf_hi(w.x);
  s[2] += bf_lo(w.y); s[3] += bf_hi(w.y);
  s[4] += bf_lo(w.z); s[5] += bf_hi(w.z);
  s[6] += bf_lo(w.w); s[7] += bf_hi(w.w);
}

constexpr int kUnroll = 4;

__global__ void __launch_bounds__(256) encode_pool_kernel(PoolArgs a) {
  __shared__ int64_t s_t0, s_p0;  // first token; rotation position of the pooled chunk
  __shared__ int s_n;
  const int tid = threadIdx.x;
  const int h = tid >> 4;   // head owned by this thread
  const int sub = tid & 15; // 16 threads per head
  const bool do_kv = h < a.hkv;
  const bool do_r = h < a.hr;
  const int D = kHeadDim;

  // Per-thread RoPE pairs i = 4*sub + j, j < 4: unit rotation by w_i.
  float cw[4], sw[4];
  double wd[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    int i = 4 * sub + j;
    wd[j] = exp2(-2.0 * (double)i / (double)D * a.log2_theta);
    double s, c;
    sincos(wd[j], &s, &c);
    cw[j] = (float)c;
    sw[j] = (float)s;
  }
  pdl_wait();  // the rotation constants above overlapped the previous kernel's tail
  pdl_trigger();

  for (int64_t c = blockIdx.x; c < a.n_chunks; c += gridDim.x) {
    if (tid == 0) {
      // owning document: the last j with doc_chunk_off[j] <= c
      int64_t lo = 0, hi = a.n_docs - 1;
      while (lo < hi) {
        int64_t mid = (lo + hi + 1) >> 1;
        if (a.doc_chunk_off[mid] <= c) lo = mid; else hi = mid - 1;
      }
      int64_t q = c - a.doc_chunk_off[lo];
      int64_t t0 = a.doc_tok_off[lo] + q * a.chunk;
      int64_t len = a.doc_tok_off[lo + 1] - t0;
      s_t0 = t0;
      s_p0 = a.rope_mode == 1 ? q : q * a.chunk;
      s_n = (int)(len < a.chunk ? len : a.chunk);
      a.chunk_doc[c] = (int32_t)lo;
    }
    __syncthreads();
    const int64_t t0 = s_t0;
    const int n = s_n;
    const int64_t p0 = s_p0;
    __syncthreads();

    float ka[4] = {0, 0, 0, 0}, kb[4] = {0, 0, 0, 0};
    float vs[8] = {0, 0, 0, 0, 0, 0, 0, 0}, rs[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float cr[4] = {1, 1, 1, 1}, sr[4] = {0, 0, 0, 0};  // rotation by u*w

    for (int u0 = 0; u0 < n; u0 += kUnroll) {
      uint2 kl[kUnroll], kh[kUnroll];
      uint4 vv[kUnroll], rr[kUnroll];
#pragma unroll
      for (int e = 0; e < kUnroll; ++e) {
        int64_t t = t0 + u0 + e;
        bool ok = (u0 + e) < n;
        if (do_kv && ok) {
          const uint16_t* kp = a.k_tok + ((size_t)t * a.hkv + h) * D;
          kl[e] = __ldg(reinterpret_cast<const uint2*>(kp + 4 * sub));
          kh[e] = __ldg(reinterpret_cast<const uint2*>(kp + 64 + 4 * sub));
          vv[e] = __ldg(reinterpret_cast<const uint4*>(a.v_tok + ((size_t)t * a.hkv + h) * D + 8 * sub));
        } else {
          kl[e] = make_uint2(0, 0); kh[e] = make_uint2(0, 0); vv[e] = make_uint4(0, 0, 0, 0);
        }
        if (do_r && ok)
          rr[e] = __ldg(reinterpret_cast<const uint4*>(a.kr_tok + ((size_t)t * a.hr + h) * D + 8 * sub));
        else
          rr[e] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int e = 0; e < kUnroll; ++e) {
        if (u0 + e < n) {
          float x0[4] = {bf_lo(kl[e].x), bf_hi(kl[e].x), bf_lo(kl[e].y), bf_hi(kl[e].y)};
          float x1[4] = {bf_lo(kh[e].x), bf_hi(kh[e].x), bf_lo(kh[e].y), bf_hi(kh[e].y)};
#pragma unroll
          if (a.rope_mode == 1) {  // pool first; the chunk is rotated below
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              ka[j] += x0[j];
              kb[j] += x1[j];
            }
          } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              ka[j] += x0[j] * cr[j] - x1[j] * sr[j];
              kb[j] += x0[j] * sr[j] + x1[j] * cr[j];
              float c2 = cr[j] * cw[j] - sr[j] * sw[j];
              float s2 = sr[j] * cw[j] + cr[j] * sw[j];
              cr[j] = c2;
              sr[j] = s2;
            }
          }
          acc8(vs, vv[e]);
          acc8(rs, rr[e]);
        }
      }
    }

    if (do_kv) {
      float oa[4], ob[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        double s, cc;
        sincos((double)p0 * wd[j], &s, &cc);
        float c0 = (float)cc, s0 = (float)s;
        oa[j] = (ka[j] * c0 - kb[j] * s0) / (float)n;
        ob[j] = (ka[j] * s0 + kb[j] * c0) / (float)n;
      }
      uint16_t* kp = a.kbar + ((size_t)c * a.hkv + h) * D;
      *reinterpret_cast<uint2*>(kp + 4 * sub) = make_uint2(pack_bf2(oa[0], oa[1]), pack_bf2(oa[2], oa[3]));
      *reinterpret_cast<uint2*>(kp + 64 + 4 * sub) = make_uint2(pack_bf2(ob[0], ob[1]), pack_bf2(ob[2], ob[3]));
      uint4 vo = make_uint4(pack_bf2(vs[0] / (float)n, vs[1] / (float)n), pack_bf2(vs[2] / (float)n, vs[3] / (float)n),
                            pack_bf2(vs[4] / (float)n, vs[5] / (float)n), pack_bf2(vs[6] / (float)n, vs[7] / (float)n));
      *reinterpret_cast<uint4*>(a.vbar + ((size_t)c * a.hkv + h) * D + 8 * sub) = vo;
    }
    float ss = 0.f;
    if (do_r) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        w[j] = pack_bf2(rs[2 * j] / (float)n, rs[2 * j + 1] / (float)n);
        float lo = bf_lo(w[j]), hi = bf_hi(w[j]);
        ss += lo * lo + hi * hi;
      }
      *reinterpret_cast<uint4*>(a.kbar_r + ((size_t)c * a.hr + h) * D + 8 * sub) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
    // 16 threads of a head are one half-warp: reduce within it.
    ss += __shfl_xor_sync(0xffffffffu, ss, 8);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    if (do_r && sub == 0) {
      float nrm = sqrtf(ss);
      a.inv_norm[(size_t)c * a.hr + h] = 1.0f / fmaxf(nrm, a.eps);
    }
  }
}

// One warp per chunk: lanes read 16 B each; the 16 lanes of a half-warp cover
// one head of 128 elements.
__global__ void bank_norms_kernel(const uint16_t* __restrict__ kbar_r, int64_t n_chunks, int hr,
                                  float eps, float* __restrict__ inv_norm) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int pairs = (hr + 1) / 2;
  pdl_wait();
  pdl_trigger();
  for (int64_t c = warp; c < n_chunks; c += n_warps) {
    for (int i = 0; i < pairs; ++i) {
      int h = 2 * i + (lane >> 4);
      float ss = 0.f;
      if (h < hr) {
        uint4 w = __ldg(reinterpret_cast<const uint4*>(kbar_r + ((size_t)c * hr + h) * kHeadDim +
                                                       8 * (lane & 15)));
        float x[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                      bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += x[e] * x[e];
      }
      ss += __shfl_xor_sync(0xffffffffu, ss, 8);
      ss += __shfl_xor_sync(0xffffffffu, ss, 4);
      ss += __shfl_xor_sync(0xffffffffu, ss, 2);
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      if (h < hr && (lane & 15) == 0) inv_norm[(size_t)c * hr + h] = 1.0f / fmaxf(sqrtf(ss), eps);
    }
  }
}

}  // namespace

msa_status launch_encode(const msa_encode_args& a, cudaStream_t st) {
  cudaError_t e = launch_pdl(doc_chunk_scan_kernel, dim3(1), dim3(1024), 0, st, a.doc_tok_off, a.n_docs, a.chunk,
                             a.doc_chunk_off);
  if (e != cudaSuccess) return cuda_fail(e, "encode: document index");
  msa_status s = launch_check("encode: document index");
  if (s != MSA_OK || a.n_chunks == 0) return s;
  PoolArgs p;
  p.k_tok = a.k_tok; p.v_tok = a.v_tok; p.kr_tok = a.kr_tok;
  p.doc_tok_off = a.doc_tok_off; p.doc_chunk_off = a.doc_chunk_off;
  p.n_docs = a.n_docs; p.n_chunks = a.n_chunks;
  p.hkv = a.hkv; p.hr = a.hr; p.chunk = a.chunk; p.rope_mode = a.rope_mode;
  p.log2_theta = log2((double)a.rope_theta);
  p.eps = a.eps;
  p.kbar = a.kbar; p.vbar = a.vbar; p.kbar_r = a.kbar_r; p.inv_norm = a.kr_inv_norm;
  p.chunk_doc = a.chunk_doc;
  int heads = a.hkv > a.hr ? a.hkv : a.hr;
  int threads = 32 * ((heads + 1) / 2);  // whole warps: the norm reduction shuffles full warps
  int64_t grid = a.n_chunks < 148 * 40 ? a.n_chunks : 148 * 40;
  record_debug_event(0, st);
  e = launch_pdl(encode_pool_kernel, dim3((unsigned)grid), dim3(threads), 0, st, p);
  if (e != cudaSuccess) return cuda_fail(e, "encode: pooling");
  msa_status s2 = launch_check("encode: pooling");
  record_debug_event(1, st);
  return s2;
}

msa_status launch_bank_norms(const uint16_t* kbar_r, int64_t n_chunks, int hr, float eps,
                             float* inv_norm, cudaStream_t st) {
  if (n_chunks == 0) return MSA_OK;
  int64_t warps = n_chunks;
  int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  cudaError_t e = launch_pdl(bank_norms_kernel, dim3((unsigned)blocks), dim3(256), 0, st, kbar_r, n_chunks, hr, eps,
                             inv_norm);
  if (e != cudaSuccess) return cuda_fail(e, "bank norms");
  return launch_check("bank norms");
}

}  // namespace msa
