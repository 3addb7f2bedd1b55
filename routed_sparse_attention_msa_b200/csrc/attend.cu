// Sparse attention: every query row attends over its sequence's selected
// pooled K/V (already rotated at document-local positions at encode time)
// concatenated with its local K/V, with the query and the local keys rotated
// at global positions offset by k; GQA; causal over the local keys.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — the pooled
// K/V of the selected documents joined to the K/V of the query's recent context;
// Parallel (document-wise) RoPE and Global RoPE offset by k (Figure 2)]
//
// Two kernels:
//  1. rope_rows: rotates the query rows and the local keys once per call into
//     fp32 copies (local keys as bf16 high + low halves for the tensor-core
//     kernel of attend_tc.cu), and clears the merge tickets. Each angle is formed and
//     reduced modulo 2*pi in double, so positions of any size keep full
//     accuracy, and then evaluated with sincosf.
//  2. attend_split: split-K flash decoding. A CTA owns one kv head, a tile of
//     query rows of one sequence (the GQA group's q heads x rows = 4, 8 or 16
//     query vectors, the fewest that hold the sequence's rows: 4 for a decoding
//     step with 4 q heads per kv head) and one contiguous slice of the key
//     list. It walks the slice in
//     blocks of 64 keys: the block's key and value rows are staged into
//     shared memory with every load issued at once (decoding is bound by
//     memory latency, a few hundred keys per head), then logits, an online
//     softmax in fp32, and P.V. With several splits, each CTA writes an
//     unnormalised partial (o, m, l); the last CTA of the (tile, head) to
//     finish (atomic ticket, no waiting) merges them by log-sum-exp.
// The split count puts about two CTAs on every SM.
#include <math.h>

#include <algorithm>

#include "attend_params.cuh"

namespace msa {
namespace {

constexpr int kMaxVec = 16;    // query vectors per CTA (group x rows): 4, 8 or 16
constexpr int kKeyBlock = 64;  // keys per block
constexpr int kThreads = 128;
constexpr int kPad = 132;      // fp32 row stride in shared memory (bank-conflict free)

template <int VEC>
struct Smem {
  float q[VEC][kHeadDim];
  float k[kKeyBlock][kPad];
  float v[kKeyBlock][kPad];
  float p[VEC][kKeyBlock];
  float m[VEC], l[VEC], corr[VEC];
  int g[VEC];
  bool last;
};

// One thread per (row, group of 4 heads, pair) of the query rows, then of the
// local keys: the angle depends on the position and the pair only, so it is
// formed once per thread and applied to the group's heads (loads issued
// together).
constexpr int kRopeHeads = 4;

__global__ void rope_rows_kernel(const __grid_constant__ AttnParams p) {
  pdl_wait();
  pdl_trigger();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (p.tickets && idx < (int64_t)p.n_tiles * p.hkv) p.tickets[idx] = 0u;
  const int gq = (p.hq + kRopeHeads - 1) / kRopeHeads, gk = (p.hkv + kRopeHeads - 1) / kRopeHeads;
  const int64_t nq = p.rope_q ? (int64_t)p.n_q * gq * 64 : 0;
  const int64_t nk = (int64_t)p.n_loc * gk * 64;
  if (idx >= nq + nk) return;
  const bool is_q = idx < nq;
  const int64_t j = is_q ? idx : idx - nq;
  const int heads = is_q ? p.hq : p.hkv;
  const int groups = is_q ? gq : gk;
  const int i = (int)(j & 63);
  const int64_t rg = j >> 6;
  const int row = (int)(rg / groups);
  const int h0 = (int)(rg % groups) * kRopeHeads;
  double pos;
  if (is_q) {
    const int s = seq_of(p.q_seq_off, p.n_seq, row);
    pos = p.pos_offset + (double)(p.q_start[s] + (row - p.q_seq_off[s]));
  } else {
    const int s = seq_of(p.loc_off, p.n_seq, row);
    pos = p.pos_offset + (double)(row - p.loc_off[s]);
  }
  const float r = reduced_angle(pos * p.inv_freq[i]);
  float sn, cs;
  sincosf(r, &sn, &cs);
  const size_t base = ((size_t)row * heads + h0) * kHeadDim + i;
  const uint16_t* src = (is_q ? p.q : p.k_loc) + base;
  float* dst = (is_q ? p.qrot : p.krot) + base;
  float x0[kRopeHeads], x1[kRopeHeads];
#pragma unroll
  for (int u = 0; u < kRopeHeads; ++u) {
    const bool in = h0 + u < heads;
    x0[u] = in ? bf1(src[u * kHeadDim]) : 0.f;
    x1[u] = in ? bf1(src[u * kHeadDim + 64]) : 0.f;
  }
#pragma unroll
  for (int u = 0; u < kRopeHeads; ++u) {
    if (h0 + u < heads) {
      const float y0 = x0[u] * cs - x1[u] * sn, y1 = x0[u] * sn + x1[u] * cs;
      if (!is_q && p.krot_split) {  // bf16 high halves [0, 128), low halves [128, 256) of the row
        uint16_t* kb = reinterpret_cast<uint16_t*>(p.krot) + ((size_t)row * heads + h0 + u) * 2 * kHeadDim;
        const uint32_t b0 = f2bf_bits(y0), b1 = f2bf_bits(y1);
        kb[i] = (uint16_t)b0;
        kb[64 + i] = (uint16_t)b1;
        kb[kHeadDim + i] = (uint16_t)f2bf_bits(y0 - __uint_as_float(b0 << 16));
        kb[kHeadDim + 64 + i] = (uint16_t)f2bf_bits(y1 - __uint_as_float(b1 << 16));
      } else {
        dst[u * kHeadDim] = y0;
        dst[u * kHeadDim + 64] = y1;
      }
    }
  }
}

// VEC query vectors per CTA: logits give each key two threads of VEC/2
// vectors; the softmax gives each warp VEC/4 vectors; P.V gives each thread 4
// dimensions of VEC/4 vectors.
template <int VEC>
__global__ void __launch_bounds__(kThreads) attend_split_kernel(const __grid_constant__ AttnParams p) {
  constexpr int VH = VEC / 2;  // vectors per thread in the logits
  constexpr int VW = VEC / 4;  // vectors per warp (softmax) and per thread (P.V)
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem<VEC>& S = *reinterpret_cast<Smem<VEC>*>(smem_raw);
  pdl_wait();
  pdl_trigger();

  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int sp_idx = blockIdx.x;
  const int kvh = blockIdx.y;
  const int tile = blockIdx.z;
  const int s = seq_of(p.tile_off, p.n_seq, tile);
  const int row0 = p.q_seq_off[s] + (tile - p.tile_off[s]) * p.rt;
  const int nr = min(p.rt, p.q_seq_off[s + 1] - row0);
  const int g0 = p.q_start[s] + (row0 - p.q_seq_off[s]);  // active index of the tile's first row

  const int64_t mem_base = p.sel_off[s];
  const int64_t n_mem = p.sel_off[s + 1] - mem_base;
  const int n_loc_s = p.loc_off[s + 1] - p.loc_off[s];
  const int lvis = max(0, min(n_loc_s, g0 + nr));  // local keys visible to the last row
  const int64_t n_keys = n_mem + lvis;
  const int64_t per = (n_keys + p.n_splits - 1) / p.n_splits;
  const int64_t k_begin = (int64_t)sp_idx * per;
  const int64_t k_end = min(n_keys, k_begin + per);
  const size_t row_stride = (size_t)p.hkv * kHeadDim;

  // query vectors v = rr * group + gg
  for (int idx = tid; idx < VEC * kHeadDim / 4; idx += kThreads) {
    const int v = idx / (kHeadDim / 4), e4 = idx % (kHeadDim / 4);
    const int rr = v / p.group, gg = v % p.group;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rr < nr)
      x = reinterpret_cast<const float4*>(p.qrot + ((size_t)(row0 + rr) * p.hq + kvh * p.group + gg) * kHeadDim)[e4];
    reinterpret_cast<float4*>(S.q[v])[e4] = x;
  }
  if (tid < VEC) {
    S.m[tid] = -INFINITY;
    S.l[tid] = 0.f;
    const int rr = tid / p.group;
    S.g[tid] = rr < nr ? g0 + rr : -1;  // -1: padding vector, sees nothing
  }

  float acc[VW][4];
#pragma unroll
  for (int i = 0; i < VW; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
  const int d0 = 4 * lane;

  for (int64_t kb = k_begin; kb < k_end; kb += kKeyBlock) {
    const int nb = (int)min((int64_t)kKeyBlock, k_end - kb);
    __syncthreads();  // previous block's K/V/P no longer in use
    // ---- stage K and V rows of the block: 64 rows x 16 chunks of 8 elements
    {
      constexpr int kChunks = kKeyBlock * (kHeadDim / 8);  // 1024
      uint4 kw[kChunks / kThreads], vw[kChunks / kThreads];
      float4 klo[kChunks / kThreads], khi[kChunks / kThreads];
      bool local[kChunks / kThreads];
#pragma unroll
      for (int u = 0; u < kChunks / kThreads; ++u) {
        const int idx = tid + u * kThreads;
        const int jj = idx >> 4, c8 = idx & 15;
        local[u] = false;
        kw[u] = vw[u] = make_uint4(0, 0, 0, 0);
        klo[u] = khi[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (jj < nb) {
          const int64_t key = kb + jj;
          if (key < n_mem) {
            const int64_t r = p.sel_chunk ? p.sel_chunk[mem_base + key] : mem_base + key;
            const size_t off = (size_t)r * row_stride + (size_t)kvh * kHeadDim + 8 * c8;
            kw[u] = *reinterpret_cast<const uint4*>(p.mem_k + off);
            vw[u] = *reinterpret_cast<const uint4*>(p.mem_v + off);
          } else {
            local[u] = true;
            const size_t lr = (size_t)(p.loc_off[s] + (key - n_mem)) * p.hkv + kvh;
            const float4* kp = reinterpret_cast<const float4*>(p.krot + lr * kHeadDim + 8 * c8);
            klo[u] = kp[0];
            khi[u] = kp[1];
            vw[u] = *reinterpret_cast<const uint4*>(p.v_loc + lr * kHeadDim + 8 * c8);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kChunks / kThreads; ++u) {
        const int idx = tid + u * kThreads;
        const int jj = idx >> 4, c8 = idx & 15;
        float4 a, b;
        if (local[u]) {
          a = klo[u];
          b = khi[u];
        } else {
          a = make_float4(bf_lo(kw[u].x), bf_hi(kw[u].x), bf_lo(kw[u].y), bf_hi(kw[u].y));
          b = make_float4(bf_lo(kw[u].z), bf_hi(kw[u].z), bf_lo(kw[u].w), bf_hi(kw[u].w));
        }
        *reinterpret_cast<float4*>(&S.k[jj][8 * c8]) = a;
        *reinterpret_cast<float4*>(&S.k[jj][8 * c8 + 4]) = b;
        *reinterpret_cast<float4*>(&S.v[jj][8 * c8]) =
            make_float4(bf_lo(vw[u].x), bf_hi(vw[u].x), bf_lo(vw[u].y), bf_hi(vw[u].y));
        *reinterpret_cast<float4*>(&S.v[jj][8 * c8 + 4]) =
            make_float4(bf_lo(vw[u].z), bf_hi(vw[u].z), bf_lo(vw[u].w), bf_hi(vw[u].w));
      }
    }
    __syncthreads();
    // ---- logits: thread -> one key, VH query vectors
    {
      const int jj = tid & (kKeyBlock - 1);
      const int vh = (tid >> 6) * VH;
      float dot[VH];
#pragma unroll
      for (int v = 0; v < VH; ++v) dot[v] = 0.f;
#pragma unroll 8
      for (int c = 0; c < kHeadDim / 4; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(&S.k[jj][4 * c]);
#pragma unroll
        for (int v = 0; v < VH; ++v) {
          const float4 qa = *reinterpret_cast<const float4*>(&S.q[vh + v][4 * c]);
          dot[v] += x.x * qa.x + x.y * qa.y + x.z * qa.z + x.w * qa.w;
        }
      }
      const int64_t key = kb + jj;
      const int lj = key < n_mem ? -1 : (int)(key - n_mem);  // local key index, or -1
#pragma unroll
      for (int v = 0; v < VH; ++v) {
        const int g = S.g[vh + v];
        const bool vis = jj < nb && g >= 0 && (lj < 0 || lj <= g);
        S.p[vh + v][jj] = vis ? dot[v] * p.scale : -INFINITY;
      }
    }
    __syncthreads();
    // ---- online softmax: warp w owns vectors VW*w .. VW*w + VW-1
#pragma unroll
    for (int vi = 0; vi < VW; ++vi) {
      const int v = VW * wid + vi;
      const float x0 = S.p[v][lane], x1 = S.p[v][lane + 32];
      float bm = fmaxf(x0, x1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
      const float m_old = S.m[v];
      const float m_new = fmaxf(m_old, bm);
      float p0 = 0.f, p1 = 0.f, corr = 1.f;
      if (m_new != -INFINITY) {
        p0 = expf(x0 - m_new);
        p1 = expf(x1 - m_new);
        corr = expf(m_old - m_new);
      }
      float sum = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      S.p[v][lane] = p0;
      S.p[v][lane + 32] = p1;
      __syncwarp();
      if (lane == 0) {
        S.l[v] = S.l[v] * corr + sum;
        S.m[v] = m_new;
        S.corr[v] = corr;
      }
    }
    __syncthreads();
    // ---- P V: thread -> dims 4*lane .. +3 of vectors wid + 4i
#pragma unroll
    for (int i = 0; i < VW; ++i) {
      const float corr = S.corr[wid + 4 * i];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][e] *= corr;
    }
    for (int j = 0; j < nb; ++j) {
      const float4 x = *reinterpret_cast<const float4*>(&S.v[j][d0]);
#pragma unroll
      for (int i = 0; i < VW; ++i) {
        const float pr = S.p[wid + 4 * i][j];
        acc[i][0] += pr * x.x;
        acc[i][1] += pr * x.y;
        acc[i][2] += pr * x.z;
        acc[i][3] += pr * x.w;
      }
    }
  }
  __syncthreads();

  // ---- write: final rows, or a partial for the merge
  if (p.n_splits == 1) {
#pragma unroll
    for (int i = 0; i < VW; ++i) {
      const int v = wid + 4 * i;
      const int rr = v / p.group, gg = v % p.group;
      if (rr >= nr) continue;
      const int row = row0 + rr, h = kvh * p.group + gg;
      const float m = S.m[v], l = S.l[v];
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      const float o[4] = {acc[i][0] * inv, acc[i][1] * inv, acc[i][2] * inv, acc[i][3] * inv};
      const size_t base = ((size_t)row * p.hq + h) * kHeadDim + d0;
      *reinterpret_cast<uint2*>(p.out + base) = make_uint2(pack_bf2(o[0], o[1]), pack_bf2(o[2], o[3]));
      if (p.out_f32) *reinterpret_cast<float4*>(p.out_f32 + base) = make_float4(o[0], o[1], o[2], o[3]);
      if (p.lse && lane == 0) p.lse[(size_t)row * p.hq + h] = l > 0.f ? m + logf(l) : -INFINITY;
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < VW; ++i) {
    const int v = wid + 4 * i;
    const int rr = v / p.group, gg = v % p.group;
    if (rr >= nr) continue;
    const size_t pi = ((size_t)(row0 + rr) * p.hq + kvh * p.group + gg) * p.n_splits + sp_idx;
    *reinterpret_cast<float4*>(p.part_o + pi * kHeadDim + d0) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    if (lane == 0) p.part_ml[pi] = make_float2(S.m[v], S.l[v]);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(p.tickets + (size_t)tile * p.hkv + kvh, 1u);
    S.last = (t == (unsigned)(p.n_splits - 1));
  }
  __syncthreads();
  if (!S.last) return;
  __threadfence();
  // ---- merge the splits of this (tile, kv head)
#pragma unroll
  for (int i = 0; i < VW; ++i) {
    const int v = wid + 4 * i;
    const int rr = v / p.group, gg = v % p.group;
    if (rr >= nr) continue;
    const int row = row0 + rr, h = kvh * p.group + gg;
    const size_t rh = (size_t)row * p.hq + h;
    float m = -INFINITY;
    for (int j = 0; j < p.n_splits; ++j) m = fmaxf(m, __ldcg(p.part_ml + rh * p.n_splits + j).x);
    float l = 0.f, o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
    if (m != -INFINITY) {
      for (int j = 0; j < p.n_splits; ++j) {
        const float2 x = __ldcg(p.part_ml + rh * p.n_splits + j);
        if (x.y > 0.f) {
          const float w = expf(x.x - m);
          const float4 o = __ldcg(reinterpret_cast<const float4*>(p.part_o + (rh * p.n_splits + j) * kHeadDim + d0));
          l += x.y * w;
          o0 += o.x * w;
          o1 += o.y * w;
          o2 += o.z * w;
          o3 += o.w * w;
        }
      }
    }
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    const float r[4] = {o0 * inv, o1 * inv, o2 * inv, o3 * inv};
    const size_t base = rh * kHeadDim + d0;
    *reinterpret_cast<uint2*>(p.out + base) = make_uint2(pack_bf2(r[0], r[1]), pack_bf2(r[2], r[3]));
    if (p.out_f32) *reinterpret_cast<float4*>(p.out_f32 + base) = make_float4(r[0], r[1], r[2], r[3]);
    if (p.lse && lane == 0) p.lse[rh] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}


// ------------------------------------------------------------------ backward
//
// Gradients of the attention (the pages' end-to-end differentiable sparse
// attention): with D = dout.out per (row, head), for every visible key j,
//   p_j = exp(scale q'.k'_j - lse),  ds_j = p_j (dout.v_j - D),
//   dq' = scale sum_j ds_j k'_j,  dk'_j = scale sum ds_j q',  dv_j = sum p_j dout,
// primes are rotated vectors; dq and the local keys' gradients are rotated
// back (by the negative angle), pooled memory keys are used as stored.

// Rotation of the pair (x, y) of dimension i by minus the angle at `pos`.
__device__ __forceinline__ void rotate_back(float& x, float& y, int i, double pos, const double* inv_freq) {
  const float r = reduced_angle(pos * inv_freq[i]);
  float sn, cs;
  sincosf(r, &sn, &cs);
  const float a = x * cs + y * sn;
  const float b = -x * sn + y * cs;
  x = a;
  y = b;
}

// D[row, head] = dout . out (one warp per (row, head)).
__global__ void attend_bwd_prep_kernel(const __grid_constant__ AttnParams p, const float* __restrict__ dout,
                                       float* __restrict__ Dvec) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= (int64_t)p.n_q * p.hq) return;
  const float4 a = reinterpret_cast<const float4*>(dout + w * kHeadDim)[lane];
  const float4 b = reinterpret_cast<const float4*>(p.out_f32 + w * kHeadDim)[lane];
  float x = a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if (lane == 0) Dvec[w] = x;
}

// Stage rows of K (fp32, rotated for local keys) and V of keys [kb, kb+nb) of
// sequence s into shared memory; `all_local` also stages local keys no row sees.
template <int KB>
__device__ __forceinline__ void stage_kv(const AttnParams& p, int s, int kvh, int64_t kb, int nb, int64_t n_mem,
                                         int64_t mem_base, float (*Sk)[kPad], float (*Sv)[kPad]) {
  const size_t row_stride = (size_t)p.hkv * kHeadDim;
  for (int idx = threadIdx.x; idx < KB * (kHeadDim / 8); idx += kThreads) {
    const int jj = idx >> 4, c8 = idx & 15;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a, va = a, vb = a;
    if (jj < nb) {
      const int64_t key = kb + jj;
      uint4 vw;
      if (key < n_mem) {
        const int64_t r = p.sel_chunk ? p.sel_chunk[mem_base + key] : mem_base + key;
        const size_t off = (size_t)r * row_stride + (size_t)kvh * kHeadDim + 8 * c8;
        const uint4 kw = *reinterpret_cast<const uint4*>(p.mem_k + off);
        vw = *reinterpret_cast<const uint4*>(p.mem_v + off);
        a = make_float4(bf_lo(kw.x), bf_hi(kw.x), bf_lo(kw.y), bf_hi(kw.y));
        b = make_float4(bf_lo(kw.z), bf_hi(kw.z), bf_lo(kw.w), bf_hi(kw.w));
      } else {
        const size_t lr = (size_t)(p.loc_off[s] + (key - n_mem)) * p.hkv + kvh;
        const float4* kp = reinterpret_cast<const float4*>(p.krot + lr * kHeadDim + 8 * c8);
        a = kp[0];
        b = kp[1];
        vw = *reinterpret_cast<const uint4*>(p.v_loc + lr * kHeadDim + 8 * c8);
      }
      va = make_float4(bf_lo(vw.x), bf_hi(vw.x), bf_lo(vw.y), bf_hi(vw.y));
      vb = make_float4(bf_lo(vw.z), bf_hi(vw.z), bf_lo(vw.w), bf_hi(vw.w));
    }
    *reinterpret_cast<float4*>(&Sk[jj][8 * c8]) = a;
    *reinterpret_cast<float4*>(&Sk[jj][8 * c8 + 4]) = b;
    *reinterpret_cast<float4*>(&Sv[jj][8 * c8]) = va;
    *reinterpret_cast<float4*>(&Sv[jj][8 * c8 + 4]) = vb;
  }
}

template <int VEC>
struct BwdQSmem {
  float q[VEC][kHeadDim];
  float go[VEC][kHeadDim];
  float k[kKeyBlock][kPad];
  float v[kKeyBlock][kPad];
  float ds[VEC][kKeyBlock];
  float lse[VEC], D[VEC];
  int g[VEC];
};

// dq: one CTA per (query tile, kv head), all keys of the sequence.
template <int VEC>
__global__ void __launch_bounds__(kThreads) attend_bwd_dq_kernel(const __grid_constant__ AttnParams p,
                                                                 const float* __restrict__ dout,
                                                                 const float* __restrict__ Dvec,
                                                                 float* __restrict__ dq) {
  constexpr int VH = VEC / 2, VW = VEC / 4;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BwdQSmem<VEC>& S = *reinterpret_cast<BwdQSmem<VEC>*>(smem_raw);
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int kvh = blockIdx.y, tile = blockIdx.z;
  const int s = seq_of(p.tile_off, p.n_seq, tile);
  const int row0 = p.q_seq_off[s] + (tile - p.tile_off[s]) * p.rt;
  const int nr = min(p.rt, p.q_seq_off[s + 1] - row0);
  const int g0 = p.q_start[s] + (row0 - p.q_seq_off[s]);
  const int64_t mem_base = p.sel_off[s];
  const int64_t n_mem = p.sel_off[s + 1] - mem_base;
  const int n_loc_s = p.loc_off[s + 1] - p.loc_off[s];
  const int64_t n_keys = n_mem + max(0, min(n_loc_s, g0 + nr));

  for (int idx = tid; idx < VEC * kHeadDim / 4; idx += kThreads) {
    const int v = idx / (kHeadDim / 4), e4 = idx % (kHeadDim / 4);
    const int rr = v / p.group, gg = v % p.group;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
    if (rr < nr) {
      const size_t o = ((size_t)(row0 + rr) * p.hq + kvh * p.group + gg) * kHeadDim;
      x = reinterpret_cast<const float4*>(p.qrot + o)[e4];
      y = reinterpret_cast<const float4*>(dout + o)[e4];
    }
    reinterpret_cast<float4*>(S.q[v])[e4] = x;
    reinterpret_cast<float4*>(S.go[v])[e4] = y;
  }
  if (tid < VEC) {
    const int rr = tid / p.group, gg = tid % p.group;
    const size_t rh = (size_t)(row0 + rr) * p.hq + kvh * p.group + gg;
    S.lse[tid] = rr < nr ? p.lse[rh] : 0.f;
    S.D[tid] = rr < nr ? Dvec[rh] : 0.f;
    S.g[tid] = rr < nr ? g0 + rr : -1;
  }
  float acc[VW][4];
#pragma unroll
  for (int i = 0; i < VW; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
  const int d0 = 4 * lane;

  for (int64_t kb = 0; kb < n_keys; kb += kKeyBlock) {
    const int nb = (int)min((int64_t)kKeyBlock, n_keys - kb);
    __syncthreads();
    stage_kv<kKeyBlock>(p, s, kvh, kb, nb, n_mem, mem_base, S.k, S.v);
    __syncthreads();
    {  // ds for (vector, key): thread -> key jj, VH vectors
      const int jj = tid & (kKeyBlock - 1);
      const int vh = (tid >> 6) * VH;
      float l[VH], dp[VH];
#pragma unroll
      for (int v = 0; v < VH; ++v) l[v] = dp[v] = 0.f;
#pragma unroll 4
      for (int c = 0; c < kHeadDim / 4; ++c) {
        const float4 kx = *reinterpret_cast<const float4*>(&S.k[jj][4 * c]);
        const float4 vx = *reinterpret_cast<const float4*>(&S.v[jj][4 * c]);
#pragma unroll
        for (int v = 0; v < VH; ++v) {
          const float4 qa = *reinterpret_cast<const float4*>(&S.q[vh + v][4 * c]);
          const float4 ga = *reinterpret_cast<const float4*>(&S.go[vh + v][4 * c]);
          l[v] += kx.x * qa.x + kx.y * qa.y + kx.z * qa.z + kx.w * qa.w;
          dp[v] += vx.x * ga.x + vx.y * ga.y + vx.z * ga.z + vx.w * ga.w;
        }
      }
      const int64_t key = kb + jj;
      const int lj = key < n_mem ? -1 : (int)(key - n_mem);
#pragma unroll
      for (int v = 0; v < VH; ++v) {
        const int g = S.g[vh + v];
        const bool vis = jj < nb && g >= 0 && (lj < 0 || lj <= g);
        const float pr = vis ? expf(l[v] * p.scale - S.lse[vh + v]) : 0.f;
        S.ds[vh + v][jj] = pr * (dp[v] - S.D[vh + v]);
      }
    }
    __syncthreads();
    for (int j = 0; j < nb; ++j) {
      const float4 x = *reinterpret_cast<const float4*>(&S.k[j][d0]);
#pragma unroll
      for (int i = 0; i < VW; ++i) {
        const float w = S.ds[wid + 4 * i][j];
        acc[i][0] += w * x.x;
        acc[i][1] += w * x.y;
        acc[i][2] += w * x.z;
        acc[i][3] += w * x.w;
      }
    }
  }
  // rotate back and write: dims 4*lane..+3 pair with lane +- 16
#pragma unroll
  for (int i = 0; i < VW; ++i) {
    const int v = wid + 4 * i;
    const int rr = v / p.group, gg = v % p.group;
    float o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float mine = acc[i][e] * p.scale;
      const float other = __shfl_xor_sync(0xffffffffu, mine, 16);
      float x = lane < 16 ? mine : other, y = lane < 16 ? other : mine;  // (dim, dim + 64)
      const int dim = 4 * (lane & 15) + e;
      if (rr < nr) rotate_back(x, y, dim, p.pos_offset + (double)(g0 + rr), p.inv_freq);
      o[e] = lane < 16 ? x : y;
    }
    if (rr < nr) {
      const size_t base = ((size_t)(row0 + rr) * p.hq + kvh * p.group + gg) * kHeadDim + d0;
      *reinterpret_cast<float4*>(dq + base) = make_float4(o[0], o[1], o[2], o[3]);
    }
  }
}

constexpr int kBwdKeys = 32;   // keys per dk/dv CTA
constexpr int kBwdVec = 16;    // query vectors per step of the dk/dv loop

struct BwdKVSmem {
  float k[kBwdKeys][kPad];
  float v[kBwdKeys][kPad];
  float q[kBwdVec][kHeadDim];
  float go[kBwdVec][kHeadDim];
  float p[kBwdVec][kBwdKeys];
  float ds[kBwdVec][kBwdKeys];
  float lse[kBwdVec], D[kBwdVec];
  int g[kBwdVec];
};

// dk, dv: one CTA per (32-key block, kv head, sequence), all query vectors of
// the sequence. Every key of the sequence (visible to some row or not) is
// written once: memory rows in selection order, local rows rotated back.
__global__ void __launch_bounds__(kThreads) attend_bwd_dkdv_kernel(const __grid_constant__ AttnParams p,
                                                                   const float* __restrict__ dout,
                                                                   const float* __restrict__ Dvec,
                                                                   float* __restrict__ dk_loc,
                                                                   float* __restrict__ dv_loc,
                                                                   float* __restrict__ dmem_k,
                                                                   float* __restrict__ dmem_v) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BwdKVSmem& S = *reinterpret_cast<BwdKVSmem*>(smem_raw);
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x;
  const int kvh = blockIdx.y, s = blockIdx.z;
  const int64_t mem_base = p.sel_off[s];
  const int64_t n_mem = p.sel_off[s + 1] - mem_base;
  const int n_loc_s = p.loc_off[s + 1] - p.loc_off[s];
  const int64_t n_all = n_mem + n_loc_s;
  const int64_t kb = (int64_t)blockIdx.x * kBwdKeys;
  if (kb >= n_all) return;
  const int nb = (int)min((int64_t)kBwdKeys, n_all - kb);
  stage_kv<kBwdKeys>(p, s, kvh, kb, nb, n_mem, mem_base, S.k, S.v);

  const int jk = tid >> 2;          // key of this thread in the accumulation
  const int dsl = (tid & 3) * 32;   // its 32 dimensions
  float ak[32], av[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) ak[e] = av[e] = 0.f;

  const int r0 = p.q_seq_off[s], r1 = p.q_seq_off[s + 1];
  const int rows_per_step = kBwdVec / p.group;
  for (int rb = r0; rb < r1; rb += rows_per_step) {
    const int nr = min(rows_per_step, r1 - rb);
    __syncthreads();  // staging above / previous step's q, go, p, ds no longer in use
    for (int idx = tid; idx < kBwdVec * kHeadDim / 4; idx += kThreads) {
      const int v = idx / (kHeadDim / 4), e4 = idx % (kHeadDim / 4);
      const int rr = v / p.group, gg = v % p.group;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f), y = x;
      if (rr < nr) {
        const size_t o = ((size_t)(rb + rr) * p.hq + kvh * p.group + gg) * kHeadDim;
        x = reinterpret_cast<const float4*>(p.qrot + o)[e4];
        y = reinterpret_cast<const float4*>(dout + o)[e4];
      }
      reinterpret_cast<float4*>(S.q[v])[e4] = x;
      reinterpret_cast<float4*>(S.go[v])[e4] = y;
    }
    if (tid < kBwdVec) {
      const int rr = tid / p.group, gg = tid % p.group;
      const size_t rh = (size_t)(rb + rr) * p.hq + kvh * p.group + gg;
      S.lse[tid] = rr < nr ? p.lse[rh] : 0.f;
      S.D[tid] = rr < nr ? Dvec[rh] : 0.f;
      S.g[tid] = rr < nr ? p.q_start[s] + (rb + rr - r0) : -1;
    }
    __syncthreads();
    {  // p and ds for (vector, key): thread -> key (tid & 31), 4 vectors
      const int jj = tid & 31;
      const int v0 = (tid >> 5) * 4;
      float l[4] = {0.f, 0.f, 0.f, 0.f}, dp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int c = 0; c < kHeadDim / 4; ++c) {
        const float4 kx = *reinterpret_cast<const float4*>(&S.k[jj][4 * c]);
        const float4 vx = *reinterpret_cast<const float4*>(&S.v[jj][4 * c]);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const float4 qa = *reinterpret_cast<const float4*>(&S.q[v0 + v][4 * c]);
          const float4 ga = *reinterpret_cast<const float4*>(&S.go[v0 + v][4 * c]);
          l[v] += kx.x * qa.x + kx.y * qa.y + kx.z * qa.z + kx.w * qa.w;
          dp[v] += vx.x * ga.x + vx.y * ga.y + vx.z * ga.z + vx.w * ga.w;
        }
      }
      const int64_t key = kb + jj;
      const int lj = key < n_mem ? -1 : (int)(key - n_mem);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int g = S.g[v0 + v];
        const bool vis = jj < nb && g >= 0 && (lj < 0 || lj <= g);
        const float pr = vis ? expf(l[v] * p.scale - S.lse[v0 + v]) : 0.f;
        S.p[v0 + v][jj] = pr;
        S.ds[v0 + v][jj] = pr * (dp[v] - S.D[v0 + v]);
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int v = 0; v < kBwdVec; ++v) {
      const float w_ds = S.ds[v][jk] * p.scale, w_p = S.p[v][jk];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 qa = *reinterpret_cast<const float4*>(&S.q[v][dsl + e]);
        const float4 ga = *reinterpret_cast<const float4*>(&S.go[v][dsl + e]);
        ak[e] += w_ds * qa.x; ak[e + 1] += w_ds * qa.y; ak[e + 2] += w_ds * qa.z; ak[e + 3] += w_ds * qa.w;
        av[e] += w_p * ga.x; av[e + 1] += w_p * ga.y; av[e + 2] += w_p * ga.z; av[e + 3] += w_p * ga.w;
      }
    }
  }
  // write: thread slices 0/2 and 1/3 of one key are the rotation pairs (d, d + 64);
  // the shuffle runs on every lane, the rotation only for local keys
  const int64_t key = kb + jk;
  const bool local = key >= n_mem;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float other = __shfl_xor_sync(0xffffffffu, ak[e], 2);
    if (local && jk < nb) {
      float x = (tid & 2) ? other : ak[e], y = (tid & 2) ? ak[e] : other;
      rotate_back(x, y, (dsl & 63) + e, p.pos_offset + (double)(key - n_mem), p.inv_freq);
      ak[e] = (tid & 2) ? y : x;
    }
  }
  if (jk >= nb) return;
  float* dk;
  float* dv;
  if (!local) {
    const size_t o = ((size_t)(mem_base + key) * p.hkv + kvh) * kHeadDim + dsl;
    dk = dmem_k + o;
    dv = dmem_v + o;
  } else {
    const size_t o = ((size_t)(p.loc_off[s] + (key - n_mem)) * p.hkv + kvh) * kHeadDim + dsl;
    dk = dk_loc + o;
    dv = dv_loc + o;
  }
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    *reinterpret_cast<float4*>(dk + e) = make_float4(ak[e], ak[e + 1], ak[e + 2], ak[e + 3]);
    *reinterpret_cast<float4*>(dv + e) = make_float4(av[e], av[e + 1], av[e + 2], av[e + 3]);
  }
}

struct Shape {
  int vec, rt, n_tiles, n_splits, n_loc;
  bool rot;   // decoding kernel: it rotates its own local keys (rope_rows does otherwise)
  bool tc;    // tensor-core kernel (many rows per sequence)
  bool dec;   // decoding kernel (attend_dec.cu)
  bool list;  // routed form listed into the workspace first (the split-K kernels, or top_k > 256)
};

// 0 automatic, 1 split-K, 2 tensor cores, 3 decoding tensor cores, 4 decoding
// kernel on CUDA cores (testing control)
int g_attend_kernel = 0;
int g_attend_splits = 0;  // forward split-K key splits: 0 = planned below, else forced (testing control)
int g_dec_rot_keys = 48;  // decoding kernel: largest local-key share per CTA it rotates itself
int g_tc_split_blocks = 2;  // tensor-core kernel: fewest 64-key blocks per key split

// allow_tc: the forward may take the tensor-core kernel when the query
// vectors of a sequence fill at least half of its 128-vector tile.
Shape plan_kernel(const msa_attend_args& a, bool allow_tc) {
  Shape sh{};
  const int group = a.hq / a.hkv;
  int max_rows = 1;
  for (int s = 0; s < a.n_seq; ++s) {
    const int rows = a.q_seq_off[s + 1] - a.q_seq_off[s];
    max_rows = rows > max_rows ? rows : max_rows;
  }
  sh.tc = allow_tc && g_attend_kernel != 1 && g_attend_kernel != 3 && g_attend_kernel != 4 && kAttnTcVec % group == 0 &&
          (g_attend_kernel == 2 || max_rows * group >= kAttnTcVec / 2);
  if (sh.tc) {
    sh.vec = kAttnTcVec;
    sh.rt = kAttnTcVec / group;
    sh.n_tiles = 0;
    int max_loc = 0;
    for (int s = 0; s < a.n_seq; ++s) {
      sh.n_tiles += (a.q_seq_off[s + 1] - a.q_seq_off[s] + sh.rt - 1) / sh.rt;
      max_loc = std::max(max_loc, a.loc_off[s + 1] - a.loc_off[s]);
    }
    sh.n_loc = a.loc_off[a.n_seq];
    // split the 64-key blocks across CTAs while (tiles x kv heads) is under one
    // wave, keeping at least g_tc_split_blocks blocks per split: a CTA pipelines
    // its blocks (the next one's copies and S overlap the current one's
    // softmax), a split pays the cluster's merge; the splits of a (tile, kv
    // head) are one cluster, so at most 8
    const int64_t ctas = (int64_t)sh.n_tiles * a.hkv;
    const int64_t blocks = (a.max_sel + max_loc + 63) / 64;
    int64_t splits = ctas > 0 ? (148 + ctas - 1) / ctas : 1;
    splits = std::min<int64_t>(splits, (blocks + g_tc_split_blocks - 1) / g_tc_split_blocks);
    if (g_attend_splits > 0) splits = g_attend_splits;  // testing control
    splits = std::min<int64_t>(std::min<int64_t>(splits, blocks), 8);
    sh.n_splits = (int)std::max<int64_t>(splits, 1);
    return sh;
  }
  sh.dec = allow_tc && (g_attend_kernel == 0 || g_attend_kernel == 4);
  // query vectors per CTA: the GQA group times enough rows, 4 to 16
  sh.vec = 4;
  while (sh.vec < kMaxVec && sh.vec < group * max_rows) sh.vec *= 2;
  if (sh.vec < group) sh.vec = group;
  sh.rt = sh.vec / group;
  sh.n_tiles = 0;
  int max_loc = 0;
  for (int s = 0; s < a.n_seq; ++s) {
    const int rows = a.q_seq_off[s + 1] - a.q_seq_off[s];
    sh.n_tiles += (rows + sh.rt - 1) / sh.rt;
    const int nl = a.loc_off[s + 1] - a.loc_off[s];
    max_loc = max_loc > nl ? max_loc : nl;
  }
  sh.n_loc = a.loc_off[a.n_seq];
  if (sh.dec) {
    // one CTA per SM (the kernel takes ~218 KB of shared memory): key splits
    // per (tile, kv head) while the grid is under 148 CTAs, each split an even
    // share of the sequence's memory keys and of its local keys; the splits of
    // a (tile, kv head) are one cluster, so at most 8
    int max_lvis = 0;
    for (int s = 0; s < a.n_seq; ++s) {
      const int rows = a.q_seq_off[s + 1] - a.q_seq_off[s];
      const int nl = a.loc_off[s + 1] - a.loc_off[s];
      max_lvis = std::max(max_lvis, std::max(0, std::min(nl, a.q_start[s] + rows)));
    }
    const int64_t pairs = std::max<int64_t>((int64_t)sh.n_tiles * a.hkv, 1);
    int64_t splits = g_attend_splits > 0 ? g_attend_splits : 148 / pairs;
    const int64_t cap = (a.max_sel + max_lvis + 63) / 64;  // at least one 64-key block each
    splits = std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(splits, cap), kDecMaxSplits));
    sh.n_splits = (int)splits;
    // a CTA rotates its own share of the local keys when that is at most
    // g_dec_rot_keys: below that the work costs less than a kernel boundary
    const int share = (int)((max_lvis + splits - 1) / splits);
    sh.rot = share <= std::min(g_dec_rot_keys, kDecRotKeysMax);
    return sh;
  }
  const int64_t max_keys = a.max_sel + max_loc;
  const int64_t ctas = (int64_t)sh.n_tiles * a.hkv;
  int64_t splits = (2 * 148 + ctas - 1) / (ctas > 0 ? ctas : 1);
  const int64_t cap = (max_keys + 31) / 32;  // at least 32 keys per split
  if (splits > cap) splits = cap;
  if (splits < 1) splits = 1;
  if (splits > 64) splits = 64;
  if (allow_tc && g_attend_splits > 0) splits = std::min<int64_t>(g_attend_splits, std::max<int64_t>(cap, 1));
  sh.n_splits = (int)splits;
  return sh;
}

Shape plan(const msa_attend_args& a, bool allow_tc) {
  Shape sh = plan_kernel(a, allow_tc);
  // the decoding and tensor-core kernels list the routed form's rows themselves
  sh.list = a.sel_off == nullptr && !((sh.dec || sh.tc) && a.top_k <= kDecRoutedMaxK);
  return sh;
}

struct Layout {
  size_t qrot, krot, part_o, part_ml, tickets, list_off, list_chunk, total;
};

Layout layout(const msa_attend_args& a, const Shape& sh) {
  Layout L{};
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t o = at;
    at += align_up(bytes, 256);
    return o;
  };
  if (sh.dec) {
    // the decoding kernel: the local keys rotated by rope_rows (bf16 high and low halves, 512 B)
    if (!sh.rot) {
      L.qrot = take((size_t)a.n_q * a.hq * kHeadDim * 4);
      L.krot = take((size_t)std::max(sh.n_loc, 1) * a.hkv * 2 * kHeadDim * 2);
    }
  } else {
    L.qrot = take((size_t)a.n_q * a.hq * kHeadDim * 4);
    L.krot = take((size_t)(sh.n_loc > 0 ? sh.n_loc : 1) * a.hkv * kHeadDim * 4);
    const size_t np = sh.n_splits > 1 ? (size_t)a.n_q * a.hq * sh.n_splits : 0;
    L.part_o = take(np * kHeadDim * 4);
    L.part_ml = take(np * 8);
    L.tickets = take((size_t)sh.n_tiles * a.hkv * 4 + 4);
  }
  if (sh.list) {  // the routed form's listing: n_seq x max_sel rows at most
    L.list_off = take((size_t)(a.n_seq + 1) * 8);
    L.list_chunk = take((size_t)std::max<int64_t>((int64_t)a.n_seq * a.max_sel, 1) * 8);
  }
  L.total = std::max<size_t>(at, 256);
  return L;
}

template <int VEC>
msa_status launch_vec(const AttnParams& P, dim3 grid, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  cudaError_t e = smem_limit_once(attend_split_kernel<VEC>, (int)sizeof(Smem<VEC>), attr);
  if (e != cudaSuccess) return cuda_fail(e, "attend: shared memory");
  e = launch_pdl(attend_split_kernel<VEC>, grid, dim3(kThreads), sizeof(Smem<VEC>), st, P);
  if (e != cudaSuccess) return cuda_fail(e, "attend: split-K with merge");
  return launch_check("attend: split-K with merge");
}

}  // namespace

size_t attend_workspace(const msa_attend_args& a, int* n_splits_out) {
  const Shape sh = plan(a, true);
  if (n_splits_out) *n_splits_out = sh.n_splits;
  return layout(a, sh).total;
}

namespace {

void fill_params(const msa_attend_args& a, const Shape& sh, const Layout& L, char* w, AttnParams& P) {
  P.q = a.q; P.k_loc = a.k_loc; P.v_loc = a.v_loc; P.mem_k = a.mem_k; P.mem_v = a.mem_v;
  P.sel_off = a.sel_off; P.sel_chunk = a.sel_chunk;
  P.top_ids = a.top_ids; P.doc_chunk_off = a.doc_chunk_off; P.n_docs = a.n_docs; P.top_k = a.top_k;
  P.max_sel = a.max_sel;
  if (sh.list) {
    P.sel_off = reinterpret_cast<const int64_t*>(w + L.list_off);
    P.sel_chunk = reinterpret_cast<const int64_t*>(w + L.list_chunk);
  }
  P.rot_in_kernel = sh.rot ? 1 : 0;
  P.rope_q = sh.dec && sh.rot ? 0 : 1;
  P.qrot = reinterpret_cast<float*>(w + L.qrot);
  P.krot = reinterpret_cast<float*>(w + L.krot);
  P.part_o = reinterpret_cast<float*>(w + L.part_o);
  P.part_ml = reinterpret_cast<float2*>(w + L.part_ml);
  P.tickets = sh.dec ? nullptr : reinterpret_cast<unsigned*>(w + L.tickets);  // the decoding kernel merges in a cluster
  P.out = a.out; P.out_f32 = a.out_f32; P.lse = a.lse;
  P.n_seq = a.n_seq; P.n_q = a.n_q; P.n_loc = sh.n_loc; P.hq = a.hq; P.hkv = a.hkv;
  P.group = a.hq / a.hkv; P.rt = sh.rt; P.n_splits = sh.n_splits; P.n_tiles = sh.n_tiles;
  P.krot_split = (sh.tc || sh.dec) ? 1 : 0;
  P.scale = a.scale > 0.f ? a.scale : 1.0f / sqrtf((float)kHeadDim);
  P.pos_offset = (double)a.pos_offset;
  P.log2_theta = log2((double)a.rope_theta);
  for (int i = 0; i < kHeadDim / 2; ++i) P.inv_freq[i] = exp2(-2.0 * (double)i / (double)kHeadDim * P.log2_theta);
  int t = 0;
  for (int s = 0; s < a.n_seq; ++s) {
    P.q_seq_off[s] = a.q_seq_off[s];
    P.q_start[s] = a.q_start[s];
    P.loc_off[s] = a.loc_off[s];
    P.tile_off[s] = t;
    t += (a.q_seq_off[s + 1] - a.q_seq_off[s] + sh.rt - 1) / sh.rt;
  }
  P.q_seq_off[a.n_seq] = a.q_seq_off[a.n_seq];
  P.loc_off[a.n_seq] = a.loc_off[a.n_seq];
  P.tile_off[a.n_seq] = t;
}

msa_status launch_rope(const AttnParams& P, const msa_attend_args& a, const Shape& sh, cudaStream_t st) {
  const int gq = (a.hq + kRopeHeads - 1) / kRopeHeads, gk = (a.hkv + kRopeHeads - 1) / kRopeHeads;
  int64_t n = (P.rope_q ? (int64_t)a.n_q * gq * 64 : 0) + (int64_t)sh.n_loc * gk * 64;
  const int64_t nt = P.tickets ? (int64_t)sh.n_tiles * a.hkv : 0;
  if (n < nt) n = nt;
  if (n < 1) n = 1;
  cudaError_t e = launch_pdl(rope_rows_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, P);
  if (e != cudaSuccess) return cuda_fail(e, "attend: rotate queries and local keys");
  return launch_check("attend: rotate queries and local keys");
}

template <int VEC>
msa_status launch_bwd_dq(const AttnParams& P, const float* dout, const float* Dvec, float* dq, dim3 grid,
                         cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  cudaError_t e = smem_limit_once(attend_bwd_dq_kernel<VEC>, (int)sizeof(BwdQSmem<VEC>), attr);
  if (e != cudaSuccess) return cuda_fail(e, "attend backward: shared memory");
  e = launch_pdl(attend_bwd_dq_kernel<VEC>, grid, dim3(kThreads), sizeof(BwdQSmem<VEC>), st, P, dout,
                             Dvec, dq);
  if (e != cudaSuccess) return cuda_fail(e, "attend backward: dq");
  return launch_check("attend backward: dq");
}

}  // namespace

msa_status launch_attend(const msa_attend_args& a, void* ws, cudaStream_t st) {
  const Shape sh = plan(a, true);
  const Layout L = layout(a, sh);
  AttnParams P{};  // kernel parameter block (4.3 KB: large kernel parameters, CUDA >= 12.1)
  char* w = reinterpret_cast<char*>(ws);
  fill_params(a, sh, L, w, P);
  msa_status s = MSA_OK;
  if (sh.list) {
    s = launch_gather_index(a.doc_chunk_off, a.n_docs, a.top_ids, a.n_seq, a.top_k,
                            reinterpret_cast<int64_t*>(w + L.list_off), reinterpret_cast<int64_t*>(w + L.list_chunk),
                            (int64_t)a.n_seq * a.max_sel, st);
    if (s != MSA_OK) return s;
  }
  if (sh.dec && sh.rot) return launch_attend_dec(P, st);  // rotates its own queries and local keys
  if (sh.dec) {  // rope_rows rotates the queries and local keys
    s = launch_rope(P, a, sh, st);
    return s != MSA_OK ? s : launch_attend_dec(P, st);
  }
  s = launch_rope(P, a, sh, st);
  if (s != MSA_OK) return s;
  if (sh.tc) return launch_attend_tc(P, st);
  if (g_attend_kernel == 3) return launch_attend_dec_tc(P, st);
  dim3 grid((unsigned)sh.n_splits, (unsigned)a.hkv, (unsigned)sh.n_tiles);
  switch (sh.vec) {
    case 4: return launch_vec<4>(P, grid, st);
    case 8: return launch_vec<8>(P, grid, st);
    default: return launch_vec<16>(P, grid, st);
  }
}

size_t attend_backward_workspace(const msa_attend_args& a) {
  const Shape sh = plan(a, false);
  const Layout L = layout(a, sh);
  return L.total + align_up((size_t)a.n_q * a.hq * sizeof(float), 256);
}

msa_status launch_attend_backward(const msa_attend_args& a, const float* dout, float* dq, float* dk_loc,
                                  float* dv_loc, float* dmem_k, float* dmem_v, void* ws, cudaStream_t st) {
  const Shape sh = plan(a, false);
  const Layout L = layout(a, sh);
  AttnParams P{};
  char* w = reinterpret_cast<char*>(ws);
  fill_params(a, sh, L, w, P);
  float* Dvec = reinterpret_cast<float*>(w + L.total);
  msa_status s = launch_rope(P, a, sh, st);
  if (s != MSA_OK) return s;
  const int64_t warps = (int64_t)a.n_q * a.hq;
  cudaError_t e = launch_pdl(attend_bwd_prep_kernel, dim3((unsigned)((warps * 32 + 255) / 256)), dim3(256), 0, st, P,
                             dout, Dvec);
  if (e != cudaSuccess) return cuda_fail(e, "attend backward: prep");
  s = launch_check("attend backward: prep");
  if (s != MSA_OK) return s;
  dim3 gq(1, (unsigned)a.hkv, (unsigned)sh.n_tiles);
  switch (sh.vec) {
    case 4: s = launch_bwd_dq<4>(P, dout, Dvec, dq, gq, st); break;
    case 8: s = launch_bwd_dq<8>(P, dout, Dvec, dq, gq, st); break;
    default: s = launch_bwd_dq<16>(P, dout, Dvec, dq, gq, st); break;
  }
  if (s != MSA_OK) return s;
  int max_loc = 0;
  for (int q = 0; q < a.n_seq; ++q) max_loc = std::max(max_loc, a.loc_off[q + 1] - a.loc_off[q]);
  const int64_t max_keys = a.max_sel + max_loc;
  static std::atomic<uint64_t> attr{0};
  e = smem_limit_once(attend_bwd_dkdv_kernel, (int)sizeof(BwdKVSmem), attr);
  if (e != cudaSuccess) return cuda_fail(e, "attend backward: shared memory");
  dim3 gk((unsigned)((max_keys + kBwdKeys - 1) / kBwdKeys > 0 ? (max_keys + kBwdKeys - 1) / kBwdKeys : 1),
          (unsigned)a.hkv, (unsigned)a.n_seq);
  e = launch_pdl(attend_bwd_dkdv_kernel, gk, dim3(kThreads), sizeof(BwdKVSmem), st, P, dout, Dvec, dk_loc, dv_loc,
                 dmem_k, dmem_v);
  if (e != cudaSuccess) return cuda_fail(e, "attend backward: dk, dv");
  return launch_check("attend backward: dk, dv");
}

}  // namespace msa

// Selects the attention kernel of later msa_attend calls in this process:
// 0 = automatic, 1 = split-K, 2 = tensor cores (any row count), 3 = the
// decoding tensor-core kernel, 4 = the decoding kernel on CUDA cores (what
// automatic picks for decoding shapes); returns the previous setting. A
// testing and benchmarking control; not declared in msa.h.
extern "C" int msa_debug_set_attend_kernel(int which) {
  const int old = msa::g_attend_kernel;
  if (which >= 0 && which <= 4) msa::g_attend_kernel = which;
  return old;
}

// Forces the number of key splits of the forward kernels in later msa_attend
// calls (split-K kernel: clamped to 1..64 and to one split per 32 keys; the
// decoding and tensor-core kernels, whose splits form one cluster: to 1..8
// and to their key blocks); 0 restores the planned count. Returns the
// previous setting. Workspace sizes follow the setting, so query
// msa_attend_workspace after changing it. A testing and benchmarking
// control; not declared in msa.h.
extern "C" int msa_debug_set_attend_splits(int n) {
  const int old = msa::g_attend_splits;
  if (n >= 0 && n <= 64) msa::g_attend_splits = n;
  return old;
}

// Largest share of a sequence's local keys (per CTA) that the decoding kernel
// rotates itself in later msa_attend calls (0..256; 0: rope_rows always does);
// returns the previous setting. Workspace sizes follow the setting. A testing
// and benchmarking control; not declared in msa.h.
extern "C" int msa_debug_set_dec_rot_keys(int n) {
  const int old = msa::g_dec_rot_keys;
  if (n >= 0 && n <= msa::kDecRotKeysMax) msa::g_dec_rot_keys = n;
  return old;
}

// Fewest 64-key blocks per key split of the many-row tensor-core attention in
// later msa_attend calls (1..64); returns the previous setting. Workspace
// sizes follow it. A benchmarking control; not declared in msa.h.
extern "C" int msa_debug_set_tc_split_blocks(int n) {
  const int old = msa::g_tc_split_blocks;
  if (n >= 1 && n <= 64) msa::g_tc_split_blocks = n;
  return old;
}
