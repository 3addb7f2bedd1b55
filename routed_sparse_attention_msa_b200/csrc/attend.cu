// Sparse attention: every query row attends over its sequence's selected
// pooled K/V (already rotated at document-local positions at encode time)
// concatenated with its local K/V, with the query and the local keys rotated
// at global positions offset by k; GQA; causal over the local keys.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — the selected
// documents' compressed K/V are concatenated with the query's local K/V;
// Parallel (document-wise) RoPE and Global RoPE offset by k (Figure 2)]
//
// Three kernels:
//  1. rope_rows: rotates the query rows and the local keys once per call into
//     fp32 copies (angles in double, so positions of any size keep full
//     accuracy); every attention CTA then reads rotated rows.
//  2. attend_split: split-K flash decoding. A CTA owns one kv head, a tile of
//     query rows of one sequence (the GQA group's q heads x rows = 16 query
//     vectors) and one contiguous slice of the key list; it walks the slice in
//     blocks of 64 keys with an online softmax in fp32 and writes an
//     unnormalised partial (o, m, l), or the final row when there is one split.
//  3. attend_merge: combines the splits' partials by log-sum-exp.
// Decoding is latency-bound (a few hundred keys per head), so the split count
// is chosen to put about two CTAs on every SM.
#include <math.h>

#include "msa_internal.cuh"

namespace msa {
namespace {

constexpr int kVec = 16;       // query vectors per CTA (group x rows)
constexpr int kKeyBlock = 64;  // keys per block
constexpr int kThreads = 128;

struct AttnParams {
  const uint16_t* q;
  const uint16_t* k_loc;
  const uint16_t* v_loc;
  const uint16_t* mem_k;
  const uint16_t* mem_v;
  const int64_t* sel_off;
  const int64_t* sel_chunk;
  float* qrot;      // [n_q, hq, d]
  float* krot;      // [n_loc, hkv, d]
  float* part_o;    // [n_q, hq, splits, d]
  float2* part_ml;  // [n_q, hq, splits]
  uint16_t* out;
  float* out_f32;
  float* lse;
  int n_seq, n_q, n_loc, hq, hkv, group, rt, n_splits, n_tiles;
  float scale;
  double pos_offset, log2_theta;
  int32_t q_seq_off[kMaxSeq + 1];
  int32_t q_start[kMaxSeq];
  int32_t loc_off[kMaxSeq + 1];
  int32_t tile_off[kMaxSeq + 1];
};

__device__ __forceinline__ int seq_of(const int32_t* off, int n_seq, int x) {
  int lo = 0, hi = n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One thread per (row, head, pair). which = 0: query rows at pos_offset + g;
// which = 1: local keys at pos_offset + j.
__global__ void rope_rows_kernel(const __grid_constant__ AttnParams p, int which) {
  const int heads = which == 0 ? p.hq : p.hkv;
  const int rows = which == 0 ? p.n_q : p.n_loc;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)rows * heads * 64) return;
  const int i = (int)(idx & 63);
  const int64_t rh = idx >> 6;
  const int row = (int)(rh / heads);
  double pos;
  if (which == 0) {
    int s = seq_of(p.q_seq_off, p.n_seq, row);
    pos = p.pos_offset + (double)(p.q_start[s] + (row - p.q_seq_off[s]));
  } else {
    int s = seq_of(p.loc_off, p.n_seq, row);
    pos = p.pos_offset + (double)(row - p.loc_off[s]);
  }
  const uint16_t* src = (which == 0 ? p.q : p.k_loc) + rh * kHeadDim;
  float* dst = (which == 0 ? p.qrot : p.krot) + rh * kHeadDim;
  double w = exp2(-2.0 * (double)i / (double)kHeadDim * p.log2_theta);
  double sn, cs;
  sincos(pos * w, &sn, &cs);
  double x0 = bf1(src[i]), x1 = bf1(src[i + 64]);
  dst[i] = (float)(x0 * cs - x1 * sn);
  dst[i + 64] = (float)(x0 * sn + x1 * cs);
}

__global__ void __launch_bounds__(kThreads) attend_split_kernel(const __grid_constant__ AttnParams p) {
  __shared__ float sq[kVec][kHeadDim];
  __shared__ float sp[kVec][kKeyBlock];
  __shared__ float s_m[kVec], s_l[kVec], s_corr[kVec];
  __shared__ int s_g[kVec];

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

  // query vectors v = rr * group + gg
  for (int idx = tid; idx < kVec * kHeadDim; idx += kThreads) {
    int v = idx / kHeadDim, e = idx % kHeadDim;
    int rr = v / p.group, gg = v % p.group;
    float x = 0.f;
    if (rr < nr) x = p.qrot[((size_t)(row0 + rr) * p.hq + kvh * p.group + gg) * kHeadDim + e];
    sq[v][e] = x;
  }
  if (tid < kVec) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
    int rr = tid / p.group;
    s_g[tid] = rr < nr ? g0 + rr : -1;  // -1: padding vector, sees nothing
  }
  __syncthreads();

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
  const int d0 = 4 * lane;
  const size_t row_stride = (size_t)p.hkv * kHeadDim;

  for (int64_t kb = k_begin; kb < k_end; kb += kKeyBlock) {
    const int nb = (int)min((int64_t)kKeyBlock, k_end - kb);
    // ---- logits: thread -> one key, 8 query vectors
    {
      const int jj = tid & (kKeyBlock - 1);
      const int vh = (tid >> 6) * 8;
      float dot[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) dot[v] = 0.f;
      int lj = -1;  // local key index, or -1 for a memory key
      if (jj < nb) {
        const int64_t key = kb + jj;
        if (key < n_mem) {
          int64_t r = p.sel_chunk ? p.sel_chunk[mem_base + key] : mem_base + key;
          const uint4* kp = reinterpret_cast<const uint4*>(p.mem_k + (size_t)r * row_stride + (size_t)kvh * kHeadDim);
#pragma unroll 4
          for (int c = 0; c < kHeadDim / 8; ++c) {
            uint4 w = kp[c];
            float x[8] = {bf_lo(w.x), bf_hi(w.x), bf_lo(w.y), bf_hi(w.y),
                          bf_lo(w.z), bf_hi(w.z), bf_lo(w.w), bf_hi(w.w)};
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 qa = *reinterpret_cast<const float4*>(&sq[vh + v][8 * c]);
              const float4 qb = *reinterpret_cast<const float4*>(&sq[vh + v][8 * c + 4]);
              dot[v] += x[0] * qa.x + x[1] * qa.y + x[2] * qa.z + x[3] * qa.w +
                        x[4] * qb.x + x[5] * qb.y + x[6] * qb.z + x[7] * qb.w;
            }
          }
        } else {
          lj = (int)(key - n_mem);
          const float4* kp = reinterpret_cast<const float4*>(
              p.krot + ((size_t)(p.loc_off[s] + lj) * p.hkv + kvh) * kHeadDim);
#pragma unroll 4
          for (int c = 0; c < kHeadDim / 4; ++c) {
            float4 x = kp[c];
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 qa = *reinterpret_cast<const float4*>(&sq[vh + v][4 * c]);
              dot[v] += x.x * qa.x + x.y * qa.y + x.z * qa.z + x.w * qa.w;
            }
          }
        }
      }
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const int g = s_g[vh + v];
        bool vis = jj < nb && g >= 0 && (lj < 0 || lj <= g);
        sp[vh + v][jj] = vis ? dot[v] * p.scale : -INFINITY;
      }
    }
    __syncthreads();
    // ---- online softmax: warp w owns vectors 4w .. 4w+3
#pragma unroll
    for (int vi = 0; vi < 4; ++vi) {
      const int v = 4 * wid + vi;
      float x0 = sp[v][lane], x1 = sp[v][lane + 32];
      float bm = fmaxf(x0, x1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
      const float m_old = s_m[v];
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
      sp[v][lane] = p0;
      sp[v][lane + 32] = p1;
      __syncwarp();
      if (lane == 0) {
        s_l[v] = s_l[v] * corr + sum;
        s_m[v] = m_new;
        s_corr[v] = corr;
      }
    }
    __syncthreads();
    // ---- P V: thread -> dims 4*lane .. +3 of vectors wid + 4i
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float corr = s_corr[wid + 4 * i];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][e] *= corr;
    }
    for (int j = 0; j < nb; ++j) {
      const int64_t key = kb + j;
      const uint16_t* vp;
      if (key < n_mem) {
        int64_t r = p.sel_chunk ? p.sel_chunk[mem_base + key] : mem_base + key;
        vp = p.mem_v + (size_t)r * row_stride + (size_t)kvh * kHeadDim;
      } else {
        vp = p.v_loc + ((size_t)(p.loc_off[s] + (key - n_mem)) * p.hkv + kvh) * kHeadDim;
      }
      const uint2 w = *reinterpret_cast<const uint2*>(vp + d0);
      const float x0 = bf_lo(w.x), x1 = bf_hi(w.x), x2 = bf_lo(w.y), x3 = bf_hi(w.y);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float pr = sp[wid + 4 * i][j];
        acc[i][0] += pr * x0;
        acc[i][1] += pr * x1;
        acc[i][2] += pr * x2;
        acc[i][3] += pr * x3;
      }
    }
    __syncthreads();
  }

  // ---- write
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int v = wid + 4 * i;
    const int rr = v / p.group, gg = v % p.group;
    if (rr >= nr) continue;
    const int row = row0 + rr;
    const int h = kvh * p.group + gg;
    const float m = s_m[v], l = s_l[v];
    if (p.n_splits == 1) {
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      float o[4] = {acc[i][0] * inv, acc[i][1] * inv, acc[i][2] * inv, acc[i][3] * inv};
      const size_t base = ((size_t)row * p.hq + h) * kHeadDim + d0;
      *reinterpret_cast<uint2*>(p.out + base) = make_uint2(pack_bf2(o[0], o[1]), pack_bf2(o[2], o[3]));
      if (p.out_f32) *reinterpret_cast<float4*>(p.out_f32 + base) = make_float4(o[0], o[1], o[2], o[3]);
      if (p.lse && lane == 0) p.lse[(size_t)row * p.hq + h] = l > 0.f ? m + logf(l) : -INFINITY;
    } else {
      const size_t pi = ((size_t)row * p.hq + h) * p.n_splits + sp_idx;
      *reinterpret_cast<float4*>(p.part_o + pi * kHeadDim + d0) =
          make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
      if (lane == 0) p.part_ml[pi] = make_float2(m, l);
    }
  }
}

// One CTA per (row, head), one thread per dimension.
__global__ void attend_merge_kernel(const __grid_constant__ AttnParams p) {
  const int rh = blockIdx.x;
  const int e = threadIdx.x;
  const float2* ml = p.part_ml + (size_t)rh * p.n_splits;
  float m = -INFINITY;
  for (int i = 0; i < p.n_splits; ++i) m = fmaxf(m, ml[i].x);
  float l = 0.f, o = 0.f;
  if (m != -INFINITY) {
    for (int i = 0; i < p.n_splits; ++i) {
      const float2 x = ml[i];
      if (x.y > 0.f) {
        const float w = expf(x.x - m);
        l += x.y * w;
        o += p.part_o[((size_t)rh * p.n_splits + i) * kHeadDim + e] * w;
      }
    }
  }
  const float r = l > 0.f ? o / l : 0.f;
  const size_t base = (size_t)rh * kHeadDim + e;
  p.out[base] = (uint16_t)f2bf_bits(r);
  if (p.out_f32) p.out_f32[base] = r;
  if (p.lse && e == 0) p.lse[rh] = l > 0.f ? m + logf(l) : -INFINITY;
}

struct Shape {
  int rt, n_tiles, n_splits, n_loc;
};

Shape plan(const msa_attend_args& a) {
  Shape sh;
  const int group = a.hq / a.hkv;
  sh.rt = kVec / group;
  sh.n_tiles = 0;
  int max_loc = 0;
  for (int s = 0; s < a.n_seq; ++s) {
    int rows = a.q_seq_off[s + 1] - a.q_seq_off[s];
    sh.n_tiles += (rows + sh.rt - 1) / sh.rt;
    max_loc = max_loc > a.loc_off[s + 1] - a.loc_off[s] ? max_loc : a.loc_off[s + 1] - a.loc_off[s];
  }
  sh.n_loc = a.loc_off[a.n_seq];
  const int64_t max_keys = a.max_sel + max_loc;
  const int64_t ctas = (int64_t)sh.n_tiles * a.hkv;
  int64_t splits = (2 * 148 + ctas - 1) / (ctas > 0 ? ctas : 1);
  int64_t cap = (max_keys + 31) / 32;  // at least 32 keys per split
  if (splits > cap) splits = cap;
  if (splits < 1) splits = 1;
  if (splits > 64) splits = 64;
  sh.n_splits = (int)splits;
  return sh;
}

}  // namespace

size_t attend_workspace(const msa_attend_args& a, int* n_splits_out) {
  Shape sh = plan(a);
  if (n_splits_out) *n_splits_out = sh.n_splits;
  size_t b = align_up((size_t)a.n_q * a.hq * kHeadDim * 4, 256);
  b += align_up((size_t)(sh.n_loc > 0 ? sh.n_loc : 1) * a.hkv * kHeadDim * 4, 256);
  if (sh.n_splits > 1) {
    b += align_up((size_t)a.n_q * a.hq * sh.n_splits * kHeadDim * 4, 256);
    b += align_up((size_t)a.n_q * a.hq * sh.n_splits * 8, 256);
  }
  return b;
}

msa_status launch_attend(const msa_attend_args& a, void* ws, cudaStream_t st) {
  Shape sh = plan(a);
  AttnParams P{};  // kernel parameter block (4.3 KB: large kernel parameters, CUDA >= 12.1)
  P.q = a.q; P.k_loc = a.k_loc; P.v_loc = a.v_loc; P.mem_k = a.mem_k; P.mem_v = a.mem_v;
  P.sel_off = a.sel_off; P.sel_chunk = a.sel_chunk;
  char* w = reinterpret_cast<char*>(ws);
  P.qrot = reinterpret_cast<float*>(w);
  w += align_up((size_t)a.n_q * a.hq * kHeadDim * 4, 256);
  P.krot = reinterpret_cast<float*>(w);
  w += align_up((size_t)(sh.n_loc > 0 ? sh.n_loc : 1) * a.hkv * kHeadDim * 4, 256);
  P.part_o = reinterpret_cast<float*>(w);
  if (sh.n_splits > 1) w += align_up((size_t)a.n_q * a.hq * sh.n_splits * kHeadDim * 4, 256);
  P.part_ml = reinterpret_cast<float2*>(w);
  P.out = a.out; P.out_f32 = a.out_f32; P.lse = a.lse;
  P.n_seq = a.n_seq; P.n_q = a.n_q; P.n_loc = sh.n_loc; P.hq = a.hq; P.hkv = a.hkv;
  P.group = a.hq / a.hkv; P.rt = sh.rt; P.n_splits = sh.n_splits; P.n_tiles = sh.n_tiles;
  P.scale = a.scale > 0.f ? a.scale : 1.0f / sqrtf((float)kHeadDim);
  P.pos_offset = (double)a.pos_offset;
  P.log2_theta = log2((double)a.rope_theta);
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

  int64_t nq = (int64_t)a.n_q * a.hq * 64;
  rope_rows_kernel<<<(unsigned)((nq + 255) / 256), 256, 0, st>>>(P, 0);
  msa_status s = launch_check("attend: rotate queries");
  if (s != MSA_OK) return s;
  if (sh.n_loc > 0) {
    int64_t nk = (int64_t)sh.n_loc * a.hkv * 64;
    rope_rows_kernel<<<(unsigned)((nk + 255) / 256), 256, 0, st>>>(P, 1);
    s = launch_check("attend: rotate local keys");
    if (s != MSA_OK) return s;
  }
  dim3 grid((unsigned)sh.n_splits, (unsigned)a.hkv, (unsigned)sh.n_tiles);
  attend_split_kernel<<<grid, kThreads, 0, st>>>(P);
  s = launch_check("attend: split-K");
  if (s != MSA_OK || sh.n_splits == 1) return s;
  attend_merge_kernel<<<(unsigned)(a.n_q * a.hq), kHeadDim, 0, st>>>(P);
  return launch_check("attend: merge");
}

}  // namespace msa
