// Sparse attention for a few query rows per sequence (decoding), on the
// tensor cores with the operands swapped.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — the pooled
// K/V of the selected documents joined to the K/V of the query's recent context;
// Parallel (document-wise) RoPE and Global RoPE offset by k (Figure 2)]
//
// Same result as the split-K kernel in attend.cu. A decoding CTA holds at most
// 16 query vectors (its rows x the GQA group's q heads) of one kv head, too
// few to fill an M = 128 tile, so the keys take the M side instead:
//   S^T = K Q^T     tcgen05 M128 (keys) x N16 (vectors) x K128 (dims),
//   softmax         per vector over the TMEM lanes (keys): each thread holds
//                   one key's 16 logits; block maxima by warp shuffles and a
//                   4-warp exchange, running sums per thread, P^T to shared
//                   memory as bf16 (the B operand: vectors x keys),
//   O^T += V^T P^T  tcgen05 M128 (dims) x N16 (vectors) x K128 (keys),
//                   accumulated in TMEM across blocks against a reference max
//                   that moves only when the running max passes it by more
//                   than 2^11.5 (then the columns of O^T are rescaled).
// Keys come in blocks of 128: the pooled memory rows by cp.async straight
// into the 128-byte-swizzled K-major layout (one DRAM round trip per block),
// the rotated fp32 local keys and queries as bf16 high + low parts (S sums
// Khi Qhi + Khi Qlo + Klo Qhi), V transposed through registers. Key ranges are
// split across CTAs as in the split-K kernel, with the same last-CTA merge
// (here in log2 units). Every mbarrier wait is bounded in time, and every
// warp is reconverged (__all_sync) after it.
#include <cuda.h>

#include "attend_params.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

using namespace tc;

constexpr int kDN = 16;          // query vectors per CTA (MMA N), padded with zeros
constexpr int kDK = 128;         // keys per block (M of S^T, K of O^T)
constexpr int kDThreads = 128;   // 4 warps = the 4 TMEM lane quadrants
constexpr int kKAtomD = kDK * 128;  // 16 KB: 128 keys x 64 dims (bf16)
constexpr int kQAtomD = kDN * 128;  // 2 KB: 16 vectors x 64 dims
constexpr int kVAtomD = 128 * 128;  // 16 KB: 128 dims x 64 keys
constexpr int kPAtomD = kDN * 128;  // 2 KB: 16 vectors x 64 keys
constexpr int offKhi = 0;                     // 2 atoms: dims 0-63, 64-127
constexpr int offKlo = offKhi + 2 * kKAtomD;  // 2 atoms (local keys only)
constexpr int offVT = offKlo + 2 * kKAtomD;   // 2 atoms: keys 0-63, 64-127
constexpr int offQhi = offVT + 2 * kVAtomD;   // 2 atoms: dims 0-63, 64-127
constexpr int offQlo = offQhi + 2 * kQAtomD;
constexpr int offP = offQlo + 2 * kQAtomD;    // 2 atoms: keys 0-63, 64-127
constexpr int offIdx = offP + 2 * kPAtomD;    // 128 bank rows (int64)
constexpr int offRed = offIdx + kDK * 8;      // [4 warps][16] reduction scratch
constexpr int offMref = offRed + 4 * kDN * 4; // [16] reference max per vector (log2 units)
constexpr int offCorr = offMref + kDN * 4;    // [16] this block's rescale factor per vector
constexpr int offBar = offCorr + kDN * 4;     // mbarrier, TMEM slot, abort flag
constexpr int kSmemDec = 1024 + offBar + 64;
constexpr int kTmemColsDec = 32;  // S^T: columns 0..15, O^T: columns 16..31
// D fp32, A/B bf16, both K-major; N = 16, M = 128
constexpr uint32_t kIdescDec = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kDN >> 3) << 17) | (8u << 24);
static_assert(offBar % 8 == 0, "mbarrier alignment");
static_assert(offQhi % 1024 == 0 && offQlo % 1024 == 0 && offP % 1024 == 0, "swizzle atom alignment");

// 16-byte piece c (0..7) of row r of a 128-byte-swizzled K-major atom.
__device__ __forceinline__ uint8_t* swz_d(uint8_t* atom, int r, int c) {
  return atom + r * 128 + ((c ^ (r & 7)) << 4);
}

__device__ __forceinline__ float bf_round_d(float x) { return __uint_as_float(f2bf_bits(x) << 16); }

// Eight fp32 values -> 16-byte bf16 high part and 16-byte bf16 remainder.
__device__ __forceinline__ void split8_d(const float* x, uint4& hi, uint4& lo) {
  float h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = bf_round_d(x[i]);
    l[i] = x[i] - h[i];
  }
  hi = make_uint4(pack_bf2(h[0], h[1]), pack_bf2(h[2], h[3]), pack_bf2(h[4], h[5]), pack_bf2(h[6], h[7]));
  lo = make_uint4(pack_bf2(l[0], l[1]), pack_bf2(l[2], l[3]), pack_bf2(l[4], l[5]), pack_bf2(l[6], l[7]));
}

__device__ __forceinline__ void cp_async16(uint8_t* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__global__ void __launch_bounds__(kDThreads, 1) attend_dec_tc_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int64_t* s_idx = reinterpret_cast<int64_t*>(smem + offIdx);
  float* s_red = reinterpret_cast<float*>(smem + offRed);
  float* s_mref = reinterpret_cast<float*>(smem + offMref);
  float* s_corr = reinterpret_cast<float*>(smem + offCorr);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + offBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sp_idx = blockIdx.x, kvh = blockIdx.y, tile = blockIdx.z;
  const int s = seq_of(p.tile_off, p.n_seq, tile);
  const int row0 = p.q_seq_off[s] + (tile - p.tile_off[s]) * p.rt;
  const int nr = min(p.rt, p.q_seq_off[s + 1] - row0);
  const int g0 = p.q_start[s] + (row0 - p.q_seq_off[s]);  // active index of the tile's first row
  const int n_loc_s = p.loc_off[s + 1] - p.loc_off[s];
  const int lvis = max(0, min(n_loc_s, g0 + nr));  // local keys visible to the last row
  const int nvec = nr * p.group;                    // valid query vectors (<= 16)
  const size_t row_stride = (size_t)p.hkv * kHeadDim;

  if (tid == 0) {
    mbar_init(smem_u32(bar), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid < kDN) s_mref[tid] = -INFINITY;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)kTmemColsDec));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  pdl_wait();  // the rotated rows and the selection come from earlier kernels
  pdl_trigger();
  const int64_t mem_base = __ldg(p.sel_off + s);
  const int64_t n_mem = __ldg(p.sel_off + s + 1) - mem_base;
  const int64_t n_keys = n_mem + lvis;
  const int64_t per = (n_keys + p.n_splits - 1) / p.n_splits;
  const int64_t k_begin = (int64_t)sp_idx * per;
  const int64_t k_end = min(n_keys, k_begin + per);

  // ---- Q^T operand (vectors x dims), high and low parts; vectors past nvec are zero
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int id = tid + kDThreads * u;  // 256 pieces: 16 vectors x 16 pieces of 8 dims
    const int vr = id >> 4, c16 = id & 15;
    float f[8];
    if (vr < nvec) {
      const int rr = vr / p.group, gg = vr % p.group;
      const float4* qv = reinterpret_cast<const float4*>(
          p.qrot + ((size_t)(row0 + rr) * p.hq + kvh * p.group + gg) * kHeadDim + 8 * c16);
      const float4 a = __ldg(qv), b = __ldg(qv + 1);
      f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = 0.f;
    }
    uint4 hi, lo;
    split8_d(f, hi, lo);
    *reinterpret_cast<uint4*>(swz_d(smem + offQhi + (c16 >> 3) * kQAtomD, vr, c16 & 7)) = hi;
    *reinterpret_cast<uint4*>(swz_d(smem + offQlo + (c16 >> 3) * kQAtomD, vr, c16 & 7)) = lo;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
  const uint32_t tmem_s = tmem, tmem_o = tmem + kDN;

  float l_part[kDN];  // this thread's keys' share of each vector's sum (relative to s_mref)
#pragma unroll
  for (int v = 0; v < kDN; ++v) l_part[v] = 0.f;
  uint32_t phase = 0;
  bool ok = true, pv_pending = false;
  int blk = 0;
  const float sl2 = p.scale * 1.4426950408889634f;  // logits in log2 units

  for (int64_t kb = k_begin; kb < k_end; kb += kDK, ++blk) {
    const int nb = (int)min((int64_t)kDK, k_end - kb);
    const bool has_local = kb + nb > n_mem;
    if (pv_pending) {  // the previous block's P.V still reads V^T and P
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), phase, abort_flag));
      phase ^= 1;
      pv_pending = false;
      if (!__syncthreads_and(ok)) { ok = false; break; }
      tc_fence_after();
    }
    if (tid < nb && kb + tid < n_mem)
      s_idx[tid] = p.sel_chunk ? __ldg(p.sel_chunk + mem_base + kb + tid) : mem_base + kb + tid;
    __syncthreads();

    // ---- K (keys x dims): memory rows by cp.async, local rows split into high and low parts
#pragma unroll 4
    for (int u = 0; u < 16; ++u) {
      const int id = tid + kDThreads * u;  // 2048 pieces: 128 keys x 16 pieces of 8 dims
      const int jj = id >> 4, c16 = id & 15;
      const int64_t key = kb + jj;
      uint8_t* dhi = swz_d(smem + offKhi + (c16 >> 3) * kKAtomD, jj, c16 & 7);
      uint8_t* dlo = swz_d(smem + offKlo + (c16 >> 3) * kKAtomD, jj, c16 & 7);
      if (jj < nb && key < n_mem) {
        cp_async16(dhi, p.mem_k + (size_t)s_idx[jj] * row_stride + (size_t)kvh * kHeadDim + 8 * c16);
        if (has_local) *reinterpret_cast<uint4*>(dlo) = make_uint4(0, 0, 0, 0);
      } else if (jj < nb) {
        const float4* kr = reinterpret_cast<const float4*>(
            p.krot + ((size_t)(p.loc_off[s] + (key - n_mem)) * p.hkv + kvh) * kHeadDim + 8 * c16);
        const float4 a = __ldg(kr), b = __ldg(kr + 1);
        const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint4 hi, lo;
        split8_d(f, hi, lo);
        *reinterpret_cast<uint4*>(dhi) = hi;
        *reinterpret_cast<uint4*>(dlo) = lo;
      } else {
        *reinterpret_cast<uint4*>(dhi) = make_uint4(0, 0, 0, 0);
        if (has_local) *reinterpret_cast<uint4*>(dlo) = make_uint4(0, 0, 0, 0);
      }
    }
    // ---- V^T (dims x keys): key pair jp (keys 2 jp, 2 jp + 1) x dims 16 dg .. 16 dg + 15
#pragma unroll 1
    for (int u = 0; u < 4; ++u) {
      const int id = tid + kDThreads * u;  // 512 items: 64 key pairs x 8 groups of 16 dims
      const int jp = id & 63, dg = id >> 6;
      uint4 x[2][2];
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        const int jj = 2 * jp + k2;
        const int64_t key = kb + jj;
        const uint16_t* vrow = nullptr;
        if (jj < nb && key < n_mem)
          vrow = p.mem_v + (size_t)s_idx[jj] * row_stride + (size_t)kvh * kHeadDim;
        else if (jj < nb)
          vrow = p.v_loc + ((size_t)(p.loc_off[s] + (key - n_mem)) * p.hkv + kvh) * kHeadDim;
#pragma unroll
        for (int i = 0; i < 2; ++i)
          x[k2][i] = vrow ? __ldg(reinterpret_cast<const uint4*>(vrow + 16 * dg) + i) : make_uint4(0, 0, 0, 0);
      }
      uint8_t* atom = smem + offVT + (jp >> 5) * kVAtomD;  // keys 0-63 or 64-127
      const int jpl = jp & 31;                             // pair within the atom's 64 keys
#pragma unroll
      for (int d = 0; d < 16; ++d) {
        const uint4& a = x[0][d >> 3];
        const uint4& b = x[1][d >> 3];
        const int w = (d >> 1) & 3;
        const uint32_t wa = w == 0 ? a.x : w == 1 ? a.y : w == 2 ? a.z : a.w;
        const uint32_t wb = w == 0 ? b.x : w == 1 ? b.y : w == 2 ? b.z : b.w;
        *reinterpret_cast<uint32_t*>(swz_d(atom, 16 * dg + d, jpl >> 2) + 4 * (jpl & 3)) =
            __byte_perm(wa, wb, (d & 1) ? 0x7632 : 0x5410);
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();  // the MMAs read these bytes through the async proxy
    tc_fence_before();
    __syncthreads();

    // ---- S^T = K Q^T
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t ko = (uint32_t)((k >> 2) * kKAtomD + (k & 3) * 32);
        const uint32_t qo = (uint32_t)((k >> 2) * kQAtomD + (k & 3) * 32);
        const uint64_t dk = sw128_desc(smem_u32(smem + offKhi) + ko);
        const uint64_t dqh = sw128_desc(smem_u32(smem + offQhi) + qo);
        tc_mma(tmem_s, dk, dqh, kIdescDec, k > 0 ? 1u : 0u);
        tc_mma(tmem_s, dk, sw128_desc(smem_u32(smem + offQlo) + qo), kIdescDec, 1u);
        if (has_local) tc_mma(tmem_s, sw128_desc(smem_u32(smem + offKlo) + ko), dqh, kIdescDec, 1u);
      }
      tc_commit(smem_u32(bar));
    }
    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), phase, abort_flag));
    phase ^= 1;
    if (!__syncthreads_and(ok)) { ok = false; break; }
    tc_fence_after();

    // ---- softmax over the keys (TMEM lanes) of each vector (column)
    float sv[kDN];
    tmem_ld16(tmem_s + lane_base, sv);
    tmem_ld_wait();
    const int64_t key = kb + tid;
    const int lj = key < n_mem ? -1 : (int)(key - n_mem);  // local key index, or -1
#pragma unroll
    for (int v = 0; v < kDN; ++v) {
      const bool vis = tid < nb && v < nvec && (lj < 0 || lj <= g0 + v / p.group);
      sv[v] = vis ? sv[v] * sl2 : -INFINITY;
    }
#pragma unroll
    for (int v = 0; v < kDN; ++v) {
      float m = sv[v];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) s_red[warp * kDN + v] = m;
    }
    __syncthreads();
    bool move = false;
    if (tid < kDN) {
      const float bm = fmaxf(fmaxf(s_red[tid], s_red[kDN + tid]), fmaxf(s_red[2 * kDN + tid], s_red[3 * kDN + tid]));
      const float mref = s_mref[tid];
      move = bm > mref + 11.5f;  // 2^11.5 ~ e^8; also when mref is -inf and bm finite
      s_corr[tid] = !move ? 1.f : (mref == -INFINITY ? 0.f : exp2f(mref - bm));
      if (move) s_mref[tid] = bm;
    }
    const bool any_move = __syncthreads_or(move);
    uint8_t* patom = smem + offP + (tid >> 6) * kPAtomD;  // this key's 64-key atom of P
#pragma unroll
    for (int v = 0; v < kDN; ++v) {
      const float mr = s_mref[v] == -INFINITY ? 0.f : s_mref[v];  // all P are 0 then (2^-inf)
      const float pr = exp2f(sv[v] - mr);
      l_part[v] = l_part[v] * s_corr[v] + pr;
      *reinterpret_cast<uint16_t*>(swz_d(patom, v, (tid & 63) >> 3) + 2 * (tid & 7)) = (uint16_t)f2bf_bits(pr);
    }
    if (blk > 0 && any_move) {  // rescale the columns of O^T (this thread's dimension row)
      float t[kDN];
      tmem_ld16(tmem_o + lane_base, t);
      tmem_ld_wait();
#pragma unroll
      for (int v = 0; v < kDN; ++v) t[v] *= s_corr[v];
      tmem_st16(tmem_o + lane_base, t);
      tmem_st_wait();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O^T += V^T P^T (accumulated in TMEM; waited for before V^T and P are reused)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < kDK / 16; ++k) {
        const uint32_t vo = (uint32_t)((k >> 2) * kVAtomD + (k & 3) * 32);
        const uint32_t po = (uint32_t)((k >> 2) * kPAtomD + (k & 3) * 32);
        tc_mma(tmem_o, sw128_desc(smem_u32(smem + offVT) + vo), sw128_desc(smem_u32(smem + offP) + po), kIdescDec,
               (blk > 0 || k > 0) ? 1u : 0u);
      }
      tc_commit(smem_u32(bar));
    }
    pv_pending = true;
  }
  if (ok && pv_pending) {
    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(bar), phase, abort_flag));
    phase ^= 1;
    ok = __syncthreads_and(ok);
  }
  if (!ok && tid == 0) {  // a wait ran out: let the MMAs in flight finish (bounded) before TMEM is freed
    const uint64_t t0 = globaltimer();
    while (!mbar_try(smem_u32(bar), phase ^ 1) && globaltimer() - t0 < kWaitLimitNs) {
    }
  }
  tc_fence_after();

  // ---- each vector's sum over the 128 key lanes
  __syncthreads();  // s_red is reused
#pragma unroll
  for (int v = 0; v < kDN; ++v) {
    float a = l_part[v];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) s_red[warp * kDN + v] = a;
  }
  __syncthreads();
  float o_row[kDN];  // this thread's dimension (TMEM lane) of every vector's output
  if (ok && blk > 0) {  // uniform: every thread of the CTA walked the same blocks
    tmem_ld16(tmem_o + lane_base, o_row);
    tmem_ld_wait();
  } else {
#pragma unroll
    for (int v = 0; v < kDN; ++v) o_row[v] = 0.f;
  }
  const int d = tid;

  if (p.n_splits > 1) {
    // ---- split-K: unnormalised partial (o, m, l) out; the last CTA of the
    // (tile, kv head) merges by log-sum-exp (log2 units)
    __shared__ int s_last;
#pragma unroll
    for (int v = 0; v < kDN; ++v) {  // unrolled: o_row stays in registers
      if (v >= nvec) break;
      const int rr = v / p.group, gg = v % p.group;
      const size_t rh = (size_t)(row0 + rr) * p.hq + kvh * p.group + gg;
      const size_t pi = rh * p.n_splits + sp_idx;
      const float l = s_red[v] + s_red[kDN + v] + s_red[2 * kDN + v] + s_red[3 * kDN + v];
      p.part_o[pi * kHeadDim + d] = ok ? o_row[v] : 0.f;
      if (d == 0) p.part_ml[pi] = make_float2(s_mref[v], ok ? l : 0.f);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(p.tickets + (size_t)tile * p.hkv + kvh, 1u) == (unsigned)(p.n_splits - 1);
    __syncthreads();
    if (s_last) {
      __threadfence();
      for (int v = 0; v < nvec; ++v) {
        const int rr = v / p.group, gg = v % p.group;
        const size_t rh = (size_t)(row0 + rr) * p.hq + kvh * p.group + gg;
        float mm = -INFINITY;
        for (int j = 0; j < p.n_splits; ++j) {
          const float2 x = __ldcg(p.part_ml + rh * p.n_splits + j);
          if (x.y > 0.f) mm = fmaxf(mm, x.x);
        }
        float wsum = 0.f, r = 0.f;
        for (int j = 0; j < p.n_splits; ++j) {
          const float2 x = __ldcg(p.part_ml + rh * p.n_splits + j);
          if (!(x.y > 0.f)) continue;
          const float w = exp2f(x.x - mm);
          wsum += x.y * w;
          r += w * __ldcg(p.part_o + (rh * p.n_splits + j) * kHeadDim + d);
        }
        r = wsum > 0.f ? r / wsum : 0.f;
        p.out[rh * kHeadDim + d] = (uint16_t)f2bf_bits(r);
        if (p.out_f32) p.out_f32[rh * kHeadDim + d] = r;
        if (p.lse && d == 0) p.lse[rh] = wsum > 0.f ? (mm + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
      }
    }
  } else if (ok) {  // ---- one CTA per (tile, kv head): normalised output, log-sum-exp
#pragma unroll
    for (int v = 0; v < kDN; ++v) {
      if (v >= nvec) break;
      const int rr = v / p.group, gg = v % p.group;
      const size_t rh = (size_t)(row0 + rr) * p.hq + kvh * p.group + gg;
      const float l = s_red[v] + s_red[kDN + v] + s_red[2 * kDN + v] + s_red[3 * kDN + v];
      const float r = l > 0.f ? o_row[v] / l : 0.f;
      p.out[rh * kHeadDim + d] = (uint16_t)f2bf_bits(r);
      if (p.out_f32) p.out_f32[rh * kHeadDim + d] = r;
      if (p.lse && d == 0) p.lse[rh] = l > 0.f ? (s_mref[v] + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTmemColsDec));
  }
}

}  // namespace

msa_status launch_attend_dec_tc(const AttnParams& P, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  cudaError_t e = smem_limit_once(attend_dec_tc_kernel, kSmemDec, attr);
  if (e != cudaSuccess) return cuda_fail(e, "attend: decoding tensor-core kernel shared memory");
  e = launch_pdl(attend_dec_tc_kernel, dim3((unsigned)P.n_splits, (unsigned)P.hkv, (unsigned)P.n_tiles),
                             dim3(kDThreads), (size_t)kSmemDec, st, P);
  if (e != cudaSuccess) return cuda_fail(e, "attend: tensor cores (decoding)");
  return launch_check("attend: tensor cores (decoding)");
}

int attend_dec_tc_error_take() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof v) != cudaSuccess) return 0;
  if (v) {
    int z = 0;
    cudaMemcpyToSymbol(g_tc_error, &z, sizeof z);
  }
  return v;
}

}  // namespace msa
