// Sparse attention for decoding shapes: a few query rows per sequence, so a
// tile holds the GQA group's q heads x rows = at most 16 query vectors of one
// kv head.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — the pooled
// K/V of the selected documents joined to the K/V of the query's recent context;
// Parallel (document-wise) RoPE and Global RoPE offset by k (Figure 2)]
//
// Same result as the other attention kernels. A decoding step attends over a
// few hundred keys per head (a few MB per layer at 4 flop per byte), so its
// time is the chain of dependent memory round trips plus the latency of the
// instructions each warp issues; neither bandwidth nor arithmetic throughput
// bounds it. The kernel keeps that chain short, and is the call's only kernel:
//  - A CTA (one per SM) owns one kv head, one tile of query vectors and one
//    split of the key list: an even share of the sequence's memory keys (the
//    selected pooled rows) and of its local keys (the recent context).
//  - When its share of the local keys is small, the CTA rotates them
//    (global positions offset by k) and its query vectors itself, as bf16
//    high and low halves (so the logits keep fp32 accuracy), while the first
//    memory rows are already in flight; local steps come first, so those keys
//    go straight into the shared-memory stages that will compute them. With a
//    larger share, rope_rows (a kernel of its own that spreads the work over
//    the whole GPU) rotates the queries and local keys before the kernel, and
//    the keys are copied like the rest.
//    In the routed form the CTA lists the memory rows itself: the chunk
//    ranges of the sequence's selected documents, scanned in shared memory.
//  - Inside the CTA every warp is an independent flash-decoding worker: the
//    share is cut into steps of 16 keys and warp w takes steps w, w + 8, ...
//    Each warp copies its own steps' rows by cp.async into its own two
//    shared-memory stages (the next step in flight while one is computed; a
//    key's bank row is looked up a step before its copy), keeps its own
//    running max, sum and output, and synchronises with no other warp until
//    the end.
//  - A step is two warp-level bf16 MMA chains (m16n8k16, fp32 accumulate), the
//    16-vector tile as M: S = Q K^T (queries split into bf16 high + low parts,
//    local keys too), then O += P V with P taken straight from S's
//    accumulators as the A operand (rounded to bf16).
//  - At the end the 8 warps' (o, m, l) are merged through shared memory; the
//    splits of a (tile, kv head) are one thread-block cluster, whose CTAs then
//    share out the outputs and merge the splits' partials by log-sum-exp
//    straight from each other's shared memory (no partials in HBM, no
//    counters to clear between calls).
#include <math.h>

#include "attend_params.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

constexpr int kDThreads = 256;                     // 8 warps
constexpr int kDWarps = kDThreads / 32;
constexpr int kStepKeys = 16;                      // keys per warp step (the K of P.V)
constexpr int kRowB = 272;                         // bytes per staged bf16 row (256 + 16)
constexpr int kTileV = 16;                         // query vectors per tile (MMA M)
constexpr int offSK = 0;                           // within a stage: keys (bf16, or the high halves)
constexpr int offSL = offSK + kStepKeys * kRowB;   // low halves of local keys
constexpr int offSV = offSL + kStepKeys * kRowB;   // values
constexpr int kStageB = offSV + kStepKeys * kRowB; // 13,056 B
constexpr int kWarpB = 2 * kStageB;                // two stages per warp
constexpr int offQhi = kDWarps * kWarpB;           // queries [16][272 B], high and low parts
constexpr int offQlo = offQhi + kTileV * kRowB;
constexpr int kDecSmem = offQlo + kTileV * kRowB;  // 217,600 B
// end-of-CTA merge, over the warps' stages: o [8 warps][16][132] fp32 (rows padded: the
// fragment stores of a warp hit distinct banks), then m, l [8][16]
constexpr int kMRow = kHeadDim + 4;
constexpr int offMO = 0;
constexpr int offMM = offMO + kDWarps * kTileV * kMRow * 4;
constexpr int offMLs = offMM + kDWarps * kTileV * 4;
// then this CTA's merged partial for the cluster merge: o [16][128] (unnormalised), m, l [16]
constexpr int offPO = offMLs + kDWarps * kTileV * 4;
constexpr int offPM = offPO + kTileV * kHeadDim * 4;
constexpr int offPL = offPM + kTileV * 4;
static_assert(offPL + kTileV * 4 <= offQhi, "the merge fits the stages");
constexpr int kLocRowB = 2 * kHeadDim * 2;  // a local key rotated by rope_rows: high, then low halves
constexpr int kRotBatch = 4;                // local-key rotations per thread whose loads go out first
static_assert(kDecSmem <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ uint32_t saddr(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
// D += A B for one m16n8k16 tile (A row-major 16x16, B column-major 16x8), bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two floats to bf16 (round to nearest even) in one conversion: lo in bits 0-15, hi in 16-31.
__device__ __forceinline__ uint32_t cvt_bf2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// x split into bf16 parts: x ~ h + l, h = bf16(x), l = bf16(x - h); a pair per call, packed.
__device__ __forceinline__ void split_bf2(float x0, float x1, uint32_t& h, uint32_t& l) {
  h = cvt_bf2(x0, x1);
  l = cvt_bf2(x0 - bf_lo(h), x1 - bf_hi(h));
}

// ---- thread-block cluster: the splits of one (tile, kv head)
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a float in the shared memory of cluster CTA `rank`, at this CTA's address `local` of the same variable
__device__ __forceinline__ float ld_cluster_f32(uint32_t local, uint32_t rank) {
  uint32_t a;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}

// RoPE of one pair (x0 = dim i, x1 = dim i + 64) at position pos (pair frequency f). The
// angle is formed and reduced to [-pi, pi] in double; on that range the hardware sine and
// cosine (__sincosf) are within 2^-21.4 absolute, well under the 2^-17 relative precision of
// the bf16 high + low parts the results are stored in.
__device__ __forceinline__ void rope_pair(float x0, float x1, double pos, double f, float& y0, float& y1) {
  float sn, cs;
  __sincosf(reduced_angle(pos * f), &sn, &cs);
  y0 = x0 * cs - x1 * sn;
  y1 = x0 * sn + x1 * cs;
}

// One 256-byte row by the bulk-copy engine, its bytes counted on the stage's mbarrier.
__device__ __forceinline__ void bulk_row(uint32_t dst, const void* src, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], 256, [%2];"
               ::"r"(dst), "l"(src), "r"(bar) : "memory");
}

// BULK: each of lanes 0-15 moves its own key's rows with one bulk copy per row
// (completion counted on the warp's stage mbarrier) instead of the warp moving
// every row in 16-byte cp.async pieces.
template <bool BULK>
__global__ void __launch_bounds__(kDThreads, 1) attend_dec_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ int64_t s_pre[kDecRoutedMaxK + 1];  // routed form: first list position of each document
  __shared__ int64_t s_c0[kDecRoutedMaxK];       // ... and its first chunk
  __shared__ int64_t s_wsum[kDWarps];
  __shared__ uint64_t s_bar[kDWarps][2];  // BULK: each warp's two stages
  __shared__ int s_abort;
  __shared__ double s_invf[kHeadDim / 2];         // RoPE frequency of each pair

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int g = lane >> 2, c = lane & 3;  // MMA fragment coordinates
  const int sp = blockIdx.x, kvh = blockIdx.y, tile = blockIdx.z;
  const int s = seq_of(p.tile_off, p.n_seq, tile);
  const int row0 = p.q_seq_off[s] + (tile - p.tile_off[s]) * p.rt;
  const int nr = min(p.rt, p.q_seq_off[s + 1] - row0);
  const int nvec = nr * p.group;                           // valid query vectors (<= 16)
  const int g0 = p.q_start[s] + (row0 - p.q_seq_off[s]);  // active index of the tile's first row
  const int n_loc_s = p.loc_off[s + 1] - p.loc_off[s];
  const int lvis = max(0, min(n_loc_s, g0 + nr));          // local keys visible to the tile's last row
  const size_t row_stride = (size_t)p.hkv * kHeadDim;
  const float sl2 = p.scale * 1.4426950408889634f;         // logits in log2 units
  // active-context index of MMA rows g and g + 8 (-1: padding, sees nothing)
  const int ga = g < nvec ? g0 + g / p.group : -1;
  const int gb = g + 8 < nvec ? g0 + (g + 8) / p.group : -1;

  if constexpr (BULK) {
    if (tid == 0) s_abort = 0;
    if (lane == 0) {
      tc::mbar_init(tc::smem_u32(&s_bar[w][0]), 1);
      tc::mbar_init(tc::smem_u32(&s_bar[w][1]), 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
  }
  pdl_wait();  // the selection comes from an earlier kernel
  pdl_trigger();

  // ---- this split's share of the local keys [l0, l1) (known from the host's offsets): local
  // steps come first, so that a CTA's first 16 local steps are its warps' first two steps and
  // their rotated keys go straight into those stages
  const int pl = (lvis + p.n_splits - 1) / p.n_splits;
  const int l0 = min(lvis, sp * pl), l1 = min(lvis, l0 + pl);
  const int nsl = (l1 - l0 + kStepKeys - 1) / kStepKeys;  // local steps

  // loads that depend on nothing in flight go out first: the query tile (16 vectors
  // v = rr * group + gg, past nvec zero; thread -> vector qv_v, dims qv_d0 .. qv_d0 + 7, its
  // rotation partners, dims +- 64, held by lane ^ 8), the first batch of the local keys to
  // rotate (thread -> key, dims 2j, 2j + 1 and their partners + 64), and the frequencies
  if (tid < kHeadDim / 2) s_invf[tid] = p.inv_freq[tid];
  const int qv_v = tid >> 4, qv_d0 = 8 * (tid & 15);
  uint4 qraw = make_uint4(0, 0, 0, 0);
  float4 qra = make_float4(0.f, 0.f, 0.f, 0.f), qrb = qra;  // rotated by rope_rows (rope_q)
  if (qv_v < nvec) {
    const int rr = qv_v / p.group, gg = qv_v - rr * p.group;
    const size_t qi = ((size_t)(row0 + rr) * p.hq + kvh * p.group + gg) * kHeadDim + qv_d0;
    if (p.rope_q) {
      qra = __ldcg(reinterpret_cast<const float4*>(p.qrot + qi));
      qrb = __ldcg(reinterpret_cast<const float4*>(p.qrot + qi + 4));
    } else {
      qraw = __ldcg(reinterpret_cast<const uint4*>(p.q + qi));
    }
  }
  const int nrot = p.rot_in_kernel ? (l1 - l0) * 32 : 0;  // at most 16 steps' keys (the host sees to it)
  auto kloc_ptr = [&](int it) {
    return p.k_loc + ((size_t)(p.loc_off[s] + l0 + (it >> 5)) * p.hkv + kvh) * kHeadDim + 2 * (it & 31);
  };
  uint32_t ka[kRotBatch], kb2[kRotBatch];
#pragma unroll
  for (int u = 0; u < kRotBatch; ++u) {
    const int it = tid + u * kDThreads;
    if (it < nrot) {
      ka[u] = __ldcg(reinterpret_cast<const unsigned int*>(kloc_ptr(it)));
      kb2[u] = __ldcg(reinterpret_cast<const unsigned int*>(kloc_ptr(it) + 64));
    }
  }

  // ---- the sequence's memory rows: the gather listing (sel_off, sel_chunk), or in the
  // routed form the chunks of its selected documents in rank order
  const bool routed = p.sel_off == nullptr;
  int64_t mem_base = 0, n_mem;
  if (routed) {
    int64_t c0 = 0, cnt = 0;
    if (tid < p.top_k) {
      const int32_t doc = __ldcg(p.top_ids + (size_t)s * p.top_k + tid);
      if (doc >= 0 && doc < p.n_docs) {
        c0 = __ldcg(p.doc_chunk_off + doc);
        cnt = __ldcg(p.doc_chunk_off + doc + 1) - c0;
      }
    }
    int64_t x = cnt;  // inclusive scan over the block (top_k <= 256 = its threads)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) s_wsum[w] = x;
    __syncthreads();
    for (int j = 0; j < w; ++j) x += s_wsum[j];
    if (tid < p.top_k) {
      s_pre[tid] = x - cnt;
      s_c0[tid] = c0;
    }
    if (tid == p.top_k - 1) s_pre[p.top_k] = x;
    __syncthreads();
    n_mem = min(s_pre[p.top_k], p.max_sel);
  } else {
    mem_base = __ldcg(p.sel_off + s);
    n_mem = __ldcg(p.sel_off + s + 1) - mem_base;
  }

  // ---- this split's share of the memory keys [m0, m1): the steps after the local ones
  const int64_t pm = (n_mem + p.n_splits - 1) / p.n_splits;
  const int64_t m0 = min(n_mem, (int64_t)sp * pm), m1 = min(n_mem, m0 + pm);
  const int nsteps = nsl + (int)((m1 - m0 + kStepKeys - 1) / kStepKeys);

  // ---- this warp's steps w, w + 8, ...: lane kl < 16 looks up the row of key kl of a step;
  // copy instruction u then moves rows 2u and 2u + 1 whole (lanes 0-15 and 16-31, 16 B each),
  // so every instruction reads two contiguous 256-byte rows
  const int kl = lane & 15;
  uint8_t* wst = sm + w * kWarpB;
  auto row_of = [&](int i) -> int64_t {  // local key or bank row (memory) of key kl in step i; -1: none
    if (i >= nsteps) return -1;
    if (i < nsl) {
      const int key = l0 + i * kStepKeys + kl;
      return key < l1 ? (int64_t)key : -1;
    }
    const int64_t key = m0 + (int64_t)(i - nsl) * kStepKeys + kl;
    if (key >= m1) return -1;
    if (!routed) return p.sel_chunk ? __ldcg(p.sel_chunk + mem_base + key) : mem_base + key;
    int lo = 0, hi = p.top_k - 1;  // the last document whose first list position is <= key
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= key) lo = mid; else hi = mid - 1;
    }
    return s_c0[lo] + (key - s_pre[lo]);
  };
  // k_in_place: the step's local keys are rotated straight into the stage (the warp's first two
  // steps in the in-kernel rotation mode, which has at most 16 local steps), so only V is copied
  auto issue = [&](int i, int64_t r_mine, int stage, bool k_in_place) {
    if constexpr (BULK) {
      if (i < nsteps) {
        uint8_t* stg = wst + stage * kStageB;
        const bool loc = i < nsl;
        const uint32_t bar = tc::smem_u32(&s_bar[w][stage]);
        const int rows = (loc ? (k_in_place ? 1 : 3) : 2);  // 256-byte rows per valid key
        const unsigned vm = __ballot_sync(0xffffffffu, lane < kStepKeys && r_mine >= 0);
        if (lane == 0) tc::mbar_expect_tx(bar, (uint32_t)(__popc(vm) * rows * 256));
        __syncwarp();
        if (lane < kStepKeys) {
          const int so = lane * kRowB;
          if (r_mine >= 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            if (!loc) {
              const size_t off = ((size_t)r_mine * row_stride + (size_t)kvh * kHeadDim) * 2;
              bulk_row(saddr(stg + offSK + so), reinterpret_cast<const uint8_t*>(p.mem_k) + off, bar);
              bulk_row(saddr(stg + offSV + so), reinterpret_cast<const uint8_t*>(p.mem_v) + off, bar);
            } else {
              const size_t lrow = (size_t)(p.loc_off[s] + r_mine) * p.hkv + kvh;
              if (!k_in_place) {  // rotated by rope_rows: high, then low halves
                const uint8_t* kr = reinterpret_cast<const uint8_t*>(p.krot) + lrow * kLocRowB;
                bulk_row(saddr(stg + offSK + so), kr, bar);
                bulk_row(saddr(stg + offSL + so), kr + 256, bar);
              }
              bulk_row(saddr(stg + offSV + so), p.v_loc + lrow * kHeadDim, bar);
            }
          } else {
            // a key past the range: zero values (P is 0 there, and 0 x NaN would not be)
            uint4* z = reinterpret_cast<uint4*>(stg + offSV + so);
#pragma unroll
            for (int u = 0; u < 16; ++u) z[u] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      return;
    }
    if (i < nsteps) {
      uint8_t* stg = wst + stage * kStageB;
      const bool loc = i < nsl;
      const int piece = 16 * (lane & 15);
#pragma unroll
      for (int u = 0; u < kStepKeys / 2; ++u) {
        const int key = 2 * u + (lane >> 4);
        const int64_t r = __shfl_sync(0xffffffffu, r_mine, key);
        const int so = key * kRowB + piece;
        if (r >= 0) {
          if (!loc) {
            const size_t off = ((size_t)r * row_stride + (size_t)kvh * kHeadDim) * 2 + piece;
            cp16(saddr(stg + offSK + so), reinterpret_cast<const uint8_t*>(p.mem_k) + off);
            cp16(saddr(stg + offSV + so), reinterpret_cast<const uint8_t*>(p.mem_v) + off);
          } else {
            const size_t lrow = (size_t)(p.loc_off[s] + r) * p.hkv + kvh;
            if (!k_in_place) {  // rotated by rope_rows
              const uint8_t* kr = reinterpret_cast<const uint8_t*>(p.krot) + lrow * kLocRowB;  // high, then low
              cp16(saddr(stg + offSK + so), kr + piece);
              cp16(saddr(stg + offSL + so), kr + 256 + piece);
            }
            cp16(saddr(stg + offSV + so), reinterpret_cast<const uint8_t*>(p.v_loc + lrow * kHeadDim) + piece);
          }
        } else {
          // a key past the range: zero values (P is 0 there, and 0 x NaN would not be)
          *reinterpret_cast<uint4*>(stg + offSV + so) = make_uint4(0, 0, 0, 0);
        }
      }
    }
    cp_commit();
  };
  {
    const int64_t r0 = row_of(w), r1 = row_of(w + kDWarps);
    issue(w, r0, 0, p.rot_in_kernel);
    issue(w + kDWarps, r1, 1, p.rot_in_kernel);
  }
  int64_t r_next = row_of(w + 2 * kDWarps);  // row of key kl in the warp's third step
  if (!routed) __syncthreads();  // the frequencies (the routed listing's barriers cover them)

  // ---- rotate this CTA's local keys (global positions pos_offset + j) into bf16 high and low
  // halves, local step j straight into stage j / 8 of warp j % 8 (j < 16)
  auto rotate_store = [&](int it, uint32_t a, uint32_t b) {
    const int jl = it >> 5, i = 2 * (it & 31);
    const double pos = p.pos_offset + (double)(l0 + jl);
    float y0a, y1a, y0b, y1b;
    rope_pair(bf_lo(a), bf_lo(b), pos, s_invf[i], y0a, y1a);
    rope_pair(bf_hi(a), bf_hi(b), pos, s_invf[i + 1], y0b, y1b);
    uint32_t hi0, lo0, hi1, lo1;
    split_bf2(y0a, y0b, hi0, lo0);
    split_bf2(y1a, y1b, hi1, lo1);
    const int step = jl / kStepKeys;
    uint8_t* row = sm + (step % kDWarps) * kWarpB + (step / kDWarps) * kStageB + (jl % kStepKeys) * kRowB;
    *reinterpret_cast<uint32_t*>(row + offSK + 2 * i) = hi0;
    *reinterpret_cast<uint32_t*>(row + offSK + 2 * (64 + i)) = hi1;
    *reinterpret_cast<uint32_t*>(row + offSL + 2 * i) = lo0;
    *reinterpret_cast<uint32_t*>(row + offSL + 2 * (64 + i)) = lo1;
  };
#pragma unroll
  for (int u = 0; u < kRotBatch; ++u) {
    const int it = tid + u * kDThreads;
    if (it < nrot) rotate_store(it, ka[u], kb2[u]);
  }
  for (int it = tid + kRotBatch * kDThreads; it < nrot; it += kDThreads) {
    const uint32_t a = __ldcg(reinterpret_cast<const unsigned int*>(kloc_ptr(it)));
    const uint32_t b = __ldcg(reinterpret_cast<const unsigned int*>(kloc_ptr(it) + 64));
    rotate_store(it, a, b);
  }
  // ---- queries, rotated, as bf16 high and low parts (shared by the warps)
  {
    uint32_t mine[4] = {qraw.x, qraw.y, qraw.z, qraw.w}, other[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) other[e] = __shfl_xor_sync(0xffffffffu, mine[e], 8);
    float y[8] = {qra.x, qra.y, qra.z, qra.w, qrb.x, qrb.y, qrb.z, qrb.w};
    if (!p.rope_q && qv_v < nvec) {
      const double pos = p.pos_offset + (double)(g0 + qv_v / p.group);
      const bool first = qv_d0 < 64;  // this thread holds x0 (dims < 64) or x1 (dims >= 64) of its pairs
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float xm = (e & 1) ? bf_hi(mine[e >> 1]) : bf_lo(mine[e >> 1]);
        const float xo = (e & 1) ? bf_hi(other[e >> 1]) : bf_lo(other[e >> 1]);
        float y0, y1;
        rope_pair(first ? xm : xo, first ? xo : xm, pos, s_invf[(qv_d0 & 63) + e], y0, y1);
        y[e] = first ? y0 : y1;
      }
    }
    uint32_t h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) split_bf2(y[2 * i], y[2 * i + 1], h[i], l[i]);
    *reinterpret_cast<uint4*>(sm + offQhi + qv_v * kRowB + 2 * qv_d0) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(sm + offQlo + qv_v * kRowB + 2 * qv_d0) = make_uint4(l[0], l[1], l[2], l[3]);
  }
  __syncthreads();  // the query parts and the local keys written in place

  // Q as the A operand of S, all 8 k-steps (16 dims each), high and low parts: held in
  // registers for every step of the warp
  uint32_t qh[8][4], ql[8][4];
  {
    const int arow = ((lane >> 3) & 1) * 8 + (lane & 7), acol = (lane >> 4) * 8;
    const uint32_t aQhi = saddr(sm + offQhi + arow * kRowB + 2 * acol);
    const uint32_t aQlo = saddr(sm + offQlo + arow * kRowB + 2 * acol);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      ldsm_x4(aQhi + 32 * ks, qh[ks][0], qh[ks][1], qh[ks][2], qh[ks][3]);
      ldsm_x4(aQlo + 32 * ks, ql[ks][0], ql[ks][1], ql[ks][2], ql[ks][3]);
    }
  }
  // B of S for key n-tile nt: keys 8nt + (lane & 7), matrix i = dims 8i..8i+7 of a 32-dim chunk
  const int brow = lane & 7, bcol = (lane >> 3) * 8;
  // B of O (V^T via .trans) for dims 16j..16j+15: matrix i = keys + 8(i & 1), dims + 8(i >> 1)
  const int vrow = ((lane >> 3) & 1) * 8 + (lane & 7), vcol = (lane >> 4) * 8;

  float o[16][4];  // O: 16 vectors x 128 dims; n-tile n = dims 8n..8n+7
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[n][e] = 0.f;
  float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;  // running max / sum of rows g, g + 8

  int it = 0;
  for (int i = w; i < nsteps; i += kDWarps, ++it) {
    const int stage = it & 1;
    if constexpr (BULK) {  // this step's rows (the next step's may still be in flight)
      if (!__all_sync(0xffffffffu, tc::mbar_wait(tc::smem_u32(&s_bar[w][stage]), (uint32_t)((it >> 1) & 1),
                                                 &s_abort)))
        break;
    } else {
      cp_wait<1>();  // this step's copies (this lane's); the next step's may still be in flight
    }
    __syncwarp();  // ... and every lane's
    const uint8_t* stg = wst + stage * kStageB;
    const bool loc = i < nsl;
    const int64_t kb = loc ? l0 + (int64_t)i * kStepKeys : m0 + (int64_t)(i - nsl) * kStepKeys;
    const int nk = (int)min((int64_t)kStepKeys, (loc ? l1 : m1) - kb);

    // ---- S (16 vectors x 16 keys) = Q K^T: n-tiles 0 (keys 0-7) and 1 (keys 8-15), each
    // accumulated in two halves (even and odd k-steps) so that four MMA chains run side by side
    float sa[2][4], sb[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = 0.f;
#pragma unroll
    for (int k2 = 0; k2 < 4; ++k2) {  // 32 dims: k-steps 2k2 and 2k2 + 1
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(saddr(stg + offSK + (8 * nt + brow) * kRowB + 2 * (32 * k2 + bcol)), b0, b1, b2, b3);
        mma16816(sa[nt], qh[2 * k2], b0, b1);
        mma16816(sb[nt], qh[2 * k2 + 1], b2, b3);
        mma16816(sa[nt], ql[2 * k2], b0, b1);
        mma16816(sb[nt], ql[2 * k2 + 1], b2, b3);
        if (loc) {
          ldsm_x4(saddr(stg + offSL + (8 * nt + brow) * kRowB + 2 * (32 * k2 + bcol)), b0, b1, b2, b3);
          mma16816(sa[nt], qh[2 * k2], b0, b1);
          mma16816(sb[nt], qh[2 * k2 + 1], b2, b3);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[nt][e] += sb[nt][e];
    // ---- mask (log2 units), online softmax over this step's keys. sa[nt]: rows g (0, 1) and
    // g + 8 (2, 3), keys 8nt + 2c, + 1
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int jk = 8 * nt + 2 * c + (e & 1);
        const int gr = e < 2 ? ga : gb;
        const bool vis = jk < nk && gr >= 0 && (!loc || kb + jk <= gr);
        sa[nt][e] = vis ? sa[nt][e] * sl2 : -INFINITY;
      }
    float xA = fmaxf(fmaxf(sa[0][0], sa[0][1]), fmaxf(sa[1][0], sa[1][1]));
    float xB = fmaxf(fmaxf(sa[0][2], sa[0][3]), fmaxf(sa[1][2], sa[1][3]));
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
      xA = fmaxf(xA, __shfl_xor_sync(0xffffffffu, xA, x));
      xB = fmaxf(xB, __shfl_xor_sync(0xffffffffu, xB, x));
    }
    const float nA = fmaxf(mA, xA), nB = fmaxf(mB, xB);
    const float cA = nA == -INFINITY ? 1.f : exp2f(mA - nA);
    const float cB = nB == -INFINITY ? 1.f : exp2f(mB - nB);
    float pr[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pr[nt][0] = nA == -INFINITY ? 0.f : exp2f(sa[nt][0] - nA);
      pr[nt][1] = nA == -INFINITY ? 0.f : exp2f(sa[nt][1] - nA);
      pr[nt][2] = nB == -INFINITY ? 0.f : exp2f(sa[nt][2] - nB);
      pr[nt][3] = nB == -INFINITY ? 0.f : exp2f(sa[nt][3] - nB);
    }
    float sA = pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1], sB = pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
#pragma unroll
    for (int x = 1; x <= 2; x <<= 1) {
      sA += __shfl_xor_sync(0xffffffffu, sA, x);
      sB += __shfl_xor_sync(0xffffffffu, sB, x);
    }
    lA = lA * cA + sA;
    lB = lB * cB + sB;
    mA = nA;
    mB = nB;
    // P as the A operand of P.V (16 vectors x 16 keys): the accumulator layout of S's two n-tiles
    const uint32_t pa[4] = {cvt_bf2(pr[0][0], pr[0][1]), cvt_bf2(pr[0][2], pr[0][3]), cvt_bf2(pr[1][0], pr[1][1]),
                            cvt_bf2(pr[1][2], pr[1][3])};

    // ---- O = O * corr + P V over the 128 dims (16 n-tiles of 8); most steps leave the max in place
    if (__any_sync(0xffffffffu, cA != 1.f || cB != 1.f)) {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        o[n][0] *= cA; o[n][1] *= cA;
        o[n][2] *= cB; o[n][3] *= cB;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(saddr(stg + offSV + vrow * kRowB + 2 * (16 * j + vcol)), v0, v1, v2, v3);
      mma16816(o[2 * j], pa, v0, v1);
      mma16816(o[2 * j + 1], pa, v2, v3);
    }
    __syncwarp();  // every lane is done with this stage
    // the warp's step after next goes into this stage
    issue(i + 2 * kDWarps, r_next, stage, false);
    r_next = row_of(i + 3 * kDWarps);
  }
  if constexpr (!BULK) cp_wait<0>();
  __syncthreads();  // every warp is done with its stages: they hold the merge now

  // ---- merge the 8 warps: o [w][v][d], m and l [w][v]
  float* mo = reinterpret_cast<float*>(sm + offMO);
  float* mm = reinterpret_cast<float*>(sm + offMM);
  float* ml = reinterpret_cast<float*>(sm + offMLs);
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    const int d = 8 * n + 2 * c;
    *reinterpret_cast<float2*>(mo + (w * kTileV + g) * kMRow + d) = make_float2(o[n][0], o[n][1]);
    *reinterpret_cast<float2*>(mo + (w * kTileV + g + 8) * kMRow + d) = make_float2(o[n][2], o[n][3]);
  }
  if (c == 0) {
    mm[w * kTileV + g] = mA;
    mm[w * kTileV + g + 8] = mB;
    ml[w * kTileV + g] = lA;
    ml[w * kTileV + g + 8] = lB;
  }
  __syncthreads();
  const int d = tid & (kHeadDim - 1);
  const bool split = p.n_splits > 1;
  float* po = reinterpret_cast<float*>(sm + offPO);
  float* pm_ = reinterpret_cast<float*>(sm + offPM);
  float* pl_ = reinterpret_cast<float*>(sm + offPL);
  for (int v = tid >> 7; v < nvec; v += 2) {
    float m = -INFINITY;
#pragma unroll
    for (int x = 0; x < kDWarps; ++x) m = fmaxf(m, mm[x * kTileV + v]);
    float l = 0.f, r = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int x = 0; x < kDWarps; ++x) {
        const float wt = exp2f(mm[x * kTileV + v] - m);  // 0 for a warp that saw nothing
        l += ml[x * kTileV + v] * wt;
        r += mo[(x * kTileV + v) * kMRow + d] * wt;
      }
    }
    if (!split) {
      const int rr = v / p.group, gg = v - rr * p.group;
      const size_t rh = (size_t)(row0 + rr) * p.hq + kvh * p.group + gg;
      const float res = l > 0.f ? r / l : 0.f;
      p.out[rh * kHeadDim + d] = (uint16_t)f2bf_bits(res);
      if (p.out_f32) p.out_f32[rh * kHeadDim + d] = res;
      if (p.lse && d == 0) p.lse[rh] = l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else {
      po[v * kHeadDim + d] = r;
      if (d == 0) {
        pm_[v] = m;
        pl_[v] = l;
      }
    }
  }
  if (!split) return;
  // ---- the cluster merges its splits' partials (log2 units) straight from their shared
  // memory: output (v, d) number o goes to CTA o / 256 mod splits, each thread loading all
  // splits' values at once; the second barrier keeps every CTA's memory alive until then
  cluster_sync();
  {
    const int ns = p.n_splits;
    const int rank = (int)cluster_rank();
    for (int o = rank * kDThreads + tid; o < nvec * kHeadDim; o += ns * kDThreads) {
      const int v = o / kHeadDim, dd = o % kHeadDim;
      float lj[kDecMaxSplits], mj[kDecMaxSplits], oj[kDecMaxSplits];
#pragma unroll
      for (int j = 0; j < kDecMaxSplits; ++j) {
        lj[j] = 0.f;
        mj[j] = -INFINITY;
        oj[j] = 0.f;
        if (j < ns) {
          lj[j] = ld_cluster_f32(saddr(pl_ + v), j);
          mj[j] = ld_cluster_f32(saddr(pm_ + v), j);
          oj[j] = ld_cluster_f32(saddr(po + v * kHeadDim + dd), j);
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < kDecMaxSplits; ++j)
        if (lj[j] > 0.f) mx = fmaxf(mx, mj[j]);
      float wsum = 0.f, r = 0.f;
#pragma unroll
      for (int j = 0; j < kDecMaxSplits; ++j) {
        if (lj[j] > 0.f) {
          const float wt = exp2f(mj[j] - mx);
          wsum += lj[j] * wt;
          r += wt * oj[j];
        }
      }
      r = wsum > 0.f ? r / wsum : 0.f;
      const int rr = v / p.group, gg = v - rr * p.group;
      const size_t rh = (size_t)(row0 + rr) * p.hq + kvh * p.group + gg;
      p.out[rh * kHeadDim + dd] = (uint16_t)f2bf_bits(r);
      if (p.out_f32) p.out_f32[rh * kHeadDim + dd] = r;
      if (p.lse && dd == 0) p.lse[rh] = wsum > 0.f ? (mx + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
    }
  }
  cluster_sync();
}

template <bool BULK>
msa_status launch_dec(const AttnParams& P, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  cudaError_t e = smem_limit_once(attend_dec_kernel<BULK>, kDecSmem, attr);
  if (e != cudaSuccess) return cuda_fail(e, "attend: decoding kernel shared memory");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P.n_splits, (unsigned)P.hkv, (unsigned)P.n_tiles);
  cfg.blockDim = dim3(kDThreads);
  cfg.dynamicSmemBytes = (size_t)kDecSmem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;  // the splits of a (tile, kv head): one cluster
  at[1].val.clusterDim.x = (unsigned)P.n_splits;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = P.n_splits > 1 ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, attend_dec_kernel<BULK>, P);
  if (e != cudaSuccess) return cuda_fail(e, "attend: decoding kernel");
  return launch_check("attend: decoding kernel");
}

}  // namespace

int g_dec_bulk = 0;  // testing control: the decoding kernel's rows by bulk copies

msa_status launch_attend_dec(const AttnParams& P, cudaStream_t st) {
  return g_dec_bulk ? launch_dec<true>(P, st) : launch_dec<false>(P, st);
}

int attend_dec_error_take() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof v) != cudaSuccess) return 0;
  if (v) {
    int z = 0;
    cudaMemcpyToSymbol(g_tc_error, &z, sizeof z);
  }
  return v;
}

}  // namespace msa

// Moves the decoding attention kernel's rows by bulk copies (1) or by 16-byte
// cp.async pieces (0, the default) in later msa_attend calls; returns the
// previous setting. A testing and benchmarking control; not declared in msa.h.
extern "C" int msa_debug_set_dec_bulk(int on) {
  const int old = msa::g_dec_bulk;
  if (on == 0 || on == 1) msa::g_dec_bulk = on;
  return old;
}
