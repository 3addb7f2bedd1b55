// Routing scores of many query rows at once (prefill), on the tensor cores.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — cosine
// similarity averaged over heads, then maximised over query tokens; "MSA-arXiv26",
// 核心方法 — the query scored against every document's pooled routing keys]
//
//   score(s, j) = max over rows t of s and chunks c of j of
//                 sum_h invk[c,h] * invq[t,h] * (kbar_r[c,h] . qr[t,h])
//
// With hundreds of query rows per call this is a dense contraction (2 x rows
// x 1,024 flops per pooled chunk) bound by the tensor cores, not by HBM. The
// decode scorer keeps all eight heads' accumulators in TMEM at once, which
// caps a pass at 32 query columns; here the heads take turns instead: one
// K = 128 contraction per head into a 128-chunk x NB-row fp32 accumulator
// (NB = 64, 128, 160 or 192; two to four of them in TMEM, so the tensor
// cores run ahead of the epilogue), and the epilogue folds each
// head into a running sum held in registers,
//   acc_sum[c, t] += invk[c, h] * invq[t, h] * acc_h[c, t],
// so the arithmetic is the decode scorer's: bf16 products, fp32 sums, exact
// cosine scales. After the eighth head the sums are max-reduced over each
// sequence's columns and over the document's chunks, and flushed with one
// atomicMax per (sequence, document segment).
//
// Warps: 0 TMA producer (one 128 x 64 stage of pooled keys and one NB x 64
// stage of query rows per mbarrier slot), 1 MMA issuer and TMEM owner, then
// the epilogue: WQ = 2 or 3 warps per TMEM lane quadrant, each owning NB/WQ
// columns. A 128 x NB x 16 MMA reads (128 + NB) x 32 bytes of shared memory,
// so wider blocks need fewer bytes per flop; that, not the TMEM depth, sets
// the speed of the narrower variants.
// Per row block an epilogue warp needs its columns' query scales and
// sequence codes; the query-norm kernel lays both out so that they arrive by
// a few 16-byte cp.async copies, double-buffered and issued one block ahead.
// Every wait is bounded in time.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "msa_internal.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

using namespace tc;

constexpr int kM = 128;    // chunks per tile
constexpr int kKB = 64;    // contraction elements per stage (one 128-byte row)
constexpr int kHeads = 8;
constexpr int kEpiWarp0 = 2;
constexpr int kSmemMax = 232448;

// NB query rows per block, WQ epilogue warps per TMEM lane quadrant. PAIR:
// two CTAs of a cluster share one M = 256 MMA (cta_group::2); each holds its
// 128 chunks of A and half of the NB query rows of B, and receives its 128
// lanes x NB columns of the accumulator.
template <int NB, int WQ, bool PAIR = false>
struct PfCfg {
  static constexpr int kEpiWarps = 4 * WQ;
  static constexpr int kThreads = 32 * (kEpiWarp0 + kEpiWarps);
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  static constexpr int kA = kM * kKB * 2;            // 16 KB
  static constexpr int kBRows = PAIR ? NB / 2 : NB;  // query rows of B this CTA loads
  static constexpr int kB = kBRows * kKB * 2;
  static constexpr int kStage = kA + kB;
  static constexpr int kTBuf = 512 / NB < 4 ? 512 / NB : 4;  // TMEM accumulators
  static constexpr int kTmemCols = 512;
  static constexpr int kCols = NB / WQ;              // columns per epilogue warp
  static constexpr int kChunks = (kCols + 31) / 32;  // 32-column groups of the flush
  // one epilogue warp's tables: two buffers of {query scales [h][col],
  // column codes [col]}, key scales [h][lane], document ids [lane]
  static constexpr int kIqTab = kHeads * kCols * 4;
  static constexpr int kColTab = kIqTab + kCols * 4;
  static constexpr int kWarpTab = 2 * kColTab + kHeads * 32 * 4 + 32 * 4;
  static constexpr int kFixed = 1024 + 256 + kEpiWarps * kWarpTab;
  static constexpr int kStages = (kSmemMax - kFixed) / kStage < 8 ? (kSmemMax - kFixed) / kStage : 8;
  static constexpr int kSmem = kFixed + kStages * kStage;
  // instruction descriptor: D fp32, A/B bf16, both K-major, N = NB, M = 128 (256 for a pair)
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NB >> 3) << 17) |
                                     ((uint32_t)((PAIR ? 2 * kM : kM) >> 4) << 24);
  static_assert(kCols % 16 == 0 && kCols * WQ == NB && kStages >= 3 && kTBuf >= 2, "tile configuration");
};

struct PfArgs {
  const float* invk;         // [C, 8]
  const int32_t* chunk_doc;  // [C]
  const float* invq_t;       // [8, Tp]
  const int32_t* col_code;   // [T]
  uint32_t* doc_key;         // [S, D]
  int64_t n_chunks, n_docs;
  int n_rows, n_rows_pad, n_tiles, n_nb;
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// ---- CTA pair (cluster of 2) building blocks
constexpr uint32_t kPeerMask = 0xFEFFFFFFu;  // clears the CTA-rank bit: the leader's copy of a shared address

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of both CTAs (not .aligned: callers may arrive from different roles).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
// Both CTAs load their own tiles; the bytes count on the leader's barrier.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar & kPeerMask)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Completion of the pair's MMAs, arriving on the barrier at this offset in every CTA of `mask`.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               ::"r"(bar), "h"(mask)
               : "memory");
}
// Arrive on the barrier at this offset in CTA `cta` of the cluster.
__device__ __forceinline__ void mbar_arrive_cta(uint32_t bar, uint32_t cta) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\tmapa.shared::cluster.u32 ra, %0, %1;\n\t"
      "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}"
      ::"r"(bar), "r"(cta)
      : "memory");
}

// 16-byte global -> shared copy that bypasses registers; the bytes past
// src_bytes (0..16) are written as zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Two IEEE fp32 operations in one instruction (Blackwell packed fp32):
// d = a * b + c and d = a * b on a pair of lanes, rounded like fmaf / a * b.
__device__ __forceinline__ float2 fma_f32x2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, C, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\tmov.b64 C, {%6, %7};\n\t"
      "fma.rn.f32x2 D, A, B, C;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 mul_f32x2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 A, B, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "mul.rn.f32x2 D, A, B;\n\tmov.b64 {%0, %1}, D;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// Maximum of W consecutive values (W a power of two, a balanced tree).
template <int W>
__device__ __forceinline__ float max_tree(const float* x) {
  float t[W / 2];
#pragma unroll
  for (int j = 0; j < W / 2; ++j) t[j] = fmaxf(x[j], x[j + W / 2]);
#pragma unroll
  for (int w = W / 4; w > 0; w >>= 1)
#pragma unroll
    for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
  return t[0];
}

template <int NB, int WQ, bool PAIR>
__global__ void __launch_bounds__(PfCfg<NB, WQ, PAIR>::kThreads, 1)
    score_pf_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ PfArgs a) {
  using C = PfCfg<NB, WQ, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStage);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + C::kTBuf;
  uint64_t* mma_done = tempty + C::kTBuf;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* warp_tabs = smem + C::kStages * C::kStage + 256;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < C::kTBuf; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), C::kEpiWarps * (PAIR ? 2 : 1));  // one arrival per epilogue warp
    }
    mbar_init(smem_u32(mma_done), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"((uint32_t)C::kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"((uint32_t)C::kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();  // both CTAs' barriers exist before either side's copies or arrivals
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // work units: tiles, or tile pairs (this CTA takes tile 2u + rank)
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int unit0 = PAIR ? (int)blockIdx.x / 2 : (int)blockIdx.x;
  const int ustep = PAIR ? (int)gridDim.x / 2 : (int)gridDim.x;
  const int n_units = PAIR ? (a.n_tiles + 1) / 2 : a.n_tiles;
  pdl_wait();  // the prologue above overlapped the previous kernel's tail
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = unit0; u < n_units && ok; u += ustep) {
        const int tile = PAIR ? 2 * u + (int)rank : u;
        for (int nb = 0; nb < a.n_nb && ok; ++nb)
          for (int kb = 0; kb < 2 * kHeads; ++kb) {
            if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag)) { ok = false; break; }
            const uint32_t st = smem_u32(stages + s * C::kStage);
            const uint32_t fb = smem_u32(&full[s]);
            if constexpr (PAIR) {  // the leader's barrier counts both CTAs' bytes
              if (rank == 0) mbar_expect_tx(fb, 2 * C::kStage);
              tma_load_2d_pair(st, &tmap_a, kb * kKB, tile * kM, fb);
              tma_load_2d_pair(st + C::kA, &tmap_b, kb * kKB, nb * NB + (int)rank * C::kBRows, fb);
            } else {
              mbar_expect_tx(fb, C::kStage);
              tma_load_2d(st, &tmap_a, kb * kKB, tile * kM, fb);
              tma_load_2d(st + C::kA, &tmap_b, kb * kKB, nb * NB, fb);
            }
            ++issued;
            if (++s == C::kStages) { s = 0; ph ^= 1; }
          }
      }
      if (!ok && rank == 0) {  // wait (bounded) for the copies still in flight
        const int n = issued < C::kStages ? issued : C::kStages;
        int ss = s;
        uint32_t pp = ph;
        const uint64_t t0 = globaltimer();
        for (int i = 0; i < n; ++i) {
          if (--ss < 0) { ss = C::kStages - 1; pp ^= 1; }
          while (!mbar_try(smem_u32(&full[ss]), pp) && globaltimer() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA (the leader of a pair)
    if (lane == 0 && rank == 0) {
      int s = 0, b = 0;
      uint32_t ph = 0, tph = 0;  // stage ring and TMEM ring phases
      bool ok = true;
      for (int u = unit0; u < n_units && ok; u += ustep)
        for (int nb = 0; nb < a.n_nb && ok; ++nb)
          for (int h = 0; h < kHeads && ok; ++h) {
            if (!mbar_wait(smem_u32(&tempty[b]), tph ^ 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)(b * NB);
            for (int ks = 0; ks < 2; ++ks) {
              if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag)) { ok = false; break; }
              tc_fence_after();
              const uint32_t st = smem_u32(stages + s * C::kStage);
#pragma unroll
              for (int k = 0; k < kKB / 16; ++k) {
                if constexpr (PAIR)
                  tc_mma_pair(d, sw128_desc(st + k * 32), sw128_desc(st + C::kA + k * 32), C::kIdesc,
                              (ks | k) ? 1u : 0u);
                else
                  tc_mma(d, sw128_desc(st + k * 32), sw128_desc(st + C::kA + k * 32), C::kIdesc, (ks | k) ? 1u : 0u);
              }
              if constexpr (PAIR)
                tc_commit_pair(smem_u32(&empty[s]), 0x3);
              else
                tc_commit(smem_u32(&empty[s]));
              if (++s == C::kStages) { s = 0; ph ^= 1; }
            }
            if (ok) {
              if constexpr (PAIR)
                tc_commit_pair(smem_u32(&tfull[b]), 0x3);
              else
                tc_commit(smem_u32(&tfull[b]));
            }
            if (++b == C::kTBuf) { b = 0; tph ^= 1; }
          }
      // Every MMA this thread issued has completed once mma_done flips.
      if constexpr (PAIR)
        tc_commit_pair(smem_u32(mma_done), 0x1);
      else
        tc_commit(smem_u32(mma_done));
      const uint64_t t0 = globaltimer();
      while (!mbar_try(smem_u32(mma_done), 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int ew = warp - kEpiWarp0;        // 0 .. 4 WQ - 1
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int col0 = (ew >> 2) * C::kCols;  // this warp's columns within the row block
    const int row = 32 * q + lane;          // chunk within the tile
    // This warp's tables live in shared memory: the L1 left beside ~200 KB of
    // stages is small, and the head loop must not wait on L2.
    uint8_t* wt = warp_tabs + ew * C::kWarpTab;
    float* s_ik = reinterpret_cast<float*>(wt + 2 * C::kColTab);              // [h][lane]
    int* s_doc = reinterpret_cast<int*>(wt + 2 * C::kColTab + kHeads * 128);  // [lane]
    auto iq_tab = [&](int k) { return reinterpret_cast<float*>(wt + k * C::kColTab); };
    auto code_tab = [&](int k) { return reinterpret_cast<int32_t*>(wt + k * C::kColTab + C::kIqTab); };
    // Query scales [h][col] and column codes of row block nbx into buffer k,
    // asynchronously; bytes past the last row arrive as zeros.
    auto fill = [&](int nbx, int k) {
      const int tw = nbx * NB + col0;
      const int left = a.n_rows - tw;  // valid columns from tw on
      float* dq = iq_tab(k);
      for (int i = lane; i < kHeads * C::kCols / 4; i += 32) {
        const int h = i / (C::kCols / 4), j = 4 * (i % (C::kCols / 4));
        const int nbytes = left - j >= 4 ? 16 : left - j > 0 ? 4 * (left - j) : 0;
        cp_async16(dq + h * C::kCols + j, nbytes ? a.invq_t + (size_t)h * a.n_rows_pad + tw + j : a.invq_t, nbytes);
      }
      int32_t* dc = code_tab(k);
      for (int j = 4 * lane; j < C::kCols; j += 128) {
        const int nbytes = left - j >= 4 ? 16 : left - j > 0 ? 4 * (left - j) : 0;
        cp_async16(dc + j, nbytes ? a.col_code + tw + j : a.col_code, nbytes);
      }
      cp_async_commit();
    };
    fill(0, 0);
    int b = 0, blk = 0;
    uint32_t tph = 0;
    bool ok = true;
    for (int u = unit0; u < n_units && ok; u += ustep) {
      const int tile = PAIR ? 2 * u + (int)rank : u;
      const int64_t c = (int64_t)tile * kM + row;
      const bool valid = c < a.n_chunks;
      {  // key scales and document of this lane's chunk (each lane reads only its own slots)
        float4 u0 = make_float4(0.f, 0.f, 0.f, 0.f), u1 = u0;
        int d = -1;
        if (valid) {
          u0 = __ldg(reinterpret_cast<const float4*>(a.invk + c * kHeads));
          u1 = __ldg(reinterpret_cast<const float4*>(a.invk + c * kHeads + 4));
          d = __ldg(a.chunk_doc + c);
        }
        s_ik[0 * 32 + lane] = u0.x; s_ik[1 * 32 + lane] = u0.y; s_ik[2 * 32 + lane] = u0.z;
        s_ik[3 * 32 + lane] = u0.w; s_ik[4 * 32 + lane] = u1.x; s_ik[5 * 32 + lane] = u1.y;
        s_ik[6 * 32 + lane] = u1.z; s_ik[7 * 32 + lane] = u1.w;
        s_doc[lane] = d;
      }

      for (int nb = 0; nb < a.n_nb && ok; ++nb, ++blk) {
        const int tw = nb * NB + col0;  // first query row of this warp's columns
        const int cur = a.n_nb > 1 ? (blk & 1) : 0;
        const bool prefetch = a.n_nb > 1 && (nb + 1 < a.n_nb || tile + (int)gridDim.x < a.n_tiles);
        cp_async_wait_all();
        __syncwarp();
        const float* iq = iq_tab(cur);
        const int32_t* s_code = code_tab(cur);

        float acc[C::kCols];
#pragma unroll
        for (int j = 0; j < C::kCols; ++j) acc[j] = 0.f;
        for (int h = 0; h < kHeads; ++h) {
          // __all_sync: the lanes leave the wait on different polls; the warp
          // must be converged again for the aligned TMEM loads and the math.
          if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&tfull[b]), tph, abort_flag))) { ok = false; break; }
          tc_fence_after();
          const float kh = s_ik[h * 32 + lane];
          const float2 k2 = make_float2(kh, kh);
          const float* iqh = iq + h * C::kCols;
#pragma unroll
          for (int cc = 0; cc < C::kCols / 16; ++cc) {
            float v[16];
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * NB + col0 + cc * 16), v);
            tmem_ld_wait();
            if (cc == C::kCols / 16 - 1) {  // this warp's part of the accumulator is in registers
              tc_fence_before();
              __syncwarp();
              if (lane == 0) {  // one arrival per warp, on the leader's barrier for a pair
                if constexpr (PAIR)
                  mbar_arrive_cta(smem_u32(&tempty[b]), 0);
                else
                  mbar_arrive(smem_u32(&tempty[b]));
              }
            }
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {
              const float4 s4 = *reinterpret_cast<const float4*>(iqh + cc * 16 + 4 * j4);
              float* ac = acc + cc * 16 + 4 * j4;
              const float2 lo = fma_f32x2(make_float2(v[4 * j4], v[4 * j4 + 1]),
                                          mul_f32x2(k2, make_float2(s4.x, s4.y)), make_float2(ac[0], ac[1]));
              const float2 hi = fma_f32x2(make_float2(v[4 * j4 + 2], v[4 * j4 + 3]),
                                          mul_f32x2(k2, make_float2(s4.z, s4.w)), make_float2(ac[2], ac[3]));
              ac[0] = lo.x; ac[1] = lo.y; ac[2] = hi.x; ac[3] = hi.y;
            }
          }
          if (++b == C::kTBuf) { b = 0; tph ^= 1; }
          // the next row block's tables, once this head's TMEM is released
          if (h == 0 && prefetch) fill(nb + 1 < a.n_nb ? nb + 1 : 0, cur ^ 1);
        }
        if (!ok) break;

        // Max over each sequence's columns, then over the document's chunks
        // (segmented warp max), one atomicMax per segment head. Column
        // metadata is uniform across the warp; valid columns form a prefix,
        // and this warp's last valid column also closes a (partial) run.
        const int nvalid = a.n_rows - tw < C::kCols ? a.n_rows - tw : C::kCols;
        const int doc = s_doc[lane];
        // lanes whose right-hand neighbour at distance o is in the same document
        unsigned same = 0;
#pragma unroll
        for (int o = 1, i = 0; o < 32; o <<= 1, ++i) {
          const int dn = __shfl_down_sync(0xffffffffu, doc, o);
          if (lane + o < 32 && dn == doc) same |= 1u << i;
        }
        const int doc_up = __shfl_up_sync(0xffffffffu, doc, 1);
        const bool head = valid && (lane == 0 || doc_up != doc);
        float m = -INFINITY;
        auto flush = [&](float x, int sq) {
#pragma unroll
          for (int o = 1, i = 0; o < 32; o <<= 1, ++i) {
            const float xo = __shfl_down_sync(0xffffffffu, x, o);
            if (same & (1u << i)) x = fmaxf(x, xo);
          }
          if (head) atomicMax(a.doc_key + (size_t)sq * a.n_docs + doc, ord_f32(x));
        };
#pragma unroll
        for (int cc = 0; cc < C::kChunks; ++cc) {
          const int width = cc == C::kChunks - 1 ? C::kCols - 32 * cc : 32;  // columns in this group
          const int nv = nvalid - cc * 32;  // valid columns in this group (if < width)
          if (nv <= 0) break;
          const unsigned vm = nv >= 32 ? 0xffffffffu : (1u << nv) - 1u;
          const int code = lane < width ? s_code[cc * 32 + lane] : 0;
          unsigned em = __ballot_sync(0xffffffffu, lane < nv && (code & 256));
          if (nv <= width) em |= 1u << (nv - 1);
          if (width == 32 && vm == 0xffffffffu && (em & 0x7fffffffu) == 0) {  // one run through the group
            const float x = fmaxf(m, max_tree<32>(acc + (cc * 32 < C::kCols - 31 ? cc * 32 : 0)));
            if (em) {
              flush(x, __shfl_sync(0xffffffffu, code, 31) & 255);
              m = -INFINITY;
            } else {
              m = x;
            }
            continue;
          }
          int lo = 0;
          while (em) {
            const int hi = __ffs(em) - 1;
            em &= em - 1;
            float x = m;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (cc * 32 + j < C::kCols && j >= lo && j <= hi) x = fmaxf(x, acc[cc * 32 + j]);
            flush(x, __shfl_sync(0xffffffffu, code, hi) & 255);
            m = -INFINITY;
            lo = hi + 1;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (cc * 32 + j < C::kCols && j >= lo && ((vm >> j) & 1u)) m = fmaxf(m, acc[cc * 32 + j]);
        }
      }
    }
    cp_async_wait_all();  // no table copy may still be in flight at exit
  }

  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();  // the leader's MMAs are done and neither CTA still reads the other's memory
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::kTmemCols));
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::kTmemCols));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over [rows, 1024] bf16 with a (64, box_rows) box, 128-byte swizzle.
bool make_map_2d(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(kHeads * 128), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeads * 128 * 2};
  cuuint32_t box[2] = {(cuuint32_t)kKB, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NB, int WQ, bool PAIR = false>
msa_status launch_nb(const RoutePlan& p, cudaStream_t st) {
  using C = PfCfg<NB, WQ, PAIR>;
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, p.kbar_r, p.n_chunks, kM) || !make_map_2d(&mb, p.qr, p.n_rows, C::kBRows))
    return fail(MSA_ERR_CUDA, "route: cannot encode TMA tensor maps (cuTensorMapEncodeTiled)");
  PfArgs a{};
  a.invk = p.kr_inv_norm;
  a.chunk_doc = p.chunk_doc;
  a.invq_t = p.invq_t;
  a.col_code = p.col_code;
  a.doc_key = p.doc_key;
  a.n_chunks = p.n_chunks;
  a.n_docs = p.n_docs;
  a.n_rows = p.n_rows;
  a.n_rows_pad = p.n_rows_pad;
  a.n_tiles = (int)((p.n_chunks + kM - 1) / kM);
  a.n_nb = (p.n_rows + NB - 1) / NB;
  static std::atomic<uint64_t> attr_set{0};
  {
    const cudaError_t e = smem_limit_once(score_pf_kernel<NB, WQ, PAIR>, C::kSmem, attr_set);
    if (e != cudaSuccess) return cuda_fail(e, "route: many-row scorer shared memory");
  }
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e;
  if constexpr (PAIR) {  // clusters of 2 CTAs, one tile pair per cluster at a time
    const int pairs = (a.n_tiles + 1) / 2;
    const int clusters = pairs < sms / 2 ? pairs : sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * clusters));
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = (size_t)C::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, score_pf_kernel<NB, WQ, PAIR>, ma, mb, a);
  } else {
    const int grid = a.n_tiles < sms ? a.n_tiles : sms;
    e = launch_pdl(score_pf_kernel<NB, WQ, PAIR>, dim3(grid), dim3(C::kThreads), (size_t)C::kSmem, st, ma, mb, a);
  }
  if (e != cudaSuccess) return cuda_fail(e, "route: score (tensor cores, many rows)");
  return launch_check("route: score (tensor cores, many rows)");
}

}  // namespace

bool score_pf_supported(const RoutePlan& p) {
  // eight routing heads; 16-byte aligned tensor-map bases
  return p.hr == kHeads && p.n_chunks > 0 && (reinterpret_cast<uintptr_t>(p.kbar_r) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(p.qr) & 15) == 0;
}

int g_pf_block = 0;  // testing control: force a row block (0 = choose)
// 192-row blocks on CTA pairs (1) or single CTAs (0, the default: measured on
// a 161K-chunk bank with 1,024 rows the pair takes 625 us against 393 us; both
// SMs' epilogues gate one MMA, so each step waits for the slower of the two).
int g_pf_pair = 0;

msa_status launch_score_pf(const RoutePlan& p, cudaStream_t st) {
  // The row block with the least estimated time: padded columns times the
  // time per column of each variant (measured on B200 with a 161K-chunk bank;
  // wider blocks read fewer shared-memory bytes per flop).
  const int cand[4] = {64, 128, 160, 192};
  const int per_col[4] = {81, 45, 40, 36};
  int best = 128;
  int64_t best_cost = INT64_MAX;
  for (int i = 0; i < 4; ++i) {
    const int64_t blocks = (p.n_rows + cand[i] - 1) / cand[i];
    const int64_t cost = blocks * cand[i] * per_col[i];
    if (cost < best_cost) { best_cost = cost; best = cand[i]; }
  }
  if (g_pf_block) best = g_pf_block;
  if (best == 64) return launch_nb<64, 2>(p, st);
  if (best == 160) return launch_nb<160, 2>(p, st);
  if (best == 192) return g_pf_pair ? launch_nb<192, 3, true>(p, st) : launch_nb<192, 3>(p, st);
  return launch_nb<128, 2>(p, st);
}

}  // namespace msa

// Forces the many-row scorer's row block (64, 128, 160 or 192; 0 = choose by
// padding) for later route calls in this process; returns the previous
// setting. A testing and benchmarking control; not declared in msa.h.
extern "C" int msa_debug_set_pf_pair(int on) {
  const int old = msa::g_pf_pair;
  if (on == 0 || on == 1) msa::g_pf_pair = on;
  return old;
}

extern "C" int msa_debug_set_pf_block(int nb) {
  const int old = msa::g_pf_block;
  if (nb == 0 || nb == 64 || nb == 128 || nb == 160 || nb == 192) msa::g_pf_block = nb;
  return old;
}

namespace msa {

int pf_error_take() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof v) != cudaSuccess) return 0;
  if (v) {
    int z = 0;
    cudaMemcpyToSymbol(g_tc_error, &z, sizeof z);
  }
  return v;
}

}  // namespace msa
