// Routing scores on the 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — relevance by
// cosine similarity, averaged over heads, then maximised over query tokens; Top-k
// documents. "MSA-arXiv26", 核心方法 — the query is scored against every
// document's pooled routing keys]
//
//   score(s, j) = max over rows t of s and chunks c of j of
//                 sum_h invk[c,h] * invq[t,h] * (kbar_r[c,h] . qr[t,h])
//   (invq holds 1 / (hr * max(||q||, eps)), invk 1 / max(||k||, eps))
//
// The contraction is skinny: per head, A = 128 pooled chunks x 128 dims (the
// streamed operand, 32 KB from HBM), B = NB query rows x 128 dims (a few KB,
// resident in L2). Each pooled routing key is read from HBM exactly once, so
// for the row counts of decoding the kernel is bound by HBM bandwidth and the
// tensor cores only keep the arithmetic off the critical path.
//
// Persistent CTA per SM, 6 warps:
//   warp 0    TMA producer: per (tile, row block, head) one stage = two
//             128-byte-swizzled boxes of A and two of B, on an mbarrier ring.
//   warp 1    allocates TMEM; one thread issues tcgen05.mma (M=128, N=NB,
//             K=16, bf16 -> fp32) into a per-head accumulator, and commits
//             the stage back to the producer.
//   warps 2-5 epilogue: tcgen05.ld of the 8 heads' accumulators of a 128-chunk
//             tile (double-buffered in TMEM so it overlaps the next tile's
//             MMAs), the cosine scaling and head sum, the max over each
//             sequence's rows, a segmented warp max over chunks of the same
//             document, and one atomicMax per document segment on an
//             order-preserving integer encoding. Scores never reach HBM.
// Every mbarrier wait is bounded in time; on expiry the kernel records an
// error, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "msa_internal.cuh"
#include "tc_ptx.cuh"

namespace msa {

namespace {

using namespace tc;

constexpr int kHeads = 8;
constexpr int kTileM = 128;
constexpr int kThreads = 192;
constexpr int kEpiWarp0 = 2;

struct TcArgs {
  const float* invk;        // [C, 8]
  const int32_t* chunk_doc; // [C]
  const float* invq;        // [T, 8]
  uint32_t* doc_key;        // [S, D]
  int64_t n_chunks, n_docs;
  int n_rows, n_seq, n_tiles, n_nb;
  int32_t q_seq_off[kMaxSeq + 1];
};

__device__ __forceinline__ int seq_of_row(const int32_t* off, int n_seq, int t) {
  int lo = 0, hi = n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int NB>
struct Cfg {
  static constexpr int kA = kTileM * 128 * 2;   // 32 KB: one head of a 128-chunk tile
  static constexpr int kAHalf = kA / 2;         // 64 dims
  static constexpr int kB = NB * 128 * 2;       // one head of NB query rows
  static constexpr int kBHalf = kB / 2;
  static constexpr int kStage = kA + kB;
  static constexpr int kStages = NB <= 16 ? 6 : 5;
  static constexpr int kTmemCols = 2 * kHeads * NB;  // double-buffered 8 heads
  static constexpr int kWarpTab = NB * kHeads * 4 + 2 * NB * 4;  // one epilogue warp's column table
  static constexpr int kSmem = 1024 + kStages * kStage + 256 + 4 * kWarpTab;  // slack, stages, barriers, tables
  // instruction descriptor: D fp32, A/B bf16, both K-major, N = NB, M = 128
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NB >> 3) << 17) |
                                     ((uint32_t)(kTileM >> 4) << 24);
};

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ TcArgs a) {
  using C = Cfg<NB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStage);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Each epilogue warp's own table of the current row block: query scales
  // [NB][8], and per column its sequence (-1 past the last row) and whether a
  // sequence's run ends there. Private to the warp, so filling it needs only
  // __syncwarp (no barrier that a warp which gave up could leave waiting).
  float* s_invq = reinterpret_cast<float*>(smem + C::kStages * C::kStage + 256 +
                                           (warp >= kEpiWarp0 ? warp - kEpiWarp0 : 0) * C::kWarpTab);
  int* s_seq = reinterpret_cast<int*>(s_invq + NB * kHeads);
  int* s_end = s_seq + NB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull[b]), 1);
      mbar_init(smem_u32(&tempty[b]), 128);
    }
    mbar_init(smem_u32(mma_done), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)C::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The producer and the MMA warp read only the bank and the query rows, which
  // are inputs of the call and complete before the preceding kernel (the query
  // preparation) started; they begin streaming at once, overlapping that
  // kernel. The epilogue reads its outputs (query scales, the cleared document
  // keys) and waits for it first.
  if (warp >= kEpiWarp0) pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
        for (int nb = 0; nb < a.n_nb && ok; ++nb) {
          for (int h = 0; h < kHeads; ++h) {
            if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag)) { ok = false; break; }
            const uint32_t st = smem_u32(stages + s * C::kStage);
            const uint32_t fb = smem_u32(&full[s]);
            mbar_expect_tx(fb, C::kStage);
            tma_load_3d(st, &tmap_k, 0, h, tile * kTileM, fb);
            tma_load_3d(st + C::kAHalf, &tmap_k, 64, h, tile * kTileM, fb);
            tma_load_3d(st + C::kA, &tmap_q, 0, h, nb * NB, fb);
            tma_load_3d(st + C::kA + C::kBHalf, &tmap_q, 64, h, nb * NB, fb);
            ++issued;
            if (++s == C::kStages) { s = 0; ph ^= 1; }
          }
        }
      }
      if (!ok) {
        // Drain: wait (bounded) for the copies of the last stages issued.
        int n = issued < C::kStages ? issued : C::kStages;
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
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int blk = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
        for (int nb = 0; nb < a.n_nb && ok; ++nb, ++blk) {
          const int b = blk & 1;
          if (!mbar_wait(smem_u32(&tempty[b]), ((blk >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          for (int h = 0; h < kHeads; ++h) {
            if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t st = smem_u32(stages + s * C::kStage);
            const uint32_t d = tmem + (uint32_t)((b * kHeads + h) * NB);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t koff = (kk >> 2) * C::kAHalf + (kk & 3) * 32;
              const uint32_t kofb = (kk >> 2) * C::kBHalf + (kk & 3) * 32;
              tc_mma(d, sw128_desc(st + koff), sw128_desc(st + C::kA + kofb), C::kIdesc, kk > 0 ? 1u : 0u);
            }
            tc_commit(smem_u32(&empty[s]));
            if (++s == C::kStages) { s = 0; ph ^= 1; }
          }
          if (ok) tc_commit(smem_u32(&tfull[b]));
        }
      }
      // Every MMA this thread issued has completed once mma_done flips.
      tc_commit(smem_u32(mma_done));
      const uint64_t t0 = globaltimer();
      while (!mbar_try(smem_u32(mma_done), 0) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;                  // TMEM lane quadrant of this warp
    const int row = 32 * q + lane;           // chunk within the tile
    auto load_block = [&](int t0) {
      __syncwarp();
      for (int i = lane; i < NB * kHeads; i += 32) {
        const int t = t0 + i / kHeads;
        s_invq[i] = t < a.n_rows ? a.invq[(size_t)t * kHeads + (i % kHeads)] : 0.f;
      }
      for (int i = lane; i < NB; i += 32) {
        const int t = t0 + i;
        int sq = -1, end = 0;
        if (t < a.n_rows) {
          sq = seq_of_row(a.q_seq_off, a.n_seq, t);
          end = (t + 1 == a.q_seq_off[sq + 1]) || (i == NB - 1) || (t + 1 == a.n_rows);
        }
        s_seq[i] = sq;
        s_end[i] = end;
      }
      __syncwarp();
    };
    if (a.n_nb == 1) load_block(0);
    int blk = 0;
    for (int tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x) {
      const int64_t c = (int64_t)tile * kTileM + row;
      const bool valid = c < a.n_chunks;
      float invk[kHeads];
      int doc = -1;
      if (valid) {
        const float4 u0 = __ldg(reinterpret_cast<const float4*>(a.invk + c * kHeads));
        const float4 u1 = __ldg(reinterpret_cast<const float4*>(a.invk + c * kHeads + 4));
        invk[0] = u0.x; invk[1] = u0.y; invk[2] = u0.z; invk[3] = u0.w;
        invk[4] = u1.x; invk[5] = u1.y; invk[6] = u1.z; invk[7] = u1.w;
        doc = __ldg(a.chunk_doc + c);
      } else {
#pragma unroll
        for (int h = 0; h < kHeads; ++h) invk[h] = 0.f;
      }
      // lanes whose right-hand neighbour at distance o is in the same document
      unsigned same = 0;
#pragma unroll
      for (int o = 1, i = 0; o < 32; o <<= 1, ++i) {
        int dn = __shfl_down_sync(0xffffffffu, doc, o);
        if (lane + o < 32 && dn == doc) same |= 1u << i;
      }
      const int doc_up = __shfl_up_sync(0xffffffffu, doc, 1);
      const bool head = valid && (lane == 0 || doc_up != doc);  // first lane of a document segment

      bool ok = true;
      for (int nb = 0; nb < a.n_nb; ++nb, ++blk) {
        const int b = blk & 1;
        if (a.n_nb > 1) load_block(nb * NB);
        // __all_sync: the lanes leave the wait on different polls; the warp
        // must be converged again for the aligned TMEM loads and the math.
        if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&tfull[b]), (blk >> 1) & 1, abort_flag))) { ok = false; break; }
        tc_fence_after();
        // Stream over the block's columns: the score of (row, column), a
        // running max over the current sequence's columns, and a flush (warp
        // max over the document's chunks, one atomic per document) wherever a
        // sequence's run ends. Column metadata is uniform across the warp.
        float m = -INFINITY;
#pragma unroll
        for (int jh = 0; jh < NB; jh += 16) {
          float v[kHeads][16];
#pragma unroll
          for (int h = 0; h < kHeads; ++h)
            tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)((b * kHeads + h) * NB + jh), v[h]);
          tmem_ld_wait();
          if (jh + 16 >= NB) {  // every accumulator of this buffer is in registers
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[b]));
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int jj = jh + j;
            const int sq = s_seq[jj];
            if (sq < 0) break;
            const float4 qa = *reinterpret_cast<const float4*>(s_invq + jj * kHeads);
            const float4 qb = *reinterpret_cast<const float4*>(s_invq + jj * kHeads + 4);
            float sc = v[0][j] * (invk[0] * qa.x);
            sc += v[1][j] * (invk[1] * qa.y);
            sc += v[2][j] * (invk[2] * qa.z);
            sc += v[3][j] * (invk[3] * qa.w);
            sc += v[4][j] * (invk[4] * qb.x);
            sc += v[5][j] * (invk[5] * qb.y);
            sc += v[6][j] * (invk[6] * qb.z);
            sc += v[7][j] * (invk[7] * qb.w);
            m = fmaxf(m, sc);
            if (s_end[jj]) {
#pragma unroll
              for (int o = 1, i = 0; o < 32; o <<= 1, ++i) {
                const float mo = __shfl_down_sync(0xffffffffu, m, o);
                if (same & (1u << i)) m = fmaxf(m, mo);
              }
              if (head) atomicMax(a.doc_key + (size_t)sq * a.n_docs + doc, ord_f32(m));
              m = -INFINITY;
            }
          }
        }
      }
      if (!ok) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::kTmemCols));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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

// 3-D map over [outer, heads, 128] bf16 with a (64, 1, box_rows) box, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t outer, int heads, int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)outer};
  cuuint64_t strides[2] = {256, (cuuint64_t)heads * 256};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int NB>
msa_status launch_nb(const RoutePlan& p, cudaStream_t st) {
  using C = Cfg<NB>;
  CUtensorMap mk, mq;
  if (!make_map(&mk, p.kbar_r, p.n_chunks, p.hr, kTileM) || !make_map(&mq, p.qr, p.n_rows, p.hr, NB))
    return fail(MSA_ERR_CUDA, "route: cannot encode TMA tensor maps (cuTensorMapEncodeTiled)");
  TcArgs a;
  a.invk = p.kr_inv_norm;
  a.chunk_doc = p.chunk_doc;
  a.invq = p.invq;
  a.doc_key = p.doc_key;
  a.n_chunks = p.n_chunks;
  a.n_docs = p.n_docs;
  a.n_rows = p.n_rows;
  a.n_seq = p.n_seq;
  a.n_tiles = (int)((p.n_chunks + kTileM - 1) / kTileM);
  a.n_nb = (p.n_rows + NB - 1) / NB;
  for (int i = 0; i <= p.n_seq; ++i) a.q_seq_off[i] = p.q_seq_off[i];
  static std::atomic<uint64_t> attr_set{0};
  {
    const cudaError_t e = smem_limit_once(score_tc_kernel<NB>, C::kSmem, attr_set);
    if (e != cudaSuccess) return cuda_fail(e, "route: tensor-core kernel shared memory");
  }
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int grid = a.n_tiles < sms ? a.n_tiles : sms;
  cudaError_t e = launch_pdl(score_tc_kernel<NB>, dim3(grid), dim3(kThreads), (size_t)C::kSmem, st, mk, mq, a);
  if (e != cudaSuccess) return cuda_fail(e, "route: score (tensor cores)");
  return launch_check("route: score (tensor cores)");
}

}  // namespace

bool score_tc_built() { return true; }

bool score_tc_supported(const RoutePlan& p) {
  // 16-byte aligned base addresses for the tensor maps; eight routing heads.
  return p.hr == kHeads && (reinterpret_cast<uintptr_t>(p.kbar_r) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(p.qr) & 15) == 0 && p.n_chunks > 0;
}

msa_status launch_score_tc(const RoutePlan& p, cudaStream_t st) {
  if (p.n_rows <= 16) return launch_nb<16>(p, st);
  return launch_nb<32>(p, st);
}

int tc_error_take() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof v) != cudaSuccess) return 0;
  if (v) {
    int z = 0;
    cudaMemcpyToSymbol(g_tc_error, &z, sizeof z);
  }
  return v;
}

}  // namespace msa
