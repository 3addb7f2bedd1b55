// Routing scores of many query rows at once (prefill), on the tensor cores.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — cosine
// similarity mean-pooled over heads, then token-wise max; "MSA-arXiv26",
// 核心方法 — the query scored against every document's pooled routing keys]
//
// With hundreds of query rows per call the scoring is a dense contraction
// (2 x rows x 1,024 flops per pooled chunk), bound by the tensor cores rather
// than by HBM. Per-head accumulators would cap a pass at 32 query columns
// (8 heads x 32 x 2 buffers = 512 TMEM columns), so instead both cosine
// scales are folded into the operands and the head sum becomes part of the
// contraction:
//   score(t, c) = sum over (h, i) of Ahat[c, h, i] * Qhat[t, h, i],
//   Ahat = bf16(kbar_r * invk[c, h]),  Qhat = bf16(qr * invq[t, h])
// (invq includes the head mean's 1/hr). Rounding the scaled operands to
// bfloat16 moves a score by about 1e-4, well inside the 1e-3 bar. Qhat is
// written by the query-norm kernel; Ahat is made in shared memory: a
// transform warp group rescales each TMA-loaded 128-chunk x 64-dimension
// stage in place (the 128-byte swizzle permutes 16-byte pieces only within a
// chunk's own 128-byte row, so a row's scale applies to all of it).
//
// Tile: 128 chunks x NB query rows (NB = 128 or 256) x K = 1,024 in 16
// stages of 64; one fp32 accumulator of NB TMEM columns, double-buffered.
// Warps: 0 TMA producer, 1 MMA issuer (and TMEM owner), 2-5 transform, 6-9
// epilogue (a running max per sequence and a per-document flush, as in the
// decode scorer). Every wait is bounded in time.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "msa_internal.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

using namespace tc;

constexpr int kM = 128;                      // chunks per tile
constexpr int kKB = 64;                      // contraction elements per stage (one 128-byte row)
constexpr int kHeads = 8;
constexpr int kKSteps = kHeads * 128 / kKB;  // 16
constexpr int kThreads = 320;
constexpr int kEpiWarp0 = 6;

template <int NB>
struct PfCfg {
  static constexpr int kA = kM * kKB * 2;     // 16 KB
  static constexpr int kB = NB * kKB * 2;     // 16 or 32 KB
  static constexpr int kStage = kA + kB;
  static constexpr int kStages = 196608 / kStage;  // 4 or 6
  static constexpr int kTmemCols = 2 * NB;
  static constexpr int kWarpTab = NB * 2;     // int16 per column
  static constexpr int kSmem = 1024 + kStages * kStage + 256 + 4 * kWarpTab;
  // instruction descriptor: D fp32, A/B bf16, both K-major, N = NB, M = 128
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(NB >> 3) << 17) |
                                     ((uint32_t)(kM >> 4) << 24);
};

struct PfArgs {
  const float* invk;         // [C, 8]
  const int32_t* chunk_doc;  // [C]
  uint32_t* doc_key;         // [S, D]
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

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// Two bf16 (packed) times a scale, rounded back to a bf16 pair.
__device__ __forceinline__ uint32_t scale_bf2(uint32_t w, float s) {
  const __nv_bfloat162 r = __floats2bfloat162_rn(bf_lo(w) * s, bf_hi(w) * s);
  return *reinterpret_cast<const uint32_t*>(&r);
}

template <int NB>
__global__ void __launch_bounds__(kThreads, 1)
    score_pf_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ PfArgs a) {
  using C = PfCfg<NB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStage);
  uint64_t* ready = full + C::kStages;
  uint64_t* empty = ready + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // An epilogue warp's own column table for the current row block: the
  // column's sequence, +256 where a sequence's run ends, -1 past the last row.
  int16_t* s_col = reinterpret_cast<int16_t*>(smem + C::kStages * C::kStage + 256 +
                                              (warp >= kEpiWarp0 ? warp - kEpiWarp0 : 0) * C::kWarpTab);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&ready[s]), 128);
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
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x)
        for (int nb = 0; nb < a.n_nb && ok; ++nb)
          for (int kb = 0; kb < kKSteps; ++kb) {
            if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag)) { ok = false; break; }
            const uint32_t st = smem_u32(stages + s * C::kStage);
            const uint32_t fb = smem_u32(&full[s]);
            mbar_expect_tx(fb, C::kStage);
            tma_load_2d(st, &tmap_a, kb * kKB, tile * kM, fb);
            tma_load_2d(st + C::kA, &tmap_b, kb * kKB, nb * NB, fb);
            ++issued;
            if (++s == C::kStages) { s = 0; ph ^= 1; }
          }
      if (!ok) {  // wait (bounded) for the copies still in flight
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
    // ------------------------------------------------------------- MMA
    if (lane == 0) {
      int s = 0, blk = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
        for (int nb = 0; nb < a.n_nb && ok; ++nb, ++blk) {
          const int b = blk & 1;
          if (!mbar_wait(smem_u32(&tempty[b]), ((blk >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(b * NB);
          for (int kb = 0; kb < kKSteps; ++kb) {
            if (!mbar_wait(smem_u32(&ready[s]), ph, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t st = smem_u32(stages + s * C::kStage);
#pragma unroll
            for (int k = 0; k < kKB / 16; ++k)
              tc_mma(d, sw128_desc(st + k * 32), sw128_desc(st + C::kA + k * 32), C::kIdesc, (kb | k) ? 1u : 0u);
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
  } else if (warp < kEpiWarp0) {
    // ---------------------------------------- transform: A *= invk[c, h]
    const int r = threadIdx.x - 64;  // chunk row within the tile
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
      const int64_t c = (int64_t)tile * kM + r;
      float ik[kHeads];
      if (c < a.n_chunks) {
        const float4 u0 = __ldg(reinterpret_cast<const float4*>(a.invk + c * kHeads));
        const float4 u1 = __ldg(reinterpret_cast<const float4*>(a.invk + c * kHeads + 4));
        ik[0] = u0.x; ik[1] = u0.y; ik[2] = u0.z; ik[3] = u0.w;
        ik[4] = u1.x; ik[5] = u1.y; ik[6] = u1.z; ik[7] = u1.w;
      } else {
#pragma unroll
        for (int h = 0; h < kHeads; ++h) ik[h] = 0.f;
      }
      for (int nb = 0; nb < a.n_nb && ok; ++nb)
#pragma unroll
        for (int kb = 0; kb < kKSteps; ++kb) {
          if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag)) { ok = false; break; }
          const float sc = ik[kb >> 1];  // two 64-dimension stages per head
          // The row's eight 16-byte pieces are visited starting at piece
          // r mod 8, so the eight rows of each 8-thread access phase touch
          // eight different bank groups (the scale is the same for all).
          uint4* row = reinterpret_cast<uint4*>(stages + s * C::kStage + r * 128);
          uint4 w[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) w[u] = row[u ^ (r & 7)];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            row[u ^ (r & 7)] = make_uint4(scale_bf2(w[u].x, sc), scale_bf2(w[u].y, sc), scale_bf2(w[u].z, sc),
                                          scale_bf2(w[u].w, sc));
          fence_proxy_async_smem();  // the MMA reads these bytes through the async proxy
          mbar_arrive(smem_u32(&ready[s]));
          if (++s == C::kStages) { s = 0; ph ^= 1; }
        }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant of this warp
    const int row = 32 * q + lane;
    int blk = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.n_tiles && ok; tile += gridDim.x) {
      const int64_t c = (int64_t)tile * kM + row;
      const bool valid = c < a.n_chunks;
      const int doc = valid ? __ldg(a.chunk_doc + c) : -1;
      // lanes whose right-hand neighbour at distance o is in the same document
      unsigned same = 0;
#pragma unroll
      for (int o = 1, i = 0; o < 32; o <<= 1, ++i) {
        const int dn = __shfl_down_sync(0xffffffffu, doc, o);
        if (lane + o < 32 && dn == doc) same |= 1u << i;
      }
      const int doc_up = __shfl_up_sync(0xffffffffu, doc, 1);
      const bool head = valid && (lane == 0 || doc_up != doc);
      for (int nb = 0; nb < a.n_nb; ++nb, ++blk) {
        const int b = blk & 1;
        const int t0 = nb * NB;
        __syncwarp();
        for (int i = lane; i < NB; i += 32) {
          const int t = t0 + i;
          int v = -1;
          if (t < a.n_rows) {
            const int sq = seq_of_row(a.q_seq_off, a.n_seq, t);
            const bool end = (t + 1 == a.q_seq_off[sq + 1]) || (i == NB - 1);
            v = sq | (end ? 256 : 0);
          }
          s_col[i] = (int16_t)v;
        }
        __syncwarp();
        if (!mbar_wait(smem_u32(&tfull[b]), (blk >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float m = -INFINITY;
#pragma unroll 1
        for (int j0 = 0; j0 < NB; j0 += 32) {
          float v[32];
          tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * NB + j0), v);
          tmem_ld_wait();
          if (j0 + 32 >= NB) {  // the whole accumulator is in registers
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[b]));
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int cv = s_col[j0 + j];  // uniform across the warp
            if (cv < 0) break;
            m = fmaxf(m, v[j]);
            if (cv & 256) {
#pragma unroll
              for (int o = 1, i = 0; o < 32; o <<= 1, ++i) {
                const float mo = __shfl_down_sync(0xffffffffu, m, o);
                if (same & (1u << i)) m = fmaxf(m, mo);
              }
              if (head) atomicMax(a.doc_key + (size_t)(cv & 255) * a.n_docs + doc, ord_f32(m));
              m = -INFINITY;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
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

template <int NB>
msa_status launch_nb(const RoutePlan& p, cudaStream_t st) {
  using C = PfCfg<NB>;
  CUtensorMap ma, mb;
  if (!make_map_2d(&ma, p.kbar_r, p.n_chunks, kM) || !make_map_2d(&mb, p.qhat, p.n_rows, NB))
    return fail(MSA_ERR_CUDA, "route: cannot encode TMA tensor maps (cuTensorMapEncodeTiled)");
  PfArgs a{};
  a.invk = p.kr_inv_norm;
  a.chunk_doc = p.chunk_doc;
  a.doc_key = p.doc_key;
  a.n_chunks = p.n_chunks;
  a.n_docs = p.n_docs;
  a.n_rows = p.n_rows;
  a.n_seq = p.n_seq;
  a.n_tiles = (int)((p.n_chunks + kM - 1) / kM);
  a.n_nb = (p.n_rows + NB - 1) / NB;
  for (int i = 0; i <= p.n_seq; ++i) a.q_seq_off[i] = p.q_seq_off[i];
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(score_pf_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return cuda_fail(e, "route: many-row scorer shared memory");
    attr_set = true;
  }
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = a.n_tiles < sms ? a.n_tiles : sms;
  cudaError_t e = launch_pdl(score_pf_kernel<NB>, dim3(grid), dim3(kThreads), (size_t)C::kSmem, st, ma, mb, a);
  if (e != cudaSuccess) return cuda_fail(e, "route: score (tensor cores, many rows)");
  return launch_check("route: score (tensor cores, many rows)");
}

}  // namespace

bool score_pf_supported(const RoutePlan& p) {
  // eight routing heads (K = 1,024); 16-byte aligned tensor-map bases
  return p.hr == kHeads && p.n_chunks > 0 && p.qhat != nullptr &&
         (reinterpret_cast<uintptr_t>(p.kbar_r) & 15) == 0 && (reinterpret_cast<uintptr_t>(p.qhat) & 15) == 0;
}

msa_status launch_score_pf(const RoutePlan& p, cudaStream_t st) {
  if (p.n_rows <= 128) return launch_nb<128>(p, st);
  return launch_nb<256>(p, st);
}

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
