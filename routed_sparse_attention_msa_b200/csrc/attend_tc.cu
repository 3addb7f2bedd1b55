// Sparse attention for many query rows per sequence (prefill), on the tensor
// cores.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — the pooled
// K/V of the selected documents joined to the K/V of the query's recent context;
// Parallel (document-wise) RoPE and Global RoPE offset by k (Figure 2)]
//
// Same result as the split-K kernel in attend.cu (which stays the decoding
// path): every query row attends over its sequence's selected pooled K/V and
// its local K/V up to its own position, GQA, softmax in fp32. With tens of
// rows per sequence the logits and P.V are dense contractions, so here a CTA
// owns 128 query vectors (rt rows x the GQA group's q heads) of one kv head
// and walks the key list in blocks of 64:
//   S = Q K^T     tcgen05 M128 x N64 x K128 into TMEM,
//   softmax       two threads per query vector (its TMEM lane; one per 32-key
//                 half of the block, exchanging the block max through shared
//                 memory): running max and sum in fp32, the block's P
//                 rounded to bf16 into shared memory,
//   O += P V      tcgen05 M128 x N128 x K64, accumulated in TMEM across
//                 blocks (P is taken against a reference max that moves only
//                 when the running max passes it by more than 2^11.5; then
//                 the two threads rescale their halves of the O row in TMEM).
// When (tiles x kv heads) would not fill the GPU, the key blocks are split
// across CTAs: the splits of a (tile, kv head), at most 8, are one
// thread-block cluster; each leaves its unnormalised partial (o, m, l) in its
// shared memory and the cluster's CTAs share out the query vectors and merge
// the splits by log-sum-exp straight from each other's shared memory.
// The rotated queries and local keys are split into a bf16 high part and the
// bf16 rounding of the remainder (the local keys by rope_rows), and S sums
// Qhi Khi + Qlo Khi + Qhi Klo (the Qlo Klo term is below 2^-16 of the
// product), so the logits keep fp32 accuracy. The pooled memory keys are bf16
// already (exact). Key blocks are staged two deep: the next block's key and
// value rows are copied by cp.async (keys straight into their swizzled
// places) while the current block's S, softmax and P.V run; the values are
// then transposed shared-to-shared, so every MMA operand is K-major with the
// 128-byte swizzle.
// Every mbarrier wait is bounded in time, and every warp is reconverged
// (__all_sync) after it: lanes leave a polling loop on different iterations,
// and a diverged warp would run the softmax lane group by lane group.
#include <cuda.h>

#include "attend_params.cuh"
#include "tc_ptx.cuh"

namespace msa {
namespace {

using namespace tc;

constexpr int kVec = kAttnTcVec;  // query vectors per CTA = TMEM lanes
constexpr int kNK = 64;           // keys per block
constexpr int kThreadsTc = 256;  // 8 warps: (lane quadrant, half) pairs
constexpr int kQAtom = kVec * 128;  // 16 KB: 128 rows x 64 dims (bf16)
constexpr int kKAtom = kNK * 128;   // 8 KB: 64 keys x 64 dims
constexpr int kVRow = 272;          // bytes per staged value row (256 + 16)
constexpr int offQhi = 0;
constexpr int offQlo = offQhi + 2 * kQAtom;
constexpr int offStage = offQlo + 2 * kQAtom;  // two stages of one key block each:
constexpr int stKhi = 0;                       //   keys (bf16, or the high halves), 2 atoms
constexpr int stKlo = stKhi + 2 * kKAtom;      //   low halves of local keys, 2 atoms
constexpr int stV = stKlo + 2 * kKAtom;        //   value rows as stored [64][272 B]
constexpr int kStageTc = stV + kNK * kVRow;    // 50,176 B
constexpr int offVT = offStage + 2 * kStageTc;  // 128 dims x 64 keys
constexpr int offP = offVT + 128 * 128;         // 128 vectors x 64 keys
constexpr int offIdx = offP + kVec * 128;       // [2 blocks][64] bank-row indices
constexpr int offMax = offIdx + 2 * kNK * 8;    // [2][128] block maxima, then the two partial sums
constexpr int offBar = offMax + 2 * kVec * 4;
constexpr int kSmemTc = 1024 + offBar + 64;
static_assert(kStageTc % 1024 == 0 && offStage % 1024 == 0 && offVT % 1024 == 0 && offP % 1024 == 0,
              "128-byte-swizzle atoms start on 1024-byte boundaries");
static_assert(kSmemTc <= 227 * 1024, "shared memory per CTA");
constexpr int kTmemCols = 256;  // S: columns 0..63, O block: 128..255
constexpr int kMaxClusterTc = 8;  // key splits per (tile, kv head): one portable cluster
constexpr int kPO = kHeadDim + 4;  // row stride (floats) of a CTA's partial output in shared memory
static_assert(kVec * (kPO + 2) * 4 <= 2 * kStageTc, "the partial fits the stages");
// instruction descriptors: D fp32, A/B bf16, K-major; M = 128; N = 64 or 128
constexpr uint32_t kIdescS = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kNK >> 3) << 17) | (8u << 24);
constexpr uint32_t kIdescO = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(128 >> 3) << 17) | (8u << 24);

// 16-byte piece c (0..7) of row r of a 128-byte-swizzled K-major atom.
__device__ __forceinline__ uint8_t* swz(uint8_t* atom, int r, int c) { return atom + r * 128 + ((c ^ (r & 7)) << 4); }

__device__ __forceinline__ void cp16_tc(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit_tc() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait_tc() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ float bf_round(float x) { return __uint_as_float(f2bf_bits(x) << 16); }

// ---- thread-block cluster: the key splits of one (tile, kv head)
__device__ __forceinline__ uint32_t cluster_rank_tc() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_tc() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_addr(const void* local, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  return a;
}
__device__ __forceinline__ float ld_cluster(uint32_t a) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_cluster4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a) : "memory");
  return v;
}

// Eight fp32 values -> 16-byte bf16 high part and 16-byte bf16 remainder.
__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
  float h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = bf_round(x[i]);
    l[i] = x[i] - h[i];
  }
  hi = make_uint4(pack_bf2(h[0], h[1]), pack_bf2(h[2], h[3]), pack_bf2(h[4], h[5]), pack_bf2(h[6], h[7]));
  lo = make_uint4(pack_bf2(l[0], l[1]), pack_bf2(l[2], l[3]), pack_bf2(l[4], l[5]), pack_bf2(l[6], l[7]));
}

__global__ void __launch_bounds__(kThreadsTc, 1) attend_tc_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int64_t* s_idx = reinterpret_cast<int64_t*>(smem + offIdx);  // [2][64] bank rows of two blocks' memory keys
  float* s_max = reinterpret_cast<float*>(smem + offMax);      // [half][vector]
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + offBar);  // [0]: S committed, [1]: P.V committed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q = warp & 3, hs = warp >> 2;  // TMEM lane quadrant; which half of keys / dimensions
  const int v = 32 * q + lane;             // this thread's query vector (TMEM lane)
  const int tile = blockIdx.x, kvh = blockIdx.y, sp_idx = blockIdx.z;
  const int s = seq_of(p.tile_off, p.n_seq, tile);
  const int row0 = p.q_seq_off[s] + (tile - p.tile_off[s]) * p.rt;
  const int nr = min(p.rt, p.q_seq_off[s + 1] - row0);
  const int g0 = p.q_start[s] + (row0 - p.q_seq_off[s]);  // active index of the tile's first row
  const int n_loc_s = p.loc_off[s + 1] - p.loc_off[s];
  const int lvis = max(0, min(n_loc_s, g0 + nr));  // local keys visible to the last row
  const size_t row_stride = (size_t)p.hkv * kHeadDim;

  // the query vector: row rr of the tile, q head gg of the group
  const int rr = v / p.group, gg = v % p.group;
  const bool vvalid = rr < nr;
  const int gv = vvalid ? g0 + rr : -1;

  if (tid == 0) {
    mbar_init(smem_u32(&bar[0]), 1);
    mbar_init(smem_u32(&bar[1]), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"((uint32_t)kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  pdl_wait();  // the rotated rows and the selection come from earlier kernels
  pdl_trigger();
  // the sequence's memory rows: the gather listing, or in the routed form the chunks of its
  // selected documents in rank order (their first list positions scanned in shared memory)
  __shared__ int64_t s_pre[kDecRoutedMaxK + 1], s_c0[kDecRoutedMaxK], s_wsum[kThreadsTc / 32];
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
    if (lane == 31) s_wsum[warp] = x;
    __syncthreads();
    for (int j = 0; j < warp; ++j) x += s_wsum[j];
    if (tid < p.top_k) {
      s_pre[tid] = x - cnt;
      s_c0[tid] = c0;
    }
    if (tid == p.top_k - 1) s_pre[p.top_k] = x;
    __syncthreads();
    n_mem = min(s_pre[p.top_k], p.max_sel);
  } else {
    mem_base = __ldg(p.sel_off + s);
    n_mem = __ldg(p.sel_off + s + 1) - mem_base;
  }
  const int64_t n_keys = n_mem + lvis;
  // this CTA's share of the key blocks (split-K when the grid is small)
  const int64_t n_blocks = (n_keys + kNK - 1) / kNK;
  const int64_t per = (n_blocks + p.n_splits - 1) / p.n_splits;
  const int64_t k_begin = min(n_keys, (int64_t)sp_idx * per * kNK);
  const int64_t k_end = min(n_keys, k_begin + per * kNK);
  const int nblk = (int)((k_end - k_begin + kNK - 1) / kNK);

  // Key blocks are staged two deep: block b + 1's rows are copied by cp.async
  // while block b's S, softmax and P.V run. The bank row of memory key j of
  // block b is read from the selection list one block before the copy.
  auto load_idx = [&](int b, int j) -> int64_t {
    const int64_t key = k_begin + (int64_t)b * kNK + j;
    if (b >= nblk || key >= k_end || key >= n_mem) return -1;
    if (!routed) return p.sel_chunk ? __ldcg(p.sel_chunk + mem_base + key) : mem_base + key;
    int lo = 0, hi = p.top_k - 1;  // the last document whose first list position is <= key
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_pre[mid] <= key) lo = mid; else hi = mid - 1;
    }
    return s_c0[lo] + (key - s_pre[lo]);
  };
  auto issue = [&](int b) {
    if (b < nblk) {
      uint8_t* stg = smem + offStage + (b & 1) * kStageTc;
      const int64_t kb = k_begin + (int64_t)b * kNK;
      const int nb = (int)min((int64_t)kNK, k_end - kb);
      const bool has_local = kb + nb > n_mem;
      const int64_t* idx = s_idx + (b & 1) * kNK;
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // 64 rows x 16 pieces of 16 bytes; 16 threads per row
        const int id = tid + u * kThreadsTc;
        const int jj = id >> 4, c = id & 15;
        const int64_t key = kb + jj;
        uint8_t* dk = swz(stg + stKhi + (c >> 3) * kKAtom, jj, c & 7);
        uint8_t* dl = swz(stg + stKlo + (c >> 3) * kKAtom, jj, c & 7);
        uint8_t* dv = stg + stV + jj * kVRow + 16 * c;
        if (jj < nb && key < n_mem) {
          const size_t off = ((size_t)idx[jj] * row_stride + (size_t)kvh * kHeadDim) * 2 + 16 * c;
          cp16_tc(dk, reinterpret_cast<const uint8_t*>(p.mem_k) + off);
          cp16_tc(dv, reinterpret_cast<const uint8_t*>(p.mem_v) + off);
          if (has_local) *reinterpret_cast<uint4*>(dl) = make_uint4(0, 0, 0, 0);
        } else if (jj < nb) {  // a local key: rotated by rope_rows, bf16 high halves then low halves
          const size_t lrow = (size_t)(p.loc_off[s] + (key - n_mem)) * p.hkv + kvh;
          const uint8_t* kr = reinterpret_cast<const uint8_t*>(p.krot) + lrow * 512;
          cp16_tc(dk, kr + 16 * c);
          cp16_tc(dl, kr + 256 + 16 * c);
          cp16_tc(dv, reinterpret_cast<const uint8_t*>(p.v_loc + lrow * kHeadDim) + 16 * c);
        } else {
          *reinterpret_cast<uint4*>(dv) = make_uint4(0, 0, 0, 0);  // P is 0 here; 0 x NaN would not be
        }
      }
    }
    cp_commit_tc();
  };
  if (tid < kNK) {
    s_idx[tid] = load_idx(0, tid);
    s_idx[kNK + tid] = load_idx(1, tid);
  }

  {  // Q (high and low parts): this thread stages its vector's 64-dimension atom hs
    const float4* qv = reinterpret_cast<const float4*>(
        p.qrot + ((size_t)(row0 + (vvalid ? rr : 0)) * p.hq + kvh * p.group + gg) * kHeadDim + 64 * hs);
#pragma unroll
    for (int c0 = 0; c0 < 8; c0 += 4) {
      float4 x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = vvalid ? __ldg(qv + 2 * c0 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u;
        const float f[8] = {x[2 * u].x, x[2 * u].y, x[2 * u].z, x[2 * u].w,
                            x[2 * u + 1].x, x[2 * u + 1].y, x[2 * u + 1].z, x[2 * u + 1].w};
        uint4 hi, lo;
        split8(f, hi, lo);
        *reinterpret_cast<uint4*>(swz(smem + offQhi + hs * kQAtom, v, c)) = hi;
        *reinterpret_cast<uint4*>(swz(smem + offQlo + hs * kQAtom, v, c)) = lo;
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)(32 * q) << 16;
  const uint32_t tmem_o = tmem + 128;

  // Softmax state of the vector (identical in both of its threads). P is
  // taken relative to m_ref (log2 units), which moves only when the running
  // max exceeds it by more than 11.5 (then both threads rescale their halves
  // of the O row in TMEM), so P <= 2^11.5 and P.V accumulates in TMEM across
  // blocks. l_own sums this thread's keys only; the halves add at the end.
  float m_ref = -INFINITY, l_own = 0.f;
  uint32_t phase_s = 0, phase_pv = 0;
  bool ok = true;
  int pv_issued = 0;

  // S of block b goes to TMEM columns 64 (b & 1) .. + 63 (O takes 128 .. 255),
  // so block b + 1's S runs on the tensor cores while block b's softmax runs.
  auto issue_s = [&](int b) {  // one thread; block b's rows are in its stage and visible to the async proxy
    const int64_t kb = k_begin + (int64_t)b * kNK;
    const bool has_local = kb + (int)min((int64_t)kNK, k_end - kb) > n_mem;
    const uint8_t* stg = smem + offStage + (b & 1) * kStageTc;
    const uint32_t ds = tmem + (uint32_t)(64 * (b & 1));
    tc_fence_after();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t qa = (uint32_t)((k >> 2) * kQAtom + (k & 3) * 32);
      const uint32_t ko = (uint32_t)((k >> 2) * kKAtom + (k & 3) * 32);
      const uint64_t dkhi = sw128_desc(smem_u32(stg + stKhi) + ko);
      tc_mma(ds, sw128_desc(smem_u32(smem + offQhi) + qa), dkhi, kIdescS, k > 0 ? 1u : 0u);
      tc_mma(ds, sw128_desc(smem_u32(smem + offQlo) + qa), dkhi, kIdescS, 1u);
      if (has_local)
        tc_mma(ds, sw128_desc(smem_u32(smem + offQhi) + qa), sw128_desc(smem_u32(stg + stKlo) + ko), kIdescS, 1u);
    }
    tc_commit(smem_u32(&bar[0]));
  };
  issue(0);
  issue(1);
  if (nblk > 0) {
    cp_wait_tc<1>();  // block 0's copies (this thread's)
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) issue_s(0);
  }

  for (int b = 0; b < nblk; ++b) {
    const int64_t kb = k_begin + (int64_t)b * kNK;
    const int nb = (int)min((int64_t)kNK, k_end - kb);
    uint8_t* stg = smem + offStage + (b & 1) * kStageTc;
    const int64_t r2 = tid < kNK ? load_idx(b + 2, tid) : -1;  // stored before block b + 2's copies go out
    // ---- S of block b is done; so is block b - 1's P.V (V^T, P and O are free)
    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar[0]), phase_s, abort_flag));
    phase_s ^= 1;
    if (ok && b > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar[1]), phase_pv, abort_flag));
      phase_pv ^= 1;
    }
    cp_wait_tc<0>();  // this thread's copies of block b + 1
    fence_proxy_async_smem();
    tc_fence_before();
    if (!__syncthreads_and(ok)) { ok = false; break; }
    tc_fence_after();
    if (tid == 0 && b + 1 < nblk) issue_s(b + 1);  // overlaps this block's softmax

    {  // V^T from the staged rows: this thread takes keys 2 jp, 2 jp + 1 and dimensions 16 dg .. 16 dg + 15
      const int jp = tid & 31, dg = tid >> 5;
      uint4 x[2][2];
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2)
#pragma unroll
        for (int i = 0; i < 2; ++i)
          x[k2][i] = *reinterpret_cast<const uint4*>(stg + stV + (2 * jp + k2) * kVRow + 32 * dg + 16 * i);
#pragma unroll
      for (int d = 0; d < 16; ++d) {
        const uint4& a = x[0][d >> 3];
        const uint4& bq = x[1][d >> 3];
        const int w = (d >> 1) & 3;
        const uint32_t wa = w == 0 ? a.x : w == 1 ? a.y : w == 2 ? a.z : a.w;
        const uint32_t wb = w == 0 ? bq.x : w == 1 ? bq.y : w == 2 ? bq.z : bq.w;
        const int dim = 16 * dg + d;
        *reinterpret_cast<uint32_t*>(swz(smem + offVT, dim, jp >> 2) + 4 * (jp & 3)) =
            __byte_perm(wa, wb, (d & 1) ? 0x7632 : 0x5410);
      }
    }

    // ---- softmax: this thread's 32 keys (32 hs .. 32 hs + 31) of its vector
    float sv[32];
    tmem_ld32(tmem + (uint32_t)(64 * (b & 1)) + lane_base + 32 * hs, sv);
    tmem_ld_wait();
    // Logits in log2 units (scale * log2 e) so that P = 2^(s - m_ref). Key j
    // of the block is visible to this vector iff j < jvis: the block's memory
    // keys always, its local keys up to the row's own position.
    const int jmem = (int)max((int64_t)0, min((int64_t)nb, n_mem - kb));  // memory keys in the block
    const int jloc = (int)(gv - max((int64_t)0, kb - n_mem)) + 1;         // local keys it sees
    const int jvis = (!vvalid ? 0 : min(nb, jmem + max(0, min(nb - jmem, jloc)))) - 32 * hs;
    const float sl2 = p.scale * 1.4426950408889634f;
    float bmo = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      sv[j] = j < jvis ? sv[j] * sl2 : -INFINITY;
      bmo = fmaxf(bmo, sv[j]);
    }
    s_max[hs * kVec + v] = bmo;
    if (tid < kNK) s_idx[(b & 1) * kNK + tid] = r2;  // block b + 2's rows (block b's copies went out long ago)
    __syncthreads();  // also: every thread has read block b's staged values
    issue(b + 2);     // into block b's stage (its S is done, its values transposed)
    const float bm = fmaxf(s_max[v], s_max[kVec + v]);
    const bool move = bm > m_ref + 11.5f;  // 2^11.5 ~ e^8; also when m_ref is -inf and bm finite
    const float corr = !move ? 1.f : (m_ref == -INFINITY ? 0.f : exp2f(m_ref - bm));
    if (move) m_ref = bm;
    const float mr = m_ref == -INFINITY ? 0.f : m_ref;  // all P are 0 then (2^-inf)
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float pr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        pr[i] = exp2f(sv[8 * c + i] - mr);
        sum += pr[i];
      }
      *reinterpret_cast<uint4*>(swz(smem + offP, v, 4 * hs + c)) =
          make_uint4(pack_bf2(pr[0], pr[1]), pack_bf2(pr[2], pr[3]), pack_bf2(pr[4], pr[5]), pack_bf2(pr[6], pr[7]));
    }
    l_own = l_own * corr + sum;
    // rescale this thread's half of the O row when any lane of the warp moved its reference
    if (b > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float t[16];
        tmem_ld16(tmem_o + lane_base + 64 * hs + 16 * cc, t);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) t[j] *= corr;
        tmem_st16(tmem_o + lane_base + 64 * hs + 16 * cc, t);
      }
      tmem_st_wait();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O += P V (accumulated in TMEM; waited for before V^T, P and O are touched again)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < kNK / 16; ++k)
        tc_mma(tmem_o, sw128_desc(smem_u32(smem + offP) + k * 32), sw128_desc(smem_u32(smem + offVT) + k * 32),
               kIdescO, (b > 0 || k > 0) ? 1u : 0u);
      tc_commit(smem_u32(&bar[1]));
    }
    ++pv_issued;
  }
  if (ok && pv_issued > 0) {  // the last block's P.V
    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar[1]), phase_pv, abort_flag));
    phase_pv ^= 1;
    ok = __syncthreads_and(ok);
  }
  if (!ok && tid == 0) {  // a wait ran out: let the MMAs in flight finish (bounded) before TMEM is freed
    const uint64_t t0 = globaltimer();
    while ((!mbar_try(smem_u32(&bar[0]), phase_s ^ 1) || !mbar_try(smem_u32(&bar[1]), phase_pv ^ 1)) &&
           globaltimer() - t0 < kWaitLimitNs) {
    }
  }
  cp_wait_tc<0>();  // no copy in flight
  const int blk = ok ? nblk : 0;
  tc_fence_after();
  // the vector's sum over both halves
  s_max[hs * kVec + v] = l_own;
  __syncthreads();
  const float l = s_max[v] + s_max[kVec + v];
  const int row = row0 + rr, h = kvh * p.group + gg;
  const size_t rh = (size_t)row * p.hq + h;

  if (p.n_splits > 1) {
    // ---- split-K inside the cluster: this CTA's unnormalised partial (o, m, l) goes to its
    // shared memory (the stages, idle now); after the barrier CTA r merges the vectors v with
    // v % splits == r from every CTA's memory, and the second barrier keeps that memory alive
    float* po = reinterpret_cast<float*>(smem + offStage);  // [128 vectors][kPO]
    float* pm = po + kVec * kPO;                            // [128]
    float* pl = pm + kVec;                                  // [128]
    const bool have = ok && blk > 0;  // uniform: every thread of the CTA walked the same blocks
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      float t[16];
      if (have) {
        tmem_ld16(tmem_o + lane_base + 64 * hs + 16 * cc, t);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) t[j] = 0.f;
      }
      float4* dst = reinterpret_cast<float4*>(po + v * kPO + 64 * hs + 16 * cc);
      dst[0] = make_float4(t[0], t[1], t[2], t[3]);
      dst[1] = make_float4(t[4], t[5], t[6], t[7]);
      dst[2] = make_float4(t[8], t[9], t[10], t[11]);
      dst[3] = make_float4(t[12], t[13], t[14], t[15]);
    }
    if (hs == 0) {
      pm[v] = m_ref;
      pl[v] = have ? l : 0.f;
    }
    cluster_sync_tc();
    const int ns = p.n_splits;
    if (vvalid && v % ns == (int)cluster_rank_tc()) {
      float mj[kMaxClusterTc], lj[kMaxClusterTc];
#pragma unroll
      for (int j = 0; j < kMaxClusterTc; ++j) {
        lj[j] = 0.f;
        mj[j] = -INFINITY;
        if (j < ns) {
          lj[j] = ld_cluster(cluster_addr(pl + v, j));
          mj[j] = ld_cluster(cluster_addr(pm + v, j));
        }
      }
      float mm = -INFINITY;
#pragma unroll
      for (int j = 0; j < kMaxClusterTc; ++j)
        if (lj[j] > 0.f) mm = fmaxf(mm, mj[j]);
      float wj[kMaxClusterTc], wsum = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxClusterTc; ++j) {
        wj[j] = lj[j] > 0.f ? exp2f(mj[j] - mm) : 0.f;
        wsum += lj[j] * wj[j];
      }
      const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
      const size_t base = rh * kHeadDim + 64 * hs;
#pragma unroll 1
      for (int d = 0; d < 64; d += 8) {
        float r[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < kMaxClusterTc; ++j) {
          if (wj[j] > 0.f) {
            const uint32_t a = cluster_addr(po + v * kPO + 64 * hs + d, j);
            const float4 x = ld_cluster4(a), y = ld_cluster4(a + 16);
            r[0] += wj[j] * x.x; r[1] += wj[j] * x.y; r[2] += wj[j] * x.z; r[3] += wj[j] * x.w;
            r[4] += wj[j] * y.x; r[5] += wj[j] * y.y; r[6] += wj[j] * y.z; r[7] += wj[j] * y.w;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) r[i] *= inv;
        *reinterpret_cast<uint4*>(p.out + base + d) =
            make_uint4(pack_bf2(r[0], r[1]), pack_bf2(r[2], r[3]), pack_bf2(r[4], r[5]), pack_bf2(r[6], r[7]));
        if (p.out_f32) {
          reinterpret_cast<float4*>(p.out_f32 + base + d)[0] = make_float4(r[0], r[1], r[2], r[3]);
          reinterpret_cast<float4*>(p.out_f32 + base + d)[1] = make_float4(r[4], r[5], r[6], r[7]);
        }
      }
      if (p.lse && hs == 0) p.lse[rh] = wsum > 0.f ? (mm + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
    }
    cluster_sync_tc();
  } else if (ok) {  // ---- one CTA per (tile, kv head): normalised output, log-sum-exp
    const float inv = l > 0.f ? 1.0f / l : 0.f;
    const size_t base = rh * kHeadDim + 64 * hs;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      float t[16];
      if (blk > 0) {  // uniform: every thread of the CTA walked the same blocks
        tmem_ld16(tmem_o + lane_base + 64 * hs + 16 * cc, t);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) t[j] = 0.f;
      }
      if (vvalid) {
#pragma unroll
        for (int j = 0; j < 16; j += 8) {
          float r[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) r[i] = t[j + i] * inv;
          *reinterpret_cast<uint4*>(p.out + base + 16 * cc + j) =
              make_uint4(pack_bf2(r[0], r[1]), pack_bf2(r[2], r[3]), pack_bf2(r[4], r[5]), pack_bf2(r[6], r[7]));
          if (p.out_f32) {
            reinterpret_cast<float4*>(p.out_f32 + base + 16 * cc + j)[0] = make_float4(r[0], r[1], r[2], r[3]);
            reinterpret_cast<float4*>(p.out_f32 + base + 16 * cc + j)[1] = make_float4(r[4], r[5], r[6], r[7]);
          }
        }
      }
    }
    if (vvalid && hs == 0 && p.lse)  // m_ref and l are in log2 units
      p.lse[rh] = l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTmemCols));
  }
}

}  // namespace

msa_status launch_attend_tc(const AttnParams& P, cudaStream_t st) {
  static std::atomic<uint64_t> attr{0};
  cudaError_t e = smem_limit_once(attend_tc_kernel, kSmemTc, attr);
  if (e != cudaSuccess) return cuda_fail(e, "attend: tensor-core kernel shared memory");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P.n_tiles, (unsigned)P.hkv, (unsigned)P.n_splits);
  cfg.blockDim = dim3(kThreadsTc);
  cfg.dynamicSmemBytes = (size_t)kSmemTc;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;  // the key splits of a (tile, kv head): one cluster
  at[1].val.clusterDim.x = 1;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = (unsigned)P.n_splits;
  cfg.attrs = at;
  cfg.numAttrs = P.n_splits > 1 ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, attend_tc_kernel, P);
  if (e != cudaSuccess) return cuda_fail(e, "attend: tensor cores (many rows)");
  return launch_check("attend: tensor cores (many rows)");
}

int attend_tc_error_take() {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_error, sizeof v) != cudaSuccess) return 0;
  if (v) {
    int z = 0;
    cudaMemcpyToSymbol(g_tc_error, &z, sizeof z);
  }
  return v;
}

}  // namespace msa
