// Context assembly: the chunk list of each sequence's selected documents,
// and (host content tier, device-pull mode) the copy of their pooled K/V rows
// from mapped pinned host memory into a device staging buffer.
//
// ["MSA: Memory Sparse Attention", Inference Pipeline stage 2 — only the
// selected documents' K-bar/V-bar are brought in and joined to the local
// context; the Memory Parallel paragraph — the content tier is kept in host
// memory and read on selection; "MSA-arXiv26", 核心方法 / Memory Parallel inference (tiered storage)]
#include "msa_internal.cuh"

namespace msa {
namespace {

// One CTA: an exclusive scan over the (sequence, rank) pairs of the selected
// documents' chunk counts gives each document's place in the list; then all
// threads write the list together, output position j taking its document by
// a binary search over the scanned starts (coalesced stores, no per-document
// loop).
constexpr int kIndexThreads = 1024;

// An id outside [0, n_docs) lists no chunks; list positions from `cap` on are
// not written (offsets are clamped to cap), so the list never leaves its buffer.
__global__ void __launch_bounds__(kIndexThreads) gather_index_kernel(
    const int64_t* __restrict__ doc_chunk_off, int64_t n_docs, const int32_t* __restrict__ top_ids, int n_seq,
    int k, int64_t* __restrict__ sel_off, int64_t* __restrict__ sel_chunk, int64_t cap) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t s_start[kIndexThreads], s_c0[kIndexThreads];
  __shared__ int64_t carry;
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int64_t n_pairs = (int64_t)n_seq * k;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < n_pairs; base += kIndexThreads) {
    const int64_t p = base + tid;
    int64_t c0 = 0, n = 0;
    if (p < n_pairs) {
      const int32_t doc = __ldcg(top_ids + p);
      if (doc >= 0 && doc < n_docs) {
        c0 = doc_chunk_off[doc];
        n = doc_chunk_off[doc + 1] - c0;
      }
    }
    int64_t x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int64_t w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int64_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int64_t c_old = carry;
    const int64_t start = c_old + (wid > 0 ? warp_sums[wid - 1] : 0) + x - n;
    s_start[tid] = p < n_pairs ? start : INT64_MAX;
    s_c0[tid] = c0;
    if (p < n_pairs) {
      if (p % k == 0) sel_off[p / k] = min(start, cap);
      if (p == n_pairs - 1) sel_off[n_seq] = min(start + n, cap);
    }
    const int64_t c_new = c_old + warp_sums[31];
    __syncthreads();
    for (int64_t j = c_old + tid; j < min(c_new, cap); j += kIndexThreads) {
      int lo = 0, hi = kIndexThreads - 1;  // the last pair whose start is <= j
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_start[mid] <= j) lo = mid; else hi = mid - 1;
      }
      sel_chunk[j] = s_c0[lo] + (j - s_start[lo]);
    }
    __syncthreads();
    if (tid == 0) carry = c_new;
    __syncthreads();
  }
}

// One warp per selected row: 2 x hkv x 256 B read from mapped host memory.
// Every lane issues all of its 16-byte loads (K and V) before its first store
// so that each warp keeps its whole row in flight over the host link.
constexpr int kPullVecsPerLane = 4;  // hkv * 128 * 2 B / 16 B / 32 lanes, for hkv <= 8

__global__ void gather_pull_kernel(const uint16_t* __restrict__ kbar, const uint16_t* __restrict__ vbar,
                                   const int64_t* __restrict__ sel_total,
                                   const int64_t* __restrict__ sel_chunk, int64_t cap, int hkv,
                                   uint16_t* __restrict__ stage_k, uint16_t* __restrict__ stage_v) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t gw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = min(*sel_total, cap);
  const int vecs = hkv * kHeadDim / 8;  // uint4 per row
  for (int64_t j = gw; j < total; j += nw) {
    const int64_t c = sel_chunk[j];
    const uint4* sk = reinterpret_cast<const uint4*>(kbar + (size_t)c * hkv * kHeadDim);
    const uint4* sv = reinterpret_cast<const uint4*>(vbar + (size_t)c * hkv * kHeadDim);
    uint4* dk = reinterpret_cast<uint4*>(stage_k + (size_t)j * hkv * kHeadDim);
    uint4* dv = reinterpret_cast<uint4*>(stage_v + (size_t)j * hkv * kHeadDim);
    for (int i0 = 0; i0 < vecs; i0 += 32 * kPullVecsPerLane) {
      uint4 a[kPullVecsPerLane], b[kPullVecsPerLane];
#pragma unroll
      for (int u = 0; u < kPullVecsPerLane; ++u) {
        const int i = i0 + u * 32 + lane;
        if (i < vecs) {
          a[u] = sk[i];
          b[u] = sv[i];
        }
      }
#pragma unroll
      for (int u = 0; u < kPullVecsPerLane; ++u) {
        const int i = i0 + u * 32 + lane;
        if (i < vecs) {
          dk[i] = a[u];
          dv[i] = b[u];
        }
      }
    }
  }
}

}  // namespace

msa_status launch_gather_index(const int64_t* doc_chunk_off, int64_t n_docs, const int32_t* top_ids, int n_seq,
                               int k, int64_t* sel_off, int64_t* sel_chunk, int64_t cap, cudaStream_t st) {
  cudaError_t e = launch_pdl(gather_index_kernel, dim3(1), dim3(1024), 0, st, doc_chunk_off, n_docs, top_ids, n_seq,
                             k, sel_off, sel_chunk, cap);
  if (e != cudaSuccess) return cuda_fail(e, "gather: chunk list");
  return launch_check("gather: chunk list");
}

msa_status launch_gather_pull(const msa_bank_layer& b, const int64_t* sel_off, const int64_t* sel_chunk,
                              int64_t cap, uint16_t* stage_k, uint16_t* stage_v, cudaStream_t st) {
  int64_t warps = cap;
  int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  if (blocks < 1) blocks = 1;
  // sel_off[n_seq] is the total row count; the caller passes its address.
  cudaError_t e = launch_pdl(gather_pull_kernel, dim3((unsigned)blocks), dim3(256), 0, st, b.kbar, b.vbar, sel_off,
                             sel_chunk, cap, b.hkv, stage_k, stage_v);
  if (e != cudaSuccess) return cuda_fail(e, "gather: device pull from host memory");
  return launch_check("gather: device pull from host memory");
}

}  // namespace msa
