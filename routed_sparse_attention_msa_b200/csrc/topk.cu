// Top-k documents per sequence from the per-document routing scores.
//
// ["MSA: Memory Sparse Attention", Overall Design: Architecture — selects the
// Top-k documents; "MSA-arXiv26", 核心方法 — cosine similarity, top-k documents]
//
// Every document gets a 64-bit key: the order-preserving encoding of its
// score in the high word and (0xFFFFFFFF - id) in the low word, so the total
// order "score descending, then id ascending" is plain unsigned comparison
// and all keys are distinct. A document that was never scored (no chunks)
// has score word 0, below every real score.
//
// k <= 16: each warp keeps its best 16 keys sorted across lanes 0..15 (up to
// 2,048 documents: one CTA per sequence, no cross-CTA merge). A batch
// of 32 new keys is first tested against the 16th key with one ballot (after
// the first batches almost every batch is skipped); otherwise the batch is
// sorted by a 32-lane bitonic network and merged with the list by one
// bitonic merge (the list in lanes 0..15, the batch's best 16 reversed into
// lanes 16..31). Warps (as a tree), then CTAs, are combined by the same
// merge. Beyond 2,048 documents a sequence is split into CTAs of 2,048 and
// the last CTA of the sequence to finish (atomic ticket, no waiting) merges
// the CTAs' lists. 16 < k <= 32: the same structure with per-key insertion by shuffles.
// k > 32: one CTA per sequence runs an 8-pass radix select on the keys,
// collects the k keys at or above the k-th and sorts them.
#include "msa_internal.cuh"

namespace msa {
namespace {

constexpr int kWarps = 8;
constexpr int kDocsPerWarp = 128;
constexpr int kDocsPerCta = kWarps * kDocsPerWarp;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ uint64_t doc_key64(uint32_t score_key, int64_t doc) {
  return ((uint64_t)score_key << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)doc);
}

// Insert this lane's candidate `key` into the warp's sorted list (lane i holds
// the i-th largest, i < k; lanes >= k are unused). Keys are distinct.
__device__ __forceinline__ void warp_insert(uint64_t& list, uint64_t key, int k, int lane) {
  uint64_t thr = __shfl_sync(0xffffffffu, list, k - 1);
  unsigned m = __ballot_sync(0xffffffffu, key > thr);
  while (m) {
    int src = __ffs(m) - 1;
    uint64_t v = __shfl_sync(0xffffffffu, key, src);
    unsigned gt = __ballot_sync(0xffffffffu, lane < k && list > v);
    int pos = __popc(gt);
    uint64_t up = __shfl_up_sync(0xffffffffu, list, 1);
    if (lane < k) {
      if (lane == pos) list = v;
      else if (lane > pos) list = up;
    }
    thr = __shfl_sync(0xffffffffu, list, k - 1);
    m &= ~(1u << src);
    m &= __ballot_sync(0xffffffffu, key > thr);
  }
}

// 32 keys, one per lane, sorted descending across the warp.
__device__ __forceinline__ uint64_t warp_sort32_desc(uint64_t x, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t y = __shfl_xor_sync(kFull, x, stride);
      const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
      x = keep_max ? (x > y ? x : y) : (x < y ? x : y);
    }
  }
  return x;
}

// list: lanes 0..15 hold 16 keys sorted descending. other: lanes 0..15 hold
// another such list. Returns the best 16 of both, sorted, in lanes 0..15.
__device__ __forceinline__ uint64_t warp_merge16(uint64_t list, uint64_t other, int lane) {
  const uint64_t rev = __shfl_sync(kFull, other, 31 - lane);  // lane 16+i <- other[15-i]
  uint64_t x = lane < 16 ? list : rev;                        // bitonic: descending then ascending
#pragma unroll
  for (int stride = 16; stride > 0; stride >>= 1) {
    const uint64_t y = __shfl_xor_sync(kFull, x, stride);
    x = (lane & stride) == 0 ? (x > y ? x : y) : (x < y ? x : y);
  }
  return x;
}

// Fold one batch of 32 keys (one per lane) into the list (lanes 0..15).
__device__ __forceinline__ void warp_fold32(uint64_t& list, uint64_t key, int lane) {
  const uint64_t thr = __shfl_sync(kFull, list, 15);
  if (!__any_sync(kFull, key > thr)) return;
  const uint64_t sorted = warp_sort32_desc(key, lane);
  list = warp_merge16(list, sorted, lane);
}

__device__ __forceinline__ void write_result(uint64_t key, int32_t* ids, float* scores) {
  *ids = (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
  *scores = unord_f32((uint32_t)(key >> 32));
}

__global__ void __launch_bounds__(kWarps * 32) topk_warp_kernel(
    const uint32_t* __restrict__ doc_key, int64_t n_docs, int k, uint64_t* __restrict__ cand,
    unsigned* __restrict__ tickets, int32_t* __restrict__ top_ids, float* __restrict__ top_scores,
    float* __restrict__ all_scores) {
  __shared__ uint64_t s_lists[kWarps][32];
  __shared__ bool s_last;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int s = blockIdx.y;
  const int part = blockIdx.x;
  const int n_parts = gridDim.x;
  const uint32_t* keys = doc_key + (size_t)s * n_docs;

  uint64_t list = 0;
  const int64_t w0 = (int64_t)part * kDocsPerCta + (int64_t)wid * kDocsPerWarp;
  for (int it = 0; it < kDocsPerWarp / 32; ++it) {
    int64_t doc = w0 + it * 32 + lane;
    uint64_t key = 0;
    if (doc < n_docs) {
      uint32_t sk = keys[doc];
      key = doc_key64(sk, doc);
      if (all_scores) all_scores[(size_t)s * n_docs + doc] = unord_f32(sk);
    }
    warp_insert(list, key, k, lane);
  }
  s_lists[wid][lane] = list;
  __syncthreads();
  if (wid == 0) {
    uint64_t merged = s_lists[0][lane];
    for (int w = 1; w < kWarps; ++w) warp_insert(merged, lane < k ? s_lists[w][lane] : 0ull, k, lane);
    if (lane < k) cand[((size_t)s * n_parts + part) * k + lane] = merged;
    __threadfence();
    unsigned t = 0;
    if (lane == 0) t = atomicAdd(tickets + s, 1u);
    t = __shfl_sync(0xffffffffu, t, 0);
    s_last = (t == (unsigned)(n_parts - 1));
  }
  __syncthreads();
  if (!s_last || wid != 0) return;
  __threadfence();
  uint64_t fin = 0;
  const uint64_t* c = cand + (size_t)s * n_parts * k;
  for (int64_t i0 = 0; i0 < (int64_t)n_parts * k; i0 += 32) {
    int64_t i = i0 + lane;
    uint64_t key = i < (int64_t)n_parts * k ? __ldcg(c + i) : 0ull;
    warp_insert(fin, key, k, lane);
  }
  const int kk = k < n_docs ? k : (int)n_docs;
  if (lane < kk) write_result(fin, top_ids + (size_t)s * kk + lane, top_scores + (size_t)s * kk + lane);
  if (lane == 0) tickets[s] = 0u;  // ready for the next call
}

// k <= 16, 32 warps per CTA: IT batches of 32 keys per warp (1,024 * IT
// documents per CTA), every key load issued before any merging. The warps'
// lists are combined by a 5-level tree of merges in shared memory. With one
// CTA per sequence (up to 2,048 documents) the result is written directly;
// otherwise each CTA writes its list and the last CTA of the sequence to
// finish (atomic ticket, no waiting) merges them.
constexpr int kWarps16 = 32;
// Measured on 16 sequences x 10,040 documents: one CTA per sequence (16 batches
// per warp) 20 us, CTAs of 1,024 documents with the last-CTA merge 10.6 us; the
// batches of a warp are a dependent chain, so documents are spread over CTAs.
constexpr int kSinglePassDocs = 2 * 1024;  // one CTA per sequence up to this many documents
constexpr int kPartDocs = 2 * 1024;        // documents per CTA beyond it

__device__ __forceinline__ uint64_t tree_merge16(uint64_t (*lists)[16], uint64_t list, int lane, int wid) {
  // lists[w] holds warp w's best 16 (lanes 0..15 of `list` on entry); returns the overall best 16 in warp 0
  if (lane < 16) lists[wid][lane] = list;
  __syncthreads();
#pragma unroll
  for (int half = kWarps16 / 2; half > 0; half >>= 1) {
    if (wid < half) {
      list = warp_merge16(lane < 16 ? lists[wid][lane] : 0ull, lane < 16 ? lists[wid + half][lane] : 0ull, lane);
      __syncwarp();
      if (lane < 16) lists[wid][lane] = list;
    }
    __syncthreads();
  }
  return lane < 16 ? lists[0][lane] : 0ull;
}

template <int IT>
__global__ void __launch_bounds__(kWarps16 * 32) topk16_kernel(
    const uint32_t* __restrict__ doc_key, int64_t n_docs, int k, uint64_t* __restrict__ cand,
    unsigned* __restrict__ tickets, int32_t* __restrict__ top_ids, float* __restrict__ top_scores,
    float* __restrict__ all_scores) {
  __shared__ uint64_t s_lists[kWarps16][16];
  __shared__ bool s_last;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int s = blockIdx.y;
  const int part = blockIdx.x;
  const int n_parts = gridDim.x;
  const uint32_t* keys = doc_key + (size_t)s * n_docs;

  // keys of this warp's slice: document w0 + 32 it + lane
  const int64_t w0 = (int64_t)part * (kWarps16 * 32 * IT) + (int64_t)wid * (32 * IT);
  uint64_t kv[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int64_t doc = w0 + it * 32 + lane;
    kv[it] = 0;
    if (doc < n_docs) {
      const uint32_t sk = __ldcg(keys + doc);
      kv[it] = doc_key64(sk, doc);
      if (all_scores) all_scores[(size_t)s * n_docs + doc] = unord_f32(sk);
    }
  }
  uint64_t list = warp_sort32_desc(kv[0], lane);
#pragma unroll
  for (int it = 1; it < IT; ++it) warp_fold32(list, kv[it], lane);
  uint64_t merged = tree_merge16(s_lists, list, lane, wid);
  if (n_parts == 1) {  // the whole sequence in this CTA
    if (wid == 0 && lane < k) write_result(merged, top_ids + (size_t)s * k + lane, top_scores + (size_t)s * k + lane);
    return;
  }
  if (wid == 0) {
    if (lane < 16) cand[((size_t)s * n_parts + part) * 16 + lane] = merged;
    __threadfence();
    unsigned t = 0;
    if (lane == 0) t = atomicAdd(tickets + s, 1u);
    t = __shfl_sync(kFull, t, 0);
    s_last = (t == (unsigned)(n_parts - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // last CTA: every warp merges a share of the CTAs' lists, then the tree merges the warps'
  const uint64_t* c = cand + (size_t)s * n_parts * 16;
  uint64_t acc = 0;
  for (int pp = wid; pp < n_parts; pp += kWarps16)
    acc = warp_merge16(acc, lane < 16 ? __ldcg(c + (size_t)pp * 16 + lane) : 0ull, lane);
  const uint64_t fin = tree_merge16(s_lists, acc, lane, wid);
  if (wid == 0) {
    if (lane < k) write_result(fin, top_ids + (size_t)s * k + lane, top_scores + (size_t)s * k + lane);
    if (lane == 0) tickets[s] = 0u;  // ready for the next call
  }
}

int g_topk_part = 0;  // testing control: documents per CTA of the k <= 16 path (0: kPartDocs)

int part_docs() { return g_topk_part > 0 ? g_topk_part : kPartDocs; }

int topk16_parts(int64_t n_docs) {
  const int single = g_topk_part > 0 ? g_topk_part : kSinglePassDocs;
  return n_docs <= single ? 1 : (int)((n_docs + part_docs() - 1) / part_docs());
}

// Generic path: one CTA (1024 threads) per sequence.
__global__ void __launch_bounds__(1024) topk_radix_kernel(
    const uint32_t* __restrict__ doc_key, int64_t n_docs, int k, int32_t* __restrict__ top_ids,
    float* __restrict__ top_scores, float* __restrict__ all_scores) {
  extern __shared__ uint64_t s_sel[];  // [pow2 >= k]
  __shared__ unsigned s_hist[256];
  __shared__ uint64_t s_prefix, s_mask;
  __shared__ int s_krem;
  __shared__ unsigned s_count;
  pdl_wait();
  pdl_trigger();
  const int s = blockIdx.x;
  const uint32_t* keys = doc_key + (size_t)s * n_docs;
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_prefix = 0;
    s_mask = 0;
    s_krem = k;
    s_count = 0;
  }
  if (all_scores)
    for (int64_t j = tid; j < n_docs; j += blockDim.x) all_scores[(size_t)s * n_docs + j] = unord_f32(keys[j]);
  __syncthreads();
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += blockDim.x) s_hist[b] = 0;
    __syncthreads();
    const uint64_t pre = s_prefix, msk = s_mask;
    for (int64_t j = tid; j < n_docs; j += blockDim.x) {
      uint64_t key = doc_key64(keys[j], j);
      if ((key & msk) == pre) atomicAdd(&s_hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      int krem = s_krem;
      unsigned cum = 0;
      int b = 255;
      for (; b > 0; --b) {
        if ((int)(cum + s_hist[b]) >= krem) break;
        cum += s_hist[b];
      }
      s_krem = krem - (int)cum;
      s_prefix = pre | ((uint64_t)b << shift);
      s_mask = msk | (0xFFull << shift);
    }
    __syncthreads();
  }
  const uint64_t kth = s_prefix;  // the k-th largest key (keys are distinct)
  int pow2 = 1;
  while (pow2 < k) pow2 <<= 1;
  for (int i = tid; i < pow2; i += blockDim.x) s_sel[i] = 0;
  __syncthreads();
  for (int64_t j = tid; j < n_docs; j += blockDim.x) {
    uint64_t key = doc_key64(keys[j], j);
    if (key >= kth) {
      unsigned p = atomicAdd(&s_count, 1u);
      if (p < (unsigned)k) s_sel[p] = key;
    }
  }
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < pow2; i += blockDim.x) {
        int j = i ^ stride;
        if (j > i) {
          bool desc = (i & size) == 0;
          uint64_t a = s_sel[i], b = s_sel[j];
          if (desc ? (a < b) : (a > b)) {
            s_sel[i] = b;
            s_sel[j] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < k; i += blockDim.x)
    write_result(s_sel[i], top_ids + (size_t)s * k + i, top_scores + (size_t)s * k + i);
}

// Merge of per-shard top-k lists (Memory Parallel): one CTA per sequence
// loads every shard's k (score, local id) pairs, forms the global keys with
// the shard's document offset, sorts them (bitonic, descending) in shared
// memory and keeps the best k. Entries with a negative id are padding.
constexpr int kMaxShards = 64;
struct MergeArgs {
  const int32_t* ids;    // [G, S, k]
  const float* scores;   // [G, S, k]
  int32_t* top_ids;      // [S, k_out]
  float* top_scores;     // [S, k_out]
  int n_shards, n_seq, k, k_out, pow2;
  int64_t id_offset[kMaxShards];
};

__global__ void __launch_bounds__(1024) topk_merge_kernel(const __grid_constant__ MergeArgs a) {
  extern __shared__ uint64_t s_keys[];  // [pow2]
  pdl_wait();
  pdl_trigger();
  const int s = blockIdx.x, tid = threadIdx.x;
  const int n = a.n_shards * a.k;
  for (int i = tid; i < a.pow2; i += blockDim.x) {
    uint64_t key = 0;
    if (i < n) {
      const int g = i / a.k, j = i % a.k;
      const size_t src = ((size_t)g * a.n_seq + s) * a.k + j;
      const int32_t id = a.ids[src];
      if (id >= 0) {
        const float sc = a.scores[src];
        const uint32_t o = __float_as_uint(sc) == 0xff800000u ? 0u : ord_f32(sc);  // -inf: never scored
        key = doc_key64(o, (int64_t)id + a.id_offset[g]);
      }
    }
    s_keys[i] = key;
  }
  __syncthreads();
  for (int size = 2; size <= a.pow2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < a.pow2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool desc = (i & size) == 0;
          const uint64_t x = s_keys[i], y = s_keys[j];
          if (desc ? (x < y) : (x > y)) {
            s_keys[i] = y;
            s_keys[j] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < a.k_out; i += blockDim.x)
    write_result(s_keys[i], a.top_ids + (size_t)s * a.k_out + i, a.top_scores + (size_t)s * a.k_out + i);
}

}  // namespace

msa_status launch_topk_merge(const int32_t* ids, const float* scores, const int64_t* id_offset, int n_shards,
                             int n_seq, int k, int k_out, int32_t* top_ids, float* top_scores, cudaStream_t st) {
  if (n_shards <= 0 || n_shards > kMaxShards) return fail(MSA_ERR_UNSUPPORTED, "topk_merge: %d shards (1..%d)", n_shards, kMaxShards);
  MergeArgs a{};
  a.ids = ids; a.scores = scores; a.top_ids = top_ids; a.top_scores = top_scores;
  a.n_shards = n_shards; a.n_seq = n_seq; a.k = k; a.k_out = k_out;
  int pow2 = 1;
  while (pow2 < n_shards * k) pow2 <<= 1;
  a.pow2 = pow2;
  for (int g = 0; g < n_shards; ++g) a.id_offset[g] = id_offset[g];
  const size_t smem = (size_t)pow2 * sizeof(uint64_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "topk_merge: shared memory");
  }
  cudaError_t e = launch_pdl(topk_merge_kernel, dim3(n_seq), dim3(1024), smem, st, a);
  if (e != cudaSuccess) return cuda_fail(e, "topk_merge");
  return launch_check("topk_merge");
}

size_t topk_workspace(int n_seq, int64_t n_docs, int k) {
  int64_t parts = k <= 16 ? topk16_parts(n_docs) : (n_docs + kDocsPerCta - 1) / kDocsPerCta;
  if (k > 32) return 256;
  const int kc = k <= 16 ? 16 : k;
  return align_up((size_t)n_seq * parts * kc * sizeof(uint64_t), 256) +
         align_up((size_t)n_seq * sizeof(unsigned), 256);
}

// ws must be zero-initialised once (the tickets reset themselves).
msa_status launch_topk(const uint32_t* doc_key, int n_seq, int64_t n_docs, int k, int32_t* top_ids,
                       float* top_scores, float* all_scores, void* ws, cudaStream_t st) {
  if (k > n_docs) k = (int)n_docs;
  if (k <= 32) {
    int64_t parts = (n_docs + kDocsPerCta - 1) / kDocsPerCta;
    const int kc = k <= 16 ? 16 : k;
    uint64_t* cand = reinterpret_cast<uint64_t*>(ws);
    unsigned* tickets = reinterpret_cast<unsigned*>(
        reinterpret_cast<char*>(ws) + align_up((size_t)n_seq * parts * kc * sizeof(uint64_t), 256));
    cudaError_t e;
    if (k <= 16) {
      parts = topk16_parts(n_docs);
      cand = reinterpret_cast<uint64_t*>(ws);
      tickets = reinterpret_cast<unsigned*>(reinterpret_cast<char*>(ws) +
                                            align_up((size_t)n_seq * parts * 16 * sizeof(uint64_t), 256));
      const dim3 grid((unsigned)parts, (unsigned)n_seq);
      const int64_t per_cta = parts == 1 ? n_docs : part_docs();  // documents one CTA covers
      const int it = per_cta <= 1024 ? 1 : per_cta <= 2048 ? 2 : per_cta <= 4096 ? 4 : per_cta <= 8192 ? 8 : 16;
      auto go = [&](auto kernel) {
        return launch_pdl(kernel, grid, dim3(kWarps16 * 32), 0, st, doc_key, n_docs, k, cand, tickets, top_ids,
                          top_scores, all_scores);
      };
      switch (it) {
        case 1: e = go(topk16_kernel<1>); break;
        case 2: e = go(topk16_kernel<2>); break;
        case 4: e = go(topk16_kernel<4>); break;
        case 8: e = go(topk16_kernel<8>); break;
        default: e = go(topk16_kernel<16>); break;
      }
    } else {
      const dim3 grid((unsigned)parts, (unsigned)n_seq);
      e = launch_pdl(topk_warp_kernel, grid, dim3(kWarps * 32), 0, st, doc_key, n_docs, k, cand, tickets, top_ids,
                     top_scores, all_scores);
    }
    if (e != cudaSuccess) return cuda_fail(e, "route: top-k");
    return launch_check("route: top-k");
  }
  int pow2 = 1;
  while (pow2 < k) pow2 <<= 1;
  size_t smem = (size_t)pow2 * sizeof(uint64_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "route: top-k shared memory");
  }
  cudaError_t e = launch_pdl(topk_radix_kernel, dim3(n_seq), dim3(1024), smem, st, doc_key, n_docs, k, top_ids,
                             top_scores, all_scores);
  if (e != cudaSuccess) return cuda_fail(e, "route: top-k (radix)");
  return launch_check("route: top-k (radix)");
}

}  // namespace msa

// Documents per CTA of the k <= 16 top-k in later msa_route calls (1024..16384,
// a power of two: 1,024 per batch of the CTA's 32 warps; 0 restores the
// planned 2,048); returns the previous
// setting. Workspace sizes follow it. A benchmarking control; not declared in
// msa.h.
extern "C" int msa_debug_set_topk_part(int n) {
  const int old = msa::g_topk_part;
  if (n == 0 || (n >= 1024 && n <= 16384 && (n & (n - 1)) == 0)) msa::g_topk_part = n;
  return old;
}
