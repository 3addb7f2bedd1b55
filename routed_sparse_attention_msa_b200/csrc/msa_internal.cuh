// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "msa.h"

namespace msa {

// ---------------------------------------------------------------- errors
msa_status fail(msa_status s, const char* fmt, ...);
msa_status cuda_fail(cudaError_t e, const char* what);
msa_status launch_check(const char* what);
// Benchmark instrumentation: records the pending debug event `which` (0 begin, 1 end) on st.
void record_debug_event(int which, cudaStream_t st);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device, once per device: the attribute belongs to each device's copy of the
// kernel, so a process that drives several GPUs must set it on every one.
// `done` holds one bit per device ordinal (< 64; others set it every call).
template <typename Kernel>
cudaError_t smem_limit_once(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t)1 << dev : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ------------------------------------------------ programmatic dependent launch
// Every kernel of the path is launched so that it may start while its
// predecessor on the stream is still finishing. Each kernel calls pdl_wait()
// before it reads or writes any memory that another kernel touches (that wait
// returns once the predecessor, and transitively everything before it, has
// completed and its writes are visible), then pdl_trigger() so that its own
// successor can be scheduled. Launched without the attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

constexpr int kHeadDim = 128;
constexpr int kMaxSeq = 256;

// ------------------------------------------------------- small device math
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ float bf1(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// fp32 -> bf16, round to nearest even (NaN kept quiet).
__device__ __forceinline__ uint32_t f2bf_bits(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return u >> 16;
}
__device__ __forceinline__ uint32_t pack_bf2(float lo, float hi) {
  return f2bf_bits(lo) | (f2bf_bits(hi) << 16);
}

// Order-preserving map of fp32 to uint32 (larger float -> larger integer).
// 0 is below every encoded value and marks "no score".
__device__ __forceinline__ uint32_t ord_f32(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__host__ __device__ __forceinline__ float unord_f32(uint32_t o) {
  if (o == 0u) return -INFINITY;
  uint32_t u = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float f;
  __builtin_memcpy(&f, &u, 4);
  return f;
#endif
}

// ------------------------------------------------------------ host launchers

// encode.cu
msa_status launch_encode(const msa_encode_args& a, cudaStream_t st);
msa_status launch_bank_norms(const uint16_t* kbar_r, int64_t n_chunks, int hr, float eps,
                             float* inv_norm, cudaStream_t st);

// Routing plan shared by the scoring kernels: the query rows of one call,
// their sequences, and the workspace pieces.
struct RoutePlan {
  const uint16_t* qr;          // [T, hr, d]
  const float* kr_inv_norm;    // [C, hr]
  const int32_t* chunk_doc;    // [C]
  const uint16_t* kbar_r;      // [C, hr, d]
  int64_t n_chunks, n_docs;
  int32_t hr, n_rows, n_seq;
  int32_t q_seq_off[kMaxSeq + 1];
  float* invq;                 // ws [T, hr]: 1 / (hr * max(||q||, eps))
  float* invq_t;               // ws [hr, Tp]: the same, head-major (Tp = T rounded up to 4)
  int32_t* col_code;           // ws [T]: row's sequence | 256 if the row ends its sequence
  int32_t n_rows_pad;          // Tp
  uint32_t* doc_key;           // ws [S, D]: ordered doc scores (0 = none)
  void* zero;                  // ws bytes to clear before scoring (doc keys, top-k state)
  size_t zero_bytes;           // multiple of 16
};

// score.cu
msa_status launch_qprep(const RoutePlan& p, float eps, cudaStream_t st);
msa_status launch_score_simt(const RoutePlan& p, cudaStream_t st);
// score_tc.cu
msa_status launch_score_tc(const RoutePlan& p, cudaStream_t st);
bool score_tc_supported(const RoutePlan& p);
bool score_tc_built();
int tc_error_take();  // 1 if a tensor-core kernel's bounded wait ran out since the last call
// wait_probe.cu: a bounded wait that runs out (failure-path test)
msa_status launch_wait_probe(cudaStream_t st);
int probe_error_take();
// score_pf.cu: the many-row (prefill) tensor-core scorer
msa_status launch_score_pf(const RoutePlan& p, cudaStream_t st);
bool score_pf_supported(const RoutePlan& p);
int pf_error_take();

// route_backward.cu
msa_status launch_route_backward(const msa_bank_layer& b, const uint16_t* qr, const int32_t* q_seq_off, int n_seq,
                                 float eps, const int32_t* pair_seq, const int32_t* pair_doc,
                                 const float* pair_dscore, int n_pairs, float* dqr, float* dkr,
                                 int64_t* argmax_chunk, int32_t* argmax_row, cudaStream_t st);

// topk.cu
size_t topk_workspace(int n_seq, int64_t n_docs, int k);
msa_status launch_topk(const uint32_t* doc_key, int n_seq, int64_t n_docs, int k,
                       int32_t* top_ids, float* top_scores, float* all_scores, void* ws,
                       cudaStream_t st);

msa_status launch_topk_merge(const int32_t* ids, const float* scores, const int64_t* id_offset, int n_shards,
                             int n_seq, int k, int k_out, int32_t* top_ids, float* top_scores, cudaStream_t st);

// gather.cu
msa_status launch_gather_index(const int64_t* doc_chunk_off, int64_t n_docs, const int32_t* top_ids, int n_seq,
                               int k, int64_t* sel_off, int64_t* sel_chunk, int64_t cap, cudaStream_t st);
msa_status launch_gather_pull(const msa_bank_layer& b, const int64_t* sel_off,
                              const int64_t* sel_chunk, int64_t cap, uint16_t* stage_k,
                              uint16_t* stage_v, cudaStream_t st);

// attend.cu
size_t attend_workspace(const msa_attend_args& a, int* n_splits_out);
msa_status launch_attend(const msa_attend_args& a, void* ws, cudaStream_t st);
size_t attend_backward_workspace(const msa_attend_args& a);
msa_status launch_attend_backward(const msa_attend_args& a, const float* dout, float* dq, float* dk_loc,
                                  float* dv_loc, float* dmem_k, float* dmem_v, void* ws, cudaStream_t st);

}  // namespace msa
