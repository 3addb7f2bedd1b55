// msa_route_static: routing with library-owned scratch, for callers that
// cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc on their hot path: a serving
// process whose framework reserves the whole of HBM for its own pool and
// forbids other allocations, or a latency-critical loop that cannot accept
// cudaMalloc's implicit device-wide synchronisation and unbounded latency.
// This entry point takes the same inputs and outputs as msa_route but no
// workspace: its scratch is the file-scope device array below, a fixed
// MSA_ROUTE_STATIC_SCRATCH_BYTES (4 MiB, msa.h) that every GPU which loads the
// library reserves until the process exits.
//
// In host code `g_route_static_scratch` only names a host-side stand-in, not a
// device address; the device address is looked up once per device with
// cudaGetSymbolAddress and passed to the kernels.
#include <mutex>

#include "msa_internal.cuh"

namespace {

constexpr size_t kRouteStaticScratchBytes = MSA_ROUTE_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_route_static_scratch[kRouteStaticScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of this device's scratch array (set up on first use).
msa_status scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return msa::cuda_fail(e, "route_static: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return msa::fail(MSA_ERR_UNSUPPORTED, "route_static: device %d", dev);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_static_scratch);
    if (e != cudaSuccess) return msa::cuda_fail(e, "route_static: cudaGetSymbolAddress of the scratch array");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MSA_OK;
}

}  // namespace

extern "C" {

msa_status msa_route_static(const msa_bank_layer* bank, const uint16_t* qr, const int32_t* q_seq_off,
                            int32_t n_seq, int32_t n_rows, int32_t top_k, float eps, int32_t* top_ids,
                            float* top_scores, float* all_doc_scores, void* stream) {
  size_t need = 0;
  msa_status s = msa_route_workspace(bank, n_seq, n_rows, top_k, &need);
  if (s != MSA_OK) return s;
  if (need > kRouteStaticScratchBytes)
    return msa::fail(MSA_ERR_CAPACITY,
                     "route_static: this call needs %zu B of scratch; the library's static scratch holds %zu B "
                     "(use msa_route with a caller-provided workspace)",
                     need, kRouteStaticScratchBytes);
  void* scratch = nullptr;
  s = scratch_for_current_device(&scratch);
  if (s != MSA_OK) return s;
  return msa_route(bank, qr, q_seq_off, n_seq, n_rows, top_k, eps, top_ids, top_scores, all_doc_scores, scratch,
                   kRouteStaticScratchBytes, stream);
}

}  // extern "C"
