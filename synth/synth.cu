// Seeded synthetic inputs for the tests and the benchmark.
//
// This module holds no arithmetic of the method itself. It turns
// (seed, tensor id, element index) into a value, identically on the host and on
// the GPU, so that a multi-gigabyte tensor can be generated in HBM and any
// slice of it regenerated on the host for the CPU oracle without a copy.
//
// Generator: SplitMix64 (Steele, Lea and Flood, "Fast Splittable Pseudorandom
// Number Generators", OOPSLA 2014), used counter-style: draw i of a stream with
// key K is mix64(K + (i + 1) * golden_gamma), which is exactly the i-th output
// of a SplitMix64 generator started at state K.
//
// Approximate N(0,1): Irwin-Hall sum of the four 16-bit lanes of one draw,
// centred and divided by its standard deviation sqrt(4 * (2^32 - 1) / 12).
// Every step is integer arithmetic or one IEEE fp32 multiply (no contraction),
// followed by round-to-nearest-even to bfloat16 done on the bit pattern, so the
// host and the device produce bit-identical tensors.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;
// 1 / sqrt((2^32 - 1) / 3), rounded to fp32.
#define SYNTH_INV_STD 0x1.bb67aep-16f

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__host__ __device__ __forceinline__ uint64_t stream_key(uint64_t seed, uint64_t tensor_id) {
  return mix64(seed * kGamma + tensor_id + 1ULL);
}

__host__ __device__ __forceinline__ uint64_t draw(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1ULL) * kGamma);
}

__host__ __device__ __forceinline__ int32_t irwin_hall_centred(uint64_t r) {
  int32_t s = (int32_t)(r & 0xFFFF) + (int32_t)((r >> 16) & 0xFFFF) +
              (int32_t)((r >> 32) & 0xFFFF) + (int32_t)((r >> 48) & 0xFFFF);
  return s - 131070;  // 2 * 65535
}

__host__ __device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
  uint32_t u;
#ifdef __CUDA_ARCH__
  u = __float_as_uint(f);
#else
  std::memcpy(&u, &f, 4);
#endif
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;  // NaN
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

__device__ __forceinline__ uint16_t normal_bf16_dev(uint64_t key, uint64_t i, float sigma) {
  float z = __fmul_rn((float)irwin_hall_centred(draw(key, i)), SYNTH_INV_STD);
  return f32_to_bf16_bits(__fmul_rn(z, sigma));
}

inline uint16_t normal_bf16_host(uint64_t key, uint64_t i, float sigma) {
  // Two separate fp32 multiplies; built with -ffp-contract=off and SSE math.
  float z = (float)irwin_hall_centred(draw(key, i)) * SYNTH_INV_STD;
  return f32_to_bf16_bits(z * sigma);
}

__global__ void fill_normal_kernel(uint16_t* __restrict__ out, int64_t n, uint64_t key,
                                   int64_t index0, float sigma) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += stride)
    out[j] = normal_bf16_dev(key, (uint64_t)(index0 + j), sigma);
}

}  // namespace

extern "C" {

// Fills out[0..n) with draws index0..index0+n-1 of stream (seed, tensor_id),
// as bfloat16 bit patterns of sigma * N(0,1). Host memory. Returns 0.
int synth_normal_bf16_host(uint16_t* out, int64_t n, uint64_t seed, uint64_t tensor_id,
                           int64_t index0, float sigma) {
  uint64_t key = stream_key(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = normal_bf16_host(key, (uint64_t)(index0 + j), sigma);
  return 0;
}

// Same values as synth_normal_bf16_host, written to device memory on the given
// stream (a cudaStream_t passed as void*). Returns the cudaError_t of the launch.
int synth_normal_bf16_device(uint16_t* out, int64_t n, uint64_t seed, uint64_t tensor_id,
                             int64_t index0, float sigma, void* stream) {
  if (n <= 0) return 0;
  uint64_t key = stream_key(seed, tensor_id);
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  fill_normal_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(out, n, key, index0, sigma);
  return (int)cudaGetLastError();
}

// Raw 64-bit draws index0..index0+n-1 of stream (seed, tensor_id). Host memory.
int synth_u64_host(uint64_t* out, int64_t n, uint64_t seed, uint64_t tensor_id, int64_t index0) {
  uint64_t key = stream_key(seed, tensor_id);
  for (int64_t j = 0; j < n; ++j) out[j] = draw(key, (uint64_t)(index0 + j));
  return 0;
}

}  // extern "C"
