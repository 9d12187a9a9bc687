// Device (CUDA) build of the seeded input generator: fills caller-owned device
// buffers with exactly the values the host build produces (same gen_core.h,
// __d*_rn intrinsics in place of operators so no FMA contraction can occur).
#include <cuda_runtime.h>
#include <stdint.h>

#include "gen_core.h"

namespace {

constexpr int kThreads = 256;

inline unsigned grid_for(uint64_t n) {
  uint64_t g = (n + kThreads - 1) / kThreads;
  return (unsigned)(g > 148u * 64u ? 148u * 64u : (g == 0 ? 1 : g));
}

__global__ void k_normal_bf16(uint16_t* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                              double stddev) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x) {
    float f = __double2float_rn(__dmul_rn(mi_normal(seed, stream, offset + i), stddev));
    dst[i] = mi_f32_to_bf16_bits(f);
  }
}

__global__ void k_normal_f32(float* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                             double stddev) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    dst[i] = __double2float_rn(__dmul_rn(mi_normal(seed, stream, offset + i), stddev));
}

__global__ void k_uniform_f32(float* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                              double lo, double hi) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x)
    dst[i] = __double2float_rn(mi_uniform(seed, stream, offset + i, lo, hi));
}

__global__ void k_words(uint32_t* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n;
       i += (uint64_t)gridDim.x * blockDim.x) {
    uint64_t g = offset + i;
    dst[i] = mi_block(seed, stream, g >> 2).v[g & 3u];
  }
}

inline int finish() { return cudaGetLastError() == cudaSuccess ? 0 : -1; }

}  // namespace

extern "C" {

int mi_gpu_normal_bf16(void* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                       double stddev, void* cuda_stream) {
  if (n == 0) return 0;
  if (!dst) return -2;
  k_normal_bf16<<<grid_for(n), kThreads, 0, (cudaStream_t)cuda_stream>>>((uint16_t*)dst, n, seed, stream,
                                                                         offset, stddev);
  return finish();
}

int mi_gpu_normal_f32(void* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                      double stddev, void* cuda_stream) {
  if (n == 0) return 0;
  if (!dst) return -2;
  k_normal_f32<<<grid_for(n), kThreads, 0, (cudaStream_t)cuda_stream>>>((float*)dst, n, seed, stream, offset,
                                                                        stddev);
  return finish();
}

int mi_gpu_uniform_f32(void* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset, double lo,
                       double hi, void* cuda_stream) {
  if (n == 0) return 0;
  if (!dst) return -2;
  k_uniform_f32<<<grid_for(n), kThreads, 0, (cudaStream_t)cuda_stream>>>((float*)dst, n, seed, stream, offset,
                                                                         lo, hi);
  return finish();
}

int mi_gpu_words_u32(void* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                     void* cuda_stream) {
  if (n == 0) return 0;
  if (!dst) return -2;
  k_words<<<grid_for(n), kThreads, 0, (cudaStream_t)cuda_stream>>>((uint32_t*)dst, n, seed, stream, offset);
  return finish();
}

}  // extern "C"
