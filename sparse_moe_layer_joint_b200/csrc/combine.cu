// combine.cu -- the gate-weighted sum back in token order ("Inkling,
// Dissected" §02: the output is the weighted sum of the 8 contributors'
// outputs; §02b sketch: out += g_k * e_k(x)).  A gather-reduce, no scatter:
// one warp per token reads its k routed rows (through token_row) and its
// n_shared shared rows with 16-byte loads, accumulates in fp32 with the
// token's gates, and writes the bf16 row once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"
#include "moe_internal.h"

namespace moe {
namespace comb {

constexpr int THREADS = 256;
constexpr int MAXC = MOE_MAX_TOP_K + MOE_MAX_SHARED;

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& v, float g) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    a[2 * i] = fmaf(g, f.x, a[2 * i]);
    a[2 * i + 1] = fmaf(g, f.y, a[2 * i + 1]);
  }
}

__global__ void __launch_bounds__(THREADS) combine_kernel(const uint4* __restrict__ y_perm,
                                                          const int32_t* __restrict__ token_row,
                                                          const float* __restrict__ gates,
                                                          const uint4* __restrict__ y_shared, int T, int d_vec, int k,
                                                          int n_shared, int n_rows, uint4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int G = k + n_shared;
  for (int t = blockIdx.x * (THREADS / 32) + (threadIdx.x >> 5); t < T; t += gridDim.x * (THREADS / 32)) {
    // lane j < G holds contributor j's source row pointer and gate
    float g = 0.0f;
    const uint4* src = nullptr;
    if (lane < G) {
      g = gates[(size_t)t * G + lane];
      if (lane < k) {
        int r = token_row[(size_t)t * k + lane];
        if (r >= 0 && r < n_rows) src = y_perm + (size_t)r * d_vec;
        else g = 0.0f;
      } else {
        src = y_shared + ((size_t)(lane - k) * T + t) * d_vec;
      }
    }
    float gg[MAXC];
    const uint4* ss[MAXC];
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
      gg[j] = __shfl_sync(0xffffffffu, g, j);
      ss[j] = reinterpret_cast<const uint4*>(__shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(src), j));
    }
    for (int v = lane; v < d_vec; v += 32) {
      float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      uint4 buf[MAXC];
#pragma unroll
      for (int j = 0; j < MAXC; ++j)
        if (j < G && ss[j] != nullptr) buf[j] = __ldg(ss[j] + v);
#pragma unroll
      for (int j = 0; j < MAXC; ++j)
        if (j < G && ss[j] != nullptr) acc_bf16x8(a, buf[j], gg[j]);
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * i], a[2 * i + 1]);
        ow[i] = *reinterpret_cast<uint32_t*>(&h);
      }
      out[(size_t)t * d_vec + v] = o;
    }
  }
}

}  // namespace comb
}  // namespace moe

using namespace moe;

extern "C" int moe_combine(const moe_bf16* y_perm, const int32_t* token_row, const float* gates,
                           const moe_bf16* y_shared, int T, int d, int top_k, int n_shared, moe_bf16* out,
                           void* stream) {
  using namespace moe::comb;
  if (T < 0 || d <= 0 || top_k < 1 || top_k > MOE_MAX_TOP_K || n_shared < 0 || n_shared > MOE_MAX_SHARED)
    return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!y_perm || !token_row || !gates || !out || (n_shared > 0 && !y_shared)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(y_perm) || !aligned16(y_shared) || !aligned16(out) || !aligned4(token_row) || !aligned4(gates))
    return MOE_ERR_INVALID_ARG;
  if ((long long)T * top_k > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;
  const int warps_per_cta = THREADS / 32;
  long long need = (T + warps_per_cta - 1) / warps_per_cta;
  int grid = (int)(need < (long long)sms * 16 ? need : (long long)sms * 16);
  combine_kernel<<<grid, THREADS, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint4*>(y_perm), token_row, gates, reinterpret_cast<const uint4*>(y_shared), T, d / 8,
      top_k, n_shared, T * top_k, reinterpret_cast<uint4*>(out));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
