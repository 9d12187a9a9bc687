// combine.cu -- the gate-weighted sum back in token order ("Inkling,
// Dissected" §02: the output is the weighted sum of the 8 contributors'
// outputs; §02b sketch: out += g_k * e_k(x)).  A gather-reduce, no scatter:
// the work is split into (token, 32-vector slice) units, one warp per unit;
// each lane reads the unit's 16-byte vector from each of the token's k routed
// rows (through token_row) and n_shared shared rows, accumulates in fp32 with
// the token's gates in contributor order, and writes one bf16 vector.  The
// contributor count is a template parameter so the per-lane buffers stay in
// registers and several CTAs fit per SM (more bytes in flight).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"
#include "moe_internal.h"

namespace moe {
namespace comb {

constexpr int THREADS = 256;

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& v, float g) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    a[2 * i] = fmaf(g, f.x, a[2 * i]);
    a[2 * i + 1] = fmaf(g, f.y, a[2 * i + 1]);
  }
}

template <int G>
__global__ void __launch_bounds__(THREADS, 4) combine_kernel(const uint4* __restrict__ y_perm,
                                                             const int32_t* __restrict__ token_row,
                                                             const float* __restrict__ gates,
                                                             const uint4* __restrict__ y_shared, int T, int d_vec,
                                                             int k, int n_rows, uint4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int n_slices = (d_vec + 31) / 32;
  const long long units = (long long)T * n_slices;
  for (long long u = (long long)blockIdx.x * (THREADS / 32) + (threadIdx.x >> 5); u < units;
       u += (long long)gridDim.x * (THREADS / 32)) {
    const int t = (int)(u / n_slices);
    const int v = (int)(u - (long long)t * n_slices) * 32 + lane;
    // lane j < G holds contributor j's row index and gate
    float g = 0.0f;
    long long src = -1;
    if (lane < G) {
      g = __ldg(gates + (size_t)t * G + lane);
      if (lane < k) {
        const int r = __ldg(token_row + (size_t)t * k + lane);
        src = (r >= 0 && r < n_rows) ? (long long)r : -1;
      } else {
        src = (long long)(lane - k) * T + t;  // row of y_shared
      }
    }
    float gg[G];
    long long ss[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      gg[j] = __shfl_sync(0xffffffffu, g, j);
      ss[j] = __shfl_sync(0xffffffffu, src, j);
    }
    if (v >= d_vec) continue;
    uint4 buf[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      const uint4* base = j < k ? y_perm : y_shared;
      buf[j] = ss[j] >= 0 ? __ldg(base + (size_t)ss[j] * d_vec + v) : make_uint4(0, 0, 0, 0);
    }
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < G; ++j) acc_bf16x8(a, buf[j], ss[j] >= 0 ? gg[j] : 0.0f);
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

template <int G>
int launch_g(const moe_bf16* y_perm, const int32_t* token_row, const float* gates, const moe_bf16* y_shared, int T,
             int d, int k, moe_bf16* out, int sms, cudaStream_t s) {
  const int d_vec = d / 8;
  const long long units = (long long)T * ((d_vec + 31) / 32);
  const long long want = (units + THREADS / 32 - 1) / (THREADS / 32);
  const int grid = (int)(want < (long long)sms * 16 ? want : (long long)sms * 16);
  combine_kernel<G><<<grid, THREADS, 0, s>>>(reinterpret_cast<const uint4*>(y_perm), token_row, gates,
                                             reinterpret_cast<const uint4*>(y_shared), T, d_vec, k, T * k,
                                             reinterpret_cast<uint4*>(out));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
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
  cudaStream_t s = (cudaStream_t)stream;
  switch (top_k + n_shared) {
#define MOE_COMBINE_CASE(G) \
  case G:                   \
    return launch_g<G>(y_perm, token_row, gates, y_shared, T, d, top_k, out, sms, s);
    MOE_COMBINE_CASE(1) MOE_COMBINE_CASE(2) MOE_COMBINE_CASE(3) MOE_COMBINE_CASE(4)
    MOE_COMBINE_CASE(5) MOE_COMBINE_CASE(6) MOE_COMBINE_CASE(7) MOE_COMBINE_CASE(8)
    MOE_COMBINE_CASE(9) MOE_COMBINE_CASE(10) MOE_COMBINE_CASE(11) MOE_COMBINE_CASE(12)
    MOE_COMBINE_CASE(13) MOE_COMBINE_CASE(14) MOE_COMBINE_CASE(15) MOE_COMBINE_CASE(16)
#undef MOE_COMBINE_CASE
    default: return MOE_ERR_UNSUPPORTED;
  }
}
