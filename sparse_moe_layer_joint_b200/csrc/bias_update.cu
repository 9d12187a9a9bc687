// bias_update.cu -- the aux-loss-free balancing controller ("Inkling,
// Dissected" §02e): b_i <- b_i + gamma * sign(Lbar - L_i), Lbar = k*T/n_routed.
// The sign is decided in 64-bit integers as sign(k*T - n_routed*L_i), so the
// rounding of Lbar never enters, and the add is a single fp32 add of
// gamma * (+1, 0 or -1), which is exact before rounding.
//
// load_stats -- the balance of one batch from the same loads (§02d, §02g):
// the largest load and the assignments past the experts' capacity.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"
#include "moe_internal.h"

namespace moe {
namespace {

__global__ void bias_update_kernel(const int32_t* __restrict__ counts, int n_routed, long long kT, float gamma,
                                   float* __restrict__ bias) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_routed) return;
  long long diff = kT - (long long)n_routed * (long long)counts[i];
  float sgn = diff > 0 ? 1.0f : (diff < 0 ? -1.0f : 0.0f);
  bias[i] = __fadd_rn(bias[i], __fmul_rn(gamma, sgn));
}

// One CTA of 256 threads; thread i owns expert i (n_routed <= 256).
__global__ void load_stats_kernel(const int32_t* __restrict__ counts, int n_routed, int capacity,
                                  int32_t* __restrict__ stats) {
  __shared__ int wmax[8], wdrop[8];
  const int i = threadIdx.x;
  const int L = i < n_routed ? counts[i] : 0;
  int mx = L;
  int dr = L > capacity ? L - capacity : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    dr += __shfl_xor_sync(0xffffffffu, dr, o);
  }
  if ((i & 31) == 0) {
    wmax[i >> 5] = mx;
    wdrop[i >> 5] = dr;
  }
  __syncthreads();
  if (i == 0) {
    for (int w = 1; w < 8; ++w) {
      mx = max(mx, wmax[w]);
      dr += wdrop[w];
    }
    stats[0] = mx;
    stats[1] = dr;
  }
}

}  // namespace
}  // namespace moe

extern "C" int moe_bias_update(const int32_t* counts, int n_routed, int T, int top_k, float gamma, float* bias,
                               void* stream) {
  if (!counts || !bias || n_routed < 1 || n_routed > MOE_MAX_ROUTED || T < 0 || top_k < 1) return MOE_ERR_INVALID_ARG;
  if (!moe::aligned4(counts) || !moe::aligned4(bias)) return MOE_ERR_INVALID_ARG;
  if (!(gamma == gamma)) return MOE_ERR_INVALID_ARG;  // NaN
  moe::bias_update_kernel<<<1, 256, 0, (cudaStream_t)stream>>>(counts, n_routed, (long long)top_k * T, gamma, bias);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_load_stats(const int32_t* counts, int n_routed, int capacity, int32_t* stats, void* stream) {
  if (!counts || !stats || n_routed < 1 || n_routed > MOE_MAX_ROUTED || capacity < 0) return MOE_ERR_INVALID_ARG;
  if (!moe::aligned4(counts) || !moe::aligned4(stats)) return MOE_ERR_INVALID_ARG;
  moe::load_stats_kernel<<<1, 256, 0, (cudaStream_t)stream>>>(counts, n_routed, capacity, stats);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
