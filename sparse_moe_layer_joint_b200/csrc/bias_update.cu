// bias_update.cu -- the aux-loss-free balancing controller ("Inkling,
// Dissected" §02e): b_i <- b_i + gamma * sign(Lbar - L_i), Lbar = k*T/n_routed.
// The sign is decided in 64-bit integers as sign(k*T - n_routed*L_i), so the
// rounding of Lbar never enters, and the add is a single fp32 add of
// gamma * (+1, 0 or -1), which is exact before rounding.
//
// load_stats -- the balance of one batch from the same loads (§02d, §02g):
// the largest load and the assignments past the experts' capacity, and from
// them MaxVio and the drop rate.
//
// capacity_for -- the capacity of §02d/§02g ("1.25x the ideal load"):
// floor(factor * k*T / n_routed), the factor given as an exact fraction.
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
__global__ void load_stats_kernel(const int32_t* __restrict__ counts, int n_routed, long long kT, int capacity,
                                  int32_t* __restrict__ stats, float* __restrict__ metrics) {
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
    if (metrics != nullptr) {
      // MaxVio = max_i L_i / Lbar - 1 with Lbar = k*T / n_routed; drop rate = dropped / (k*T).
      // Both quotients are formed in fp64 from the exact integers and rounded once to fp32.
      metrics[0] = kT > 0 ? (float)((double)mx * (double)n_routed / (double)kT - 1.0) : 0.0f;
      metrics[1] = kT > 0 ? (float)((double)dr / (double)kT) : 0.0f;
    }
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

extern "C" int moe_load_stats(const int32_t* counts, int n_routed, int T, int top_k, int capacity, int32_t* stats,
                              float* metrics, void* stream) {
  if (!counts || !stats || n_routed < 1 || n_routed > MOE_MAX_ROUTED || capacity < 0 || T < 0 || top_k < 1)
    return MOE_ERR_INVALID_ARG;
  if (!moe::aligned4(counts) || !moe::aligned4(stats) || (metrics && !moe::aligned4(metrics)))
    return MOE_ERR_INVALID_ARG;
  moe::load_stats_kernel<<<1, 256, 0, (cudaStream_t)stream>>>(counts, n_routed, (long long)top_k * T, capacity, stats,
                                                              metrics);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" long long moe_capacity_for(long long factor_num, long long factor_den, int T, int top_k, int n_routed) {
  if (factor_num < 0 || factor_den < 1 || T < 0 || top_k < 1 || n_routed < 1) return MOE_ERR_INVALID_ARG;
  // floor(factor * k*T / n_routed) in exact integer arithmetic (128-bit: no intermediate can overflow)
  const unsigned __int128 num = (unsigned __int128)factor_num * (unsigned __int128)top_k * (unsigned __int128)T;
  const unsigned __int128 den = (unsigned __int128)factor_den * (unsigned __int128)n_routed;
  const unsigned __int128 c = num / den;
  return c > (unsigned __int128)0x7fffffff ? (long long)0x7fffffff : (long long)c;
}
