// permute.cu -- dispatch: group the T*k (token, slot) pairs by expert, rows of
// one expert in increasing token order ("Inkling, Dissected" §02: each token
// goes to exactly its k routed experts; §02d: tokens queue per expert).
//
// Four launches (two when every token fits one chunk: one_chunk_kernel does 1-3),
// all deterministic (no atomics decide a position):
//   1. chunk_hist   one CTA per 256-token chunk: hist[c][e] = picks of e in chunk c
//   2. chunk_scan   one CTA: offsets[e] = exclusive scan over experts of the
//                   rows each expert serves, min(picks, capacity);
//                   base[c][e] = picks of e in chunks before c; optional check
//                   of the caller's counts
//   3. rank         one CTA per chunk: each warp takes 32 tokens; a per-warp
//                   bitmask per expert (bit = lane) gives each pick its rank
//                   among earlier lanes, a prefix over the 8 warps its rank
//                   among earlier warps.  A pick whose rank in its expert's
//                   queue (token order) reaches the capacity is dropped
//                   (§02d: overflow tokens get nothing from that expert):
//                   token_row = -1 and no row; otherwise row offsets[e] + rank
//                   -> token_row, row_token
//   4. copy_rows    grid-wide over (token, 256-vector slice) units: each x
//                   slice is read once with 16-byte loads and written to the
//                   token's k rows.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include "moe.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace perm {

constexpr int CHUNK = 256;  // tokens per chunk (8 warps x 32)
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;

__global__ void __launch_bounds__(THREADS) chunk_hist_kernel(const int32_t* __restrict__ topk_idx, int T, int k,
                                                             int n_routed, int32_t* __restrict__ hist,
                                                             unsigned int* status) {
  __shared__ int h[MOE_MAX_ROUTED];
  for (int e = threadIdx.x; e < MOE_MAX_ROUTED; e += THREADS) h[e] = 0;
  __syncthreads();
  const int c = blockIdx.x;
  const int t0 = c * CHUNK;
  const int n = min(CHUNK, T - t0) * k;
  const int32_t* src = topk_idx + (size_t)t0 * k;
  bool bad = false;
  for (int i = threadIdx.x; i < n; i += THREADS) {
    int e = src[i];
    if (e >= 0 && e < n_routed)
      atomicAdd(&h[e], 1);
    else
      bad = true;
  }
  if (bad) set_status(status, MOE_STATUS_BAD_EXPERT);
  __syncthreads();
  for (int e = threadIdx.x; e < n_routed; e += THREADS) hist[(size_t)c * n_routed + e] = h[e];
}

// One CTA of 256 threads; thread e owns expert e.
__global__ void __launch_bounds__(THREADS) chunk_scan_kernel(const int32_t* __restrict__ hist, int n_chunks,
                                                             int n_routed, int capacity,
                                                             const int32_t* __restrict__ counts,
                                                             int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ base, unsigned int* status) {
  __shared__ int warp_sum[WARPS];
  const int e = threadIdx.x;
  int total = 0;
  if (e < n_routed) {
    for (int c = 0; c < n_chunks; ++c) total += hist[(size_t)c * n_routed + e];
    if (counts != nullptr && counts[e] != total) set_status(status, MOE_STATUS_COUNT_MISMATCH);
  }
  const int served = total < capacity ? total : capacity;
  // exclusive scan of the served rows over experts
  const int lane = e & 31, w = e >> 5;
  int v = served;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_sum[w] = v;
  __syncthreads();
  int before = 0;
  for (int i = 0; i < w; ++i) before += warp_sum[i];
  const int excl = before + v - served;
  if (e < n_routed) offsets[e] = excl;
  if (e == n_routed - 1) offsets[n_routed] = excl + served;
  if (e < n_routed) {
    int run = 0;
    for (int c = 0; c < n_chunks; ++c) {
      base[(size_t)c * n_routed + e] = run;
      run += hist[(size_t)c * n_routed + e];
    }
  }
}

__global__ void __launch_bounds__(THREADS) rank_kernel(const int32_t* __restrict__ topk_idx,
                                                       const int32_t* __restrict__ base,
                                                       const int32_t* __restrict__ offsets, int T, int k,
                                                       int n_routed, int capacity, int32_t* __restrict__ row_token,
                                                       int32_t* __restrict__ token_row) {
  __shared__ uint32_t mask[WARPS][MOE_MAX_ROUTED];
  __shared__ int pre[WARPS][MOE_MAX_ROUTED];
  __shared__ int off[MOE_MAX_ROUTED];
  const int c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < WARPS * MOE_MAX_ROUTED; i += THREADS) (&mask[0][0])[i] = 0u;
  __syncthreads();
  const int t = c * CHUNK + warp * 32 + lane;
  const bool valid = t < T;
  int ex[MOE_MAX_TOP_K];
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOP_K; ++j) {
    ex[j] = -1;
    if (j < k && valid) {
      int e = topk_idx[(size_t)t * k + j];
      if (e >= 0 && e < n_routed) {
        ex[j] = e;
        atomicOr(&mask[warp][e], 1u << lane);
      }
    }
  }
  __syncthreads();
  // prefix over warps, per expert
  for (int e = threadIdx.x; e < n_routed; e += THREADS) {
    off[e] = offsets[e];
    int run = base[(size_t)c * n_routed + e];
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      pre[w][e] = run;
      run += __popc(mask[w][e]);
    }
  }
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOP_K; ++j) {
    if (ex[j] >= 0) {
      const int rank = pre[warp][ex[j]] + __popc(mask[warp][ex[j]] & lt);  // place in the expert's queue
      const int pos = rank < capacity ? off[ex[j]] + rank : -1;
      token_row[(size_t)t * k + j] = pos;
      if (pos >= 0) row_token[pos] = t;
    } else if (j < k && valid) {
      token_row[(size_t)t * k + j] = -1;
    }
  }
}

// Launches 1-3 in one CTA when all tokens fit one chunk (T <= 256): the histogram is the popcount of the
// rank masks, the scan runs over the experts, and the ranks follow with a base of zero, so every output
// equals the three launches' bit for bit.
__global__ void __launch_bounds__(THREADS) one_chunk_kernel(const int32_t* __restrict__ topk_idx, int T, int k,
                                                            int n_routed, int capacity,
                                                            const int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ row_token,
                                                            int32_t* __restrict__ token_row, unsigned int* status) {
  __shared__ uint32_t mask[WARPS][MOE_MAX_ROUTED];
  __shared__ int pre[WARPS][MOE_MAX_ROUTED];
  __shared__ int off[MOE_MAX_ROUTED];
  __shared__ int warp_sum[WARPS];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < WARPS * MOE_MAX_ROUTED; i += THREADS) (&mask[0][0])[i] = 0u;
  __syncthreads();
  const int t = threadIdx.x;  // one token per thread
  const bool valid = t < T;
  int ex[MOE_MAX_TOP_K];
  bool bad = false;
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOP_K; ++j) {
    ex[j] = -1;
    if (j < k && valid) {
      const int e = topk_idx[(size_t)t * k + j];
      if (e >= 0 && e < n_routed) {
        ex[j] = e;
        atomicOr(&mask[warp][e], 1u << lane);
      } else {
        bad = true;
      }
    }
  }
  if (bad) set_status(status, MOE_STATUS_BAD_EXPERT);
  __syncthreads();
  // thread e owns expert e: its picks per warp, in token order, and its served rows
  const int e = threadIdx.x;
  int total = 0;
  if (e < n_routed) {
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
      pre[w][e] = total;
      total += __popc(mask[w][e]);
    }
    if (counts != nullptr && counts[e] != total) set_status(status, MOE_STATUS_COUNT_MISMATCH);
  }
  const int served = total < capacity ? total : capacity;
  int v = served;  // exclusive scan of the served rows over experts
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_sum[warp] = v;
  __syncthreads();
  int before = 0;
  for (int i = 0; i < warp; ++i) before += warp_sum[i];
  const int excl = before + v - served;
  if (e < n_routed) {
    offsets[e] = excl;
    off[e] = excl;
  }
  if (e == n_routed - 1) offsets[n_routed] = excl + served;
  __syncthreads();
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < MOE_MAX_TOP_K; ++j) {
    if (ex[j] >= 0) {
      const int rank = pre[warp][ex[j]] + __popc(mask[warp][ex[j]] & lt);  // place in the expert's queue
      const int pos = rank < capacity ? off[ex[j]] + rank : -1;
      token_row[(size_t)t * k + j] = pos;
      if (pos >= 0) row_token[pos] = t;
    } else if (j < k && valid) {
      token_row[(size_t)t * k + j] = -1;
    }
  }
}

// Launches 1-3 in one CTA where a single chunk holds every token; MOE_PERMUTE_ONE_CHUNK=0 keeps three.
static bool one_chunk_for(int n_chunks) {
  const char* env = getenv("MOE_PERMUTE_ONE_CHUNK");
  if (env && env[0] == '0' && env[1] == '\0') return false;
  return n_chunks == 1;
}

// x_perm[token_row[t][j]] = x[t] for every slot j: a block copies one token at a time; each thread
// loads up to COPY_VPT of the row's 16-byte vectors (v, v + THREADS, ...) before writing each of them k
// times, so several loads are in flight per thread.
constexpr int COPY_VPT = 4;

__global__ void __launch_bounds__(THREADS) copy_rows_kernel(const uint4* __restrict__ x,
                                                            const int32_t* __restrict__ token_row, int T, int d_vec,
                                                            int k, int n_rows, uint4* __restrict__ x_perm) {
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    int rows[MOE_MAX_TOP_K];
#pragma unroll
    for (int j = 0; j < MOE_MAX_TOP_K; ++j) rows[j] = j < k ? __ldg(token_row + (size_t)t * k + j) : -1;
    const uint4* src = x + (size_t)t * d_vec;
    for (int v0 = threadIdx.x; v0 < d_vec; v0 += THREADS * COPY_VPT) {
      uint4 val[COPY_VPT];
#pragma unroll
      for (int i = 0; i < COPY_VPT; ++i)
        if (v0 + i * THREADS < d_vec) val[i] = __ldg(src + v0 + i * THREADS);
#pragma unroll
      for (int j = 0; j < MOE_MAX_TOP_K; ++j) {
        const int r = rows[j];
        if (r < 0 || r >= n_rows) continue;
        uint4* dst = x_perm + (size_t)r * d_vec + v0;
#pragma unroll
        for (int i = 0; i < COPY_VPT; ++i)
          if (v0 + i * THREADS < d_vec) dst[i * THREADS] = val[i];
      }
    }
  }
}

// The launches shared by moe_permute, moe_permute_capped and moe_permute_noalloc.
static int launch_permute(const moe_bf16* x, const int32_t* topk_idx, const int32_t* counts, int T, int d,
                          int n_routed, int top_k, int capacity, int32_t* offsets, moe_bf16* x_perm,
                          int32_t* row_token, int32_t* token_row, void* scratch, cudaStream_t s) {
  unsigned int* status = status_ptr();
  if (!status) return MOE_ERR_CUDA;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;
  const int n_chunks = (T + CHUNK - 1) / CHUNK;
  if (one_chunk_for(n_chunks)) {
    one_chunk_kernel<<<1, THREADS, 0, s>>>(topk_idx, T, top_k, n_routed, capacity, counts, offsets, row_token,
                                            token_row, status);
  } else {
    int32_t* hist = reinterpret_cast<int32_t*>(scratch);
    int32_t* base = hist + (size_t)n_chunks * n_routed;
    chunk_hist_kernel<<<n_chunks, THREADS, 0, s>>>(topk_idx, T, top_k, n_routed, hist, status);
    chunk_scan_kernel<<<1, THREADS, 0, s>>>(hist, n_chunks, n_routed, capacity, counts, offsets, base, status);
    rank_kernel<<<n_chunks, THREADS, 0, s>>>(topk_idx, base, offsets, T, top_k, n_routed, capacity, row_token,
                                             token_row);
  }
  if (x_perm == nullptr) return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;  // indices only
  const int d_vec = d / 8;
  const int grid = (int)((long long)T < (long long)sms * 8 ? T : (long long)sms * 8);  // one token per block at a time
  copy_rows_kernel<<<grid, THREADS, 0, s>>>(reinterpret_cast<const uint4*>(x), token_row, T, d_vec, top_k,
                                            T * top_k, reinterpret_cast<uint4*>(x_perm));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace perm
}  // namespace moe

using namespace moe;

extern "C" size_t moe_permute_scratch_bytes(int T, int n_routed) {
  if (T <= 0 || n_routed <= 0) return 256;
  size_t n_chunks = ((size_t)T + perm::CHUNK - 1) / perm::CHUNK;
  return 2 * n_chunks * (size_t)n_routed * sizeof(int32_t) + 256;
}

static int permute_entry(const moe_bf16* x, const int32_t* topk_idx, const int32_t* counts, int T, int d,
                         int n_routed, int top_k, int capacity, int32_t* offsets, moe_bf16* x_perm,
                         int32_t* row_token, int32_t* token_row, void* scratch, size_t scratch_bytes,
                         void* stream) {
  using namespace moe::perm;
  if (T < 0 || d <= 0 || n_routed < 1 || top_k < 1 || capacity < 0) return MOE_ERR_INVALID_ARG;
  if (top_k > MOE_MAX_TOP_K || top_k > n_routed || n_routed > MOE_MAX_ROUTED) return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!topk_idx || !offsets || !row_token || !token_row || !scratch || (x_perm && !x)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm) || !aligned4(topk_idx) || !aligned4(counts) || !aligned4(offsets) ||
      !aligned4(row_token) || !aligned4(token_row) || !aligned16(scratch))
    return MOE_ERR_INVALID_ARG;
  if ((long long)T * top_k > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (scratch_bytes < moe_permute_scratch_bytes(T, n_routed)) return MOE_ERR_SCRATCH;
  cudaStream_t s = (cudaStream_t)stream;
  if (T == 0) {
    if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (n_routed + 1), s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  return launch_permute(x, topk_idx, counts, T, d, n_routed, top_k, capacity, offsets, x_perm, row_token,
                        token_row, scratch, s);
}

extern "C" int moe_permute(const moe_bf16* x, const int32_t* topk_idx, const int32_t* counts, int T, int d,
                           int n_routed, int top_k, int32_t* offsets, moe_bf16* x_perm, int32_t* row_token,
                           int32_t* token_row, void* scratch, size_t scratch_bytes, void* stream) {
  return permute_entry(x, topk_idx, counts, T, d, n_routed, top_k, 0x7fffffff, offsets, x_perm, row_token,
                       token_row, scratch, scratch_bytes, stream);
}

extern "C" int moe_permute_capped(const moe_bf16* x, const int32_t* topk_idx, const int32_t* counts, int T, int d,
                                  int n_routed, int top_k, int capacity, int32_t* offsets, moe_bf16* x_perm,
                                  int32_t* row_token, int32_t* token_row, void* scratch, size_t scratch_bytes,
                                  void* stream) {
  return permute_entry(x, topk_idx, counts, T, d, n_routed, top_k, capacity, offsets, x_perm, row_token,
                       token_row, scratch, scratch_bytes, stream);
}

// ---------------------------------------------------------------------------
// moe_permute_noalloc: the same three launches, with the scratch held in this
// file's device array instead of a caller buffer (for callers that cannot
// allocate device memory).  The array's host-side name is not a device
// address: its address is fetched once per device with cudaGetSymbolAddress,
// with that device current, and passed to the kernels.
// ---------------------------------------------------------------------------
#include <mutex>

namespace moe {
namespace perm {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES];

static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[64] = {nullptr};

// Device address of this device's copy of the array (set up on first use).
static int noalloc_scratch(void** out) {
  int dev;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace perm
}  // namespace moe

extern "C" int moe_permute_noalloc(const moe_bf16* x, const int32_t* topk_idx, const int32_t* counts, int T, int d,
                                   int n_routed, int top_k, int32_t* offsets, moe_bf16* x_perm, int32_t* row_token,
                                   int32_t* token_row, void* stream) {
  using namespace moe::perm;
  if (T < 0 || d <= 0 || n_routed < 1 || top_k < 1) return MOE_ERR_INVALID_ARG;
  if (top_k > MOE_MAX_TOP_K || top_k > n_routed || n_routed > MOE_MAX_ROUTED) return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!topk_idx || !offsets || !row_token || !token_row || (x_perm && !x)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm) || !aligned4(topk_idx) || !aligned4(counts) || !aligned4(offsets) ||
      !aligned4(row_token) || !aligned4(token_row))
    return MOE_ERR_INVALID_ARG;
  if ((long long)T * top_k > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (moe_permute_scratch_bytes(T, n_routed) > (size_t)MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES) return MOE_ERR_SCRATCH;
  void* scratch = nullptr;
  int rc = noalloc_scratch(&scratch);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  if (T == 0) {
    if (cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (n_routed + 1), s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  // Every part of the scratch that is read is written first in the same call
  // (hist by chunk_hist, base by chunk_scan), so nothing needs clearing.
  return launch_permute(x, topk_idx, counts, T, d, n_routed, top_k, 0x7fffffff, offsets, x_perm, row_token,
                        token_row, scratch, s);
}
