// ep.cu -- expert parallelism over peer memory ("Inkling, Dissected" §02d:
// the experts live on different GPUs, each token's rows travel to the GPUs of
// its experts and come back; the pages call this the all-to-all schedule).
//
// Rank q of W owns the routed experts [q*E/W, (q+1)*E/W).  Every rank keeps a
// receive buffer of rows in its own HBM, grouped by its experts and, within an
// expert, by source rank, so the owner runs ONE grouped GEMM over everything it
// received.  Given the per-expert counts of every rank (an all-gather of
// W x E int32), a source rank knows where each of its rows lands:
//
//   send_base[e] = sum over e' of e's owner with e' < e of sum_s cnt[s][e']
//                + sum_{s < rank} cnt[s][e]
//   destination of the p-th row of expert e on this rank = send_base[e] + p
//
// and the owner's group offsets are the same sums restricted to its experts.
// Dispatch writes each routed row straight into the owner's buffer (16-byte
// stores through a peer pointer: over NVLink when the owner is another GPU);
// the combine gathers each token's outputs back from the owners' buffers (peer
// loads) in the same contributor order and fp32 arithmetic as the one-GPU
// combine, so one rank gives bit-identical results to it.  Ordering between
// ranks (rows landed before the owner's GEMM, outputs written before the
// combine) is the caller's: a collective or barrier between the calls.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "moe.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace ep {

constexpr int THREADS = 256;

// One CTA: thread e sums expert e's counts over the ranks; the owner-segment
// prefixes are plain loops over at most 256 entries (a few microseconds once a step).
__global__ void __launch_bounds__(THREADS) plan_kernel(const int32_t* __restrict__ cnt, int rank, int world,
                                                        int n_routed, int32_t* __restrict__ send_base,
                                                        int32_t* __restrict__ recv_offsets) {
  __shared__ int tot[MOE_MAX_ROUTED];
  const int e = threadIdx.x;
  const int e_loc = n_routed / world;
  int pre = 0;
  if (e < n_routed) {
    int t = 0;
    for (int s = 0; s < world; ++s) {
      const int c = cnt[(size_t)s * n_routed + e];
      t += c;
      if (s < rank) pre += c;
    }
    tot[e] = t;
  }
  __syncthreads();
  if (e < n_routed) {
    const int seg = (e / e_loc) * e_loc;  // the first expert of e's owner
    int excl = 0;
    for (int i = seg; i < e; ++i) excl += tot[i];
    send_base[e] = excl + pre;
  }
  for (int el = e; el <= e_loc; el += THREADS) {  // e_loc + 1 offsets: one more than the experts
    int off = 0;
    for (int i = 0; i < el; ++i) off += tot[rank * e_loc + i];
    recv_offsets[el] = off;
  }
}

// One warp per routed (token, slot) row: copy x[t] to its place in the owner's receive buffer.
__global__ void __launch_bounds__(THREADS) dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ topk,
                                                            const int32_t* __restrict__ token_row,
                                                            const int32_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ send_base, int T, int d_vec,
                                                            int n_routed, int k, int e_loc,
                                                            uint4* const* __restrict__ recv, long long recv_rows,
                                                            unsigned int* status) {
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)T * k;
  const long long warps = (long long)gridDim.x * (THREADS / 32);
  for (long long rid = (long long)blockIdx.x * (THREADS / 32) + (threadIdx.x >> 5); rid < rows; rid += warps) {
    const int e = __ldg(topk + rid);
    const int r = __ldg(token_row + rid);
    if (e < 0 || e >= n_routed) {
      if (lane == 0) set_status(status, MOE_STATUS_BAD_EXPERT);
      continue;
    }
    if (r < 0) continue;  // an assignment that was not served
    const long long pos = (long long)r - __ldg(offsets + e);
    const long long dst_row = (long long)__ldg(send_base + e) + pos;
    if (pos < 0 || dst_row < 0 || dst_row >= recv_rows) {
      if (lane == 0) set_status(status, MOE_STATUS_RECV_OVERFLOW);
      continue;
    }
    const uint4* src = x + (rid / k) * d_vec;
    uint4* dst = recv[e / e_loc] + dst_row * d_vec;
    for (int v = lane; v < d_vec; v += 32) dst[v] = __ldg(src + v);
  }
  __threadfence_system();  // the stores reach the owner before this kernel counts as done
}

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& v, float g) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    a[2 * i] = fmaf(g, f.x, a[2 * i]);
    a[2 * i + 1] = fmaf(g, f.y, a[2 * i + 1]);
  }
}

// One warp per (token, 32-vector slice): lane j < G resolves contributor j's row (routed: in its
// owner's output buffer; shared: y_shared), then every lane sums its vector over the contributors
// in order, in fp32, with the token's gates.
template <int G>
__global__ void __launch_bounds__(THREADS, 4)
    combine_kernel(const uint4* const* __restrict__ recv_y, const int32_t* __restrict__ topk,
                   const int32_t* __restrict__ token_row, const int32_t* __restrict__ offsets,
                   const int32_t* __restrict__ send_base, const float* __restrict__ gates,
                   const uint4* __restrict__ y_shared, int T, int d_vec, int n_routed, int k, int e_loc,
                   long long recv_rows, uint4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int n_slices = (d_vec + 31) / 32;
  const long long units = (long long)T * n_slices;
  for (long long u = (long long)blockIdx.x * (THREADS / 32) + (threadIdx.x >> 5); u < units;
       u += (long long)gridDim.x * (THREADS / 32)) {
    const int t = (int)(u / n_slices);
    const int v = (int)(u - (long long)t * n_slices) * 32 + lane;
    float g = 0.0f;
    const uint4* src = nullptr;
    if (lane < G) {
      g = __ldg(gates + (size_t)t * G + lane);
      if (lane < k) {
        const int e = __ldg(topk + (size_t)t * k + lane);
        const int r = __ldg(token_row + (size_t)t * k + lane);
        if (e >= 0 && e < n_routed && r >= 0) {
          const long long dst_row = (long long)__ldg(send_base + e) + ((long long)r - __ldg(offsets + e));
          if (dst_row >= 0 && dst_row < recv_rows) src = recv_y[e / e_loc] + dst_row * d_vec;
        }
      } else {
        src = y_shared + ((size_t)(lane - k) * T + t) * d_vec;
      }
    }
    const uint4* ss[G];
    float gg[G];
#pragma unroll
    for (int j = 0; j < G; ++j) {
      gg[j] = __shfl_sync(0xffffffffu, g, j);
      ss[j] = reinterpret_cast<const uint4*>(
          __shfl_sync(0xffffffffu, (unsigned long long)reinterpret_cast<uintptr_t>(src), j));
    }
    if (v >= d_vec) continue;
    uint4 buf[G];
#pragma unroll
    for (int j = 0; j < G; ++j) buf[j] = ss[j] != nullptr ? ss[j][v] : make_uint4(0, 0, 0, 0);
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < G; ++j) acc_bf16x8(a, buf[j], ss[j] != nullptr ? gg[j] : 0.0f);
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
int launch_combine(const moe_bf16* const* recv_y, const int32_t* topk, const int32_t* token_row,
                   const int32_t* offsets, const int32_t* send_base, const float* gates, const moe_bf16* y_shared,
                   int T, int d, int n_routed, int k, int e_loc, long long recv_rows, moe_bf16* out, int sms,
                   cudaStream_t s) {
  const int d_vec = d / 8;
  const long long units = (long long)T * ((d_vec + 31) / 32);
  const long long want = (units + THREADS / 32 - 1) / (THREADS / 32);
  const int grid = (int)(want < (long long)sms * 16 ? want : (long long)sms * 16);
  combine_kernel<G><<<grid, THREADS, 0, s>>>(reinterpret_cast<const uint4* const*>(recv_y), topk, token_row, offsets,
                                             send_base, gates, reinterpret_cast<const uint4*>(y_shared), T, d_vec,
                                             n_routed, k, e_loc, recv_rows, reinterpret_cast<uint4*>(out));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

bool valid_split(int n_routed, int world, int rank) {
  return world >= 1 && world <= MOE_EP_MAX_WORLD && rank >= 0 && rank < world && n_routed >= 1 &&
         n_routed <= MOE_MAX_ROUTED && n_routed % world == 0;
}

}  // namespace ep
}  // namespace moe

using namespace moe;

extern "C" int moe_ep_plan(const int32_t* counts_all, int rank, int world, int n_routed, int32_t* send_base,
                           int32_t* recv_offsets, void* stream) {
  if (!ep::valid_split(n_routed, world, rank)) return MOE_ERR_INVALID_ARG;
  if (!counts_all || !send_base || !recv_offsets) return MOE_ERR_INVALID_ARG;
  if (!aligned4(counts_all) || !aligned4(send_base) || !aligned4(recv_offsets)) return MOE_ERR_INVALID_ARG;
  ep::plan_kernel<<<1, ep::THREADS, 0, (cudaStream_t)stream>>>(counts_all, rank, world, n_routed, send_base,
                                                               recv_offsets);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_ep_dispatch(const moe_bf16* x, const int32_t* topk_idx, const int32_t* token_row,
                               const int32_t* offsets, const int32_t* send_base, int T, int d, int n_routed,
                               int top_k, int world, moe_bf16* const* recv_x, long long recv_rows, void* stream) {
  if (!ep::valid_split(n_routed, world, 0) || T < 0 || d <= 0 || top_k < 1 || top_k > MOE_MAX_TOP_K ||
      recv_rows < 0)
    return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!x || !topk_idx || !token_row || !offsets || !send_base || !recv_x) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned4(topk_idx) || !aligned4(token_row) || !aligned4(offsets) || !aligned4(send_base) ||
      (reinterpret_cast<uintptr_t>(recv_x) & 7u) != 0)
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;
  unsigned int* status = status_ptr();
  if (!status) return MOE_ERR_CUDA;
  const long long rows = (long long)T * top_k;
  const long long want = (rows + ep::THREADS / 32 - 1) / (ep::THREADS / 32);
  const int grid = (int)(want < (long long)sms * 8 ? want : (long long)sms * 8);
  ep::dispatch_kernel<<<grid, ep::THREADS, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint4*>(x), topk_idx, token_row, offsets, send_base, T, d / 8, n_routed, top_k,
      n_routed / world, reinterpret_cast<uint4* const*>(recv_x), recv_rows, status);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_ep_combine(const moe_bf16* const* recv_y, const int32_t* topk_idx, const int32_t* token_row,
                              const int32_t* offsets, const int32_t* send_base, const float* gates,
                              const moe_bf16* y_shared, int T, int d, int n_routed, int top_k, int n_shared,
                              int world, long long recv_rows, moe_bf16* out, void* stream) {
  if (!ep::valid_split(n_routed, world, 0) || T < 0 || d <= 0 || top_k < 1 || top_k > MOE_MAX_TOP_K ||
      n_shared < 0 || n_shared > MOE_MAX_SHARED || recv_rows < 0)
    return MOE_ERR_INVALID_ARG;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;
  if (!recv_y || !topk_idx || !token_row || !offsets || !send_base || !gates || !out || (n_shared > 0 && !y_shared))
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(recv_y) & 7u) != 0 || !aligned4(topk_idx) || !aligned4(token_row) ||
      !aligned4(offsets) || !aligned4(send_base) || !aligned4(gates) || !aligned16(y_shared) || !aligned16(out))
    return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  const int e_loc = n_routed / world;
  switch (top_k + n_shared) {
#define MOE_EP_COMBINE_CASE(G)                                                                                     \
  case G:                                                                                                          \
    return ep::launch_combine<G>(recv_y, topk_idx, token_row, offsets, send_base, gates, y_shared, T, d, n_routed, \
                                 top_k, e_loc, recv_rows, out, sms, s);
    MOE_EP_COMBINE_CASE(1) MOE_EP_COMBINE_CASE(2) MOE_EP_COMBINE_CASE(3) MOE_EP_COMBINE_CASE(4)
    MOE_EP_COMBINE_CASE(5) MOE_EP_COMBINE_CASE(6) MOE_EP_COMBINE_CASE(7) MOE_EP_COMBINE_CASE(8)
    MOE_EP_COMBINE_CASE(9) MOE_EP_COMBINE_CASE(10) MOE_EP_COMBINE_CASE(11) MOE_EP_COMBINE_CASE(12)
    MOE_EP_COMBINE_CASE(13) MOE_EP_COMBINE_CASE(14) MOE_EP_COMBINE_CASE(15) MOE_EP_COMBINE_CASE(16)
#undef MOE_EP_COMBINE_CASE
    default: return MOE_ERR_UNSUPPORTED;
  }
}

namespace moe {
namespace ep {

// cuMemGetAddressRange through the runtime's driver entry point: the allocation that holds a pointer
// (an IPC handle names a whole allocation; the pointer's offset in it travels beside the handle).
typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
    tried = true;
  }
  return fn;
}

int allocation_base(const void* ptr, uintptr_t* base) {
  AddressRangeFn fn = address_range_fn();
  if (!fn) return MOE_ERR_CUDA;
  CUdeviceptr b = 0;
  size_t size = 0;
  if (fn(&b, &size, (CUdeviceptr)reinterpret_cast<uintptr_t>(ptr)) != CUDA_SUCCESS) return MOE_ERR_CUDA;
  *base = (uintptr_t)b;
  return MOE_OK;
}

}  // namespace ep
}  // namespace moe

extern "C" int moe_ipc_handle_bytes(void) { return (int)sizeof(cudaIpcMemHandle_t); }

extern "C" int moe_ipc_get_handle(const void* dev_ptr, void* handle, unsigned long long* offset) {
  if (!dev_ptr || !handle || !offset) return MOE_ERR_INVALID_ARG;
  uintptr_t base = 0;
  int rc = ep::allocation_base(dev_ptr, &base);
  if (rc != MOE_OK) return rc;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return MOE_ERR_CUDA;
  memcpy(handle, &h, sizeof(h));
  *offset = (unsigned long long)(reinterpret_cast<uintptr_t>(dev_ptr) - base);
  return MOE_OK;
}

extern "C" int moe_ipc_open(const void* handle, unsigned long long offset, void** dev_ptr) {
  if (!handle || !dev_ptr) return MOE_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* base = nullptr;
  if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return MOE_ERR_CUDA;
  *dev_ptr = static_cast<char*>(base) + offset;
  return MOE_OK;
}

extern "C" int moe_ipc_close(void* dev_ptr) {
  if (!dev_ptr) return MOE_ERR_INVALID_ARG;
  uintptr_t base = 0;
  int rc = ep::allocation_base(dev_ptr, &base);
  if (rc != MOE_OK) return rc;
  return cudaIpcCloseMemHandle(reinterpret_cast<void*>(base)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
