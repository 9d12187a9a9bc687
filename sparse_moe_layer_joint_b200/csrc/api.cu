// api.cu -- library-wide pieces of libmoe: the device status word, status
// strings, the wait limit, TMA descriptor encoding (through the driver entry
// point, so the library does not link libcuda), and the bounded-wait test hook.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <unordered_map>

#include "moe.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

__device__ unsigned int g_status = 0;

std::atomic<uint64_t> g_timeout_ns{2000000000ull};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

std::mutex g_mu;
int g_sms[64] = {0};
unsigned int* g_status_ptr[64] = {nullptr};

}  // namespace

uint64_t wait_timeout_ns() { return g_timeout_ns.load(); }

unsigned int* status_ptr() {
  int dev;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<unsigned int*>(p);
  }
  return g_status_ptr[dev];
}

int device_info(int* dev, int* sms) {
  if (cudaGetDevice(dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (*dev < 0 || *dev >= 64) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sms[*dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess || v <= 0)
      return MOE_ERR_CUDA;
    g_sms[*dev] = v;
  }
  *sms = g_sms[*dev];
  return MOE_OK;
}

int ensure_smem_attr(const void* kernel, size_t bytes) {
  int dev;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  static std::mutex mu;
  // (kernel, device) -> the limit set so far; a kernel whose shared memory depends on its
  // arguments raises it again when a call needs more
  static std::unordered_map<const void*, std::unordered_map<int, size_t>> done;
  std::lock_guard<std::mutex> lk(mu);
  size_t& have = done[kernel][dev];
  if (have >= bytes) return MOE_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
    return MOE_ERR_CUDA;
  have = bytes;
  return MOE_OK;
}

namespace {

// Encoded descriptors are pure functions of (base, shape, box); repeated calls
// on the same buffers (every layer step) reuse them instead of re-encoding.
struct TmapKey {
  const void* base;
  int rank;
  int elem_bytes;  // 2: bf16, 1: bytes (packed FP4 pairs)
  uint64_t dim0, dim1, dim2;
  uint32_t box0, box1;
  bool swizzle;  // 128-byte swizzle (else none)
  bool operator==(const TmapKey& o) const {
    return base == o.base && rank == o.rank && elem_bytes == o.elem_bytes && dim0 == o.dim0 && dim1 == o.dim1 &&
           dim2 == o.dim2 && box0 == o.box0 && box1 == o.box1 && swizzle == o.swizzle;
  }
};

constexpr int kTmapCacheSize = 64;
struct TmapEntry {
  bool used = false;
  TmapKey key;
  CUtensorMap map;
};
TmapEntry g_tmap_cache[kTmapCacheSize];
int g_tmap_next = 0;
std::mutex g_tmap_mu;

}  // namespace

static int encode_tmap(CUtensorMap* map, const void* base, int elem_bytes, int rank, uint64_t dim0, uint64_t dim1,
                       uint64_t dim2, uint32_t box0, uint32_t box1, bool swizzle = true) {
  const TmapKey key{base, rank, elem_bytes, dim0, dim1, rank == 3 ? dim2 : 1, box0, box1, swizzle};
  {
    std::lock_guard<std::mutex> lk(g_tmap_mu);
    for (int i = 0; i < kTmapCacheSize; ++i) {
      if (g_tmap_cache[i].used && g_tmap_cache[i].key == key) {
        *map = g_tmap_cache[i].map;
        return MOE_OK;
      }
    }
  }
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  cuuint64_t dims[3] = {dim0, dim1, dim2};
  cuuint64_t strides[2] = {dim0 * elem_bytes, dim0 * dim1 * elem_bytes};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  memset(map, 0, sizeof(*map));
  CUresult r = fn(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, (cuuint32_t)rank, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_tmap_mu);
  TmapEntry& e = g_tmap_cache[g_tmap_next];
  g_tmap_next = (g_tmap_next + 1) % kTmapCacheSize;
  e.used = true;
  e.key = key;
  e.map = *map;
  return MOE_OK;
}

int encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                     uint32_t box0, uint32_t box1) {
  return encode_tmap(map, base, 2, rank, dim0, dim1, dim2, box0, box1);
}

int encode_tmap_u8(CUtensorMap* map, const void* base, int rank, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                   uint32_t box0, uint32_t box1) {
  return encode_tmap(map, base, 1, rank, dim0, dim1, dim2, box0, box1);
}

int encode_tmap_u8_plain(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint32_t box0,
                         uint32_t box1) {
  return encode_tmap(map, base, 1, 2, dim0, dim1, 1, box0, box1, false);
}

namespace {

// One thread waits on a barrier that expects two arrivals but gets one.
__global__ void bounded_wait_kernel(uint64_t timeout_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 2);
    abort_flag = 0;
    fence_barrier_init();
    mbar_arrive(&bar);
    mbar_wait(&bar, 0, timeout_ns, &abort_flag, status);
  }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" const char* moe_status_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, bad size or top_k)";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_TIMEOUT: return "a device-side wait ran out of time";
    case MOE_ERR_DEVICE: return "device-side error (bad expert index or inconsistent counts)";
    case MOE_ERR_SCRATCH: return "scratch buffer too small";
    default: return "unknown status";
  }
}

extern "C" int moe_get_status(void* stream, int* device_status) {
  if (!device_status) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(v), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  *device_status = (int)v;
  if (v & MOE_STATUS_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (v) return MOE_ERR_DEVICE;
  return MOE_OK;
}

extern "C" int moe_set_wait_timeout_ns(uint64_t ns) {
  if (ns == 0) return MOE_ERR_INVALID_ARG;
  g_timeout_ns.store(ns);
  return MOE_OK;
}

extern "C" int moe_debug_bounded_wait(uint64_t timeout_ns, void* stream) {
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
  unsigned int* st = status_ptr();
  if (!st) return MOE_ERR_CUDA;
  bounded_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(timeout_ns, st);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
