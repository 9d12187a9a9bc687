// moe_internal.h -- host-side helpers shared by the libmoe entry points.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Current device and its SM count (cached per device).
int device_info(int* dev, int* sms);

// Raise a kernel's dynamic shared-memory limit once per device.
int ensure_smem_attr(const void* kernel, size_t bytes);

// Encode a tiled TMA descriptor for a row-major bf16 tensor of rank 2 or 3
// (dims innermost first), box {box0, box1[, 1]}, 128-byte swizzle, zero fill
// out of bounds.
int encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                     uint32_t box0, uint32_t box1);

// The same for a byte tensor (dims and box in bytes; packed FP4 pairs).
int encode_tmap_u8(CUtensorMap* map, const void* base, int rank, uint64_t dim0, uint64_t dim1, uint64_t dim2,
                   uint32_t box0, uint32_t box1);

// A rank-2 byte tensor without swizzle (boxes land in shared memory as they lie in global memory:
// FP4 scale-factor atoms).
int encode_tmap_u8_plain(CUtensorMap* map, const void* base, uint64_t dim0, uint64_t dim1, uint32_t box0,
                         uint32_t box1);

// Limit on device-side waits for kernels launched from now on.
uint64_t wait_timeout_ns();

// Device address of the current device's status word (nullptr on failure).
unsigned int* status_ptr();

}  // namespace moe
