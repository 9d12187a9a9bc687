// Host (CPU) build of the seeded input generator: fills caller-owned host
// buffers, split over std::thread workers.  Compiled with -ffp-contract=off so
// that every double operation in gen_core.h is a separately rounded IEEE op.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <thread>
#include <vector>

#include "gen_core.h"

namespace {

template <class F>
void parallel_for(uint64_t n, int nthreads, F f) {
  if (nthreads <= 0) nthreads = (int)std::max(1u, std::thread::hardware_concurrency());
  uint64_t min_chunk = 1u << 16;
  uint64_t want = (n + min_chunk - 1) / min_chunk;
  if ((uint64_t)nthreads > want) nthreads = (int)std::max<uint64_t>(1, want);
  if (nthreads == 1) {
    f((uint64_t)0, n);
    return;
  }
  std::vector<std::thread> ts;
  uint64_t chunk = (n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    uint64_t b = (uint64_t)t * chunk, e = std::min(n, b + chunk);
    if (b >= e) break;
    ts.emplace_back([=] { f(b, e); });
  }
  for (auto& t : ts) t.join();
}

}  // namespace

extern "C" {

void mi_host_philox_block(uint64_t seed, uint32_t stream, uint64_t block, uint32_t* out4) {
  mi_u32x4 r = mi_block(seed, stream, block);
  memcpy(out4, r.v, sizeof(r.v));
}

void mi_host_philox_raw(const uint32_t* ctr4, const uint32_t* key2, uint32_t* out4) {
  mi_u32x4 c;
  memcpy(c.v, ctr4, sizeof(c.v));
  mi_u32x4 r = mi_philox4x32_10(c, key2[0], key2[1]);
  memcpy(out4, r.v, sizeof(r.v));
}

void mi_host_words_u32(uint32_t* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                       int nthreads) {
  parallel_for(n, nthreads, [&](uint64_t b, uint64_t e) {
    for (uint64_t i = b; i < e; ++i) {
      uint64_t g = offset + i;
      dst[i] = mi_block(seed, stream, g >> 2).v[g & 3u];
    }
  });
}

void mi_host_normal_f64(double* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                        int nthreads) {
  parallel_for(n, nthreads, [&](uint64_t b, uint64_t e) {
    for (uint64_t i = b; i < e; ++i) dst[i] = mi_normal(seed, stream, offset + i);
  });
}

void mi_host_normal_bf16(uint16_t* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                         double stddev, int nthreads) {
  parallel_for(n, nthreads, [&](uint64_t b, uint64_t e) {
    for (uint64_t i = b; i < e; ++i) {
      float f = (float)MI_MUL(mi_normal(seed, stream, offset + i), stddev);
      dst[i] = mi_f32_to_bf16_bits(f);
    }
  });
}

void mi_host_normal_f32(float* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                        double stddev, int nthreads) {
  parallel_for(n, nthreads, [&](uint64_t b, uint64_t e) {
    for (uint64_t i = b; i < e; ++i) dst[i] = (float)MI_MUL(mi_normal(seed, stream, offset + i), stddev);
  });
}

void mi_host_uniform_f32(float* dst, uint64_t n, uint64_t seed, uint32_t stream, uint64_t offset,
                         double lo, double hi, int nthreads) {
  parallel_for(n, nthreads, [&](uint64_t b, uint64_t e) {
    for (uint64_t i = b; i < e; ++i) dst[i] = (float)mi_uniform(seed, stream, offset + i, lo, hi);
  });
}

}  // extern "C"
