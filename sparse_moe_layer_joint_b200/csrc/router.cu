// router.cu -- router GEMM with the routing fused into its epilogue
// ("Inkling, Dissected" §02b: s_i = sigmoid(x . w_i); keep the top 6 by
// s_i + b_i; g_i = s_i / sum over kept U shared; "Under the hood", "The
// routing strategy": 256 routed + 2 shared scores, top-k over routed only).
//
// The logits of all n_routed + n_shared experts for 128 tokens are one
// 128 x 272 fp32 accumulator in TMEM: a tcgen05 MMA with N = 256 (experts
// 0..255) and one with N = 16 (experts 256..271, zero rows past the last
// expert) per 16-deep K step, fed by TMA through a 4-stage ring.
//
// Split-K across a cluster.  When there are few 128-token tiles (decode, mid
// sizes) a cluster of S CTAs (S = 2, 4 or 8) shares one tile: CTA c runs the
// MMAs of the c-th slice of K, then writes its partial 128 x 272 tile into its
// shared memory; after a cluster barrier, CTA c owns rows c*128/S .. of the
// tile and sums their S partials in cluster-rank order through distributed
// shared memory (a fixed order, so the result does not depend on timing).
//
// Routing epilogue: the logit tile is parked in shared memory (the stage ring
// is idle by then).  With a whole tile per CTA each epilogue thread routes one
// token (register top-k list); after a split-K reduction, with 128/S rows per
// CTA, each epilogue warp routes one token at a time (k rounds of a warp-wide
// argmax).  Both keep the lower index on ties, form the joint gates with the
// denominator summed over the contributors in ascending expert index, and
// count the picks in a shared-memory histogram added to the global counts once
// per CTA.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#include "moe.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace router {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B0_ROWS = 256;
constexpr int B1_ROWS = 16;
constexpr int B0_BYTES = B0_ROWS * BK * 2;
constexpr int B1_BYTES = B1_ROWS * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B0_BYTES + B1_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int RED_COLS = B0_ROWS + B1_ROWS;  // 272 logit columns per tile row
constexpr int RED_LD = RED_COLS + 4;         // row stride in shared memory: 16-byte reads of 8 consecutive rows
                                             // (one per thread) fall in distinct bank groups
constexpr int MAX_SPLIT = 8;

struct Params {
  const float* bias;
  const float* offset;  // nullable
  int T, d, n_routed, n_shared;
  int ksplit;           // CTAs (cluster size) sharing one 128-token tile: 1, 2, 4 or 8
  int32_t* topk_idx;
  float* gates;
  float gate_scale;  // the joint weights are multiplied by it (route_scale x global_scale)
  int32_t* counts;
  float* scores;  // nullable
  uint64_t timeout_ns;
  unsigned int* status;
};

struct SmemTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float bias[MOE_MAX_ROUTED];  // read as float4
  alignas(16) float off[MOE_MAX_ROUTED];
  int hist[MOE_MAX_ROUTED];
  float shared_s[BM][MOE_MAX_SHARED];
};

// The stage ring, idle once the MMAs are done, also holds the split-K partial
// tile [128][272] fp32 and the reduced rows [128/S][272] fp32 (S >= 2).
constexpr size_t SPLIT_BYTES = (size_t)BM * RED_LD * 4 + (size_t)(BM / 2) * RED_LD * 4;
constexpr size_t RING_BYTES =
    (size_t)STAGES * STAGE_BYTES > SPLIT_BYTES ? (size_t)STAGES * STAGE_BYTES : SPLIT_BYTES;

constexpr size_t SMEM_BYTES = 1024 + RING_BYTES + sizeof(SmemTail);
static_assert(SMEM_BYTES <= 227 * 1024, "router shared memory");
static_assert(RING_BYTES % 16 == 0 && offsetof(SmemTail, bias) % 16 == 0 && offsetof(SmemTail, off) % 16 == 0,
              "float4 reads of bias / offset need 16-byte alignment");
static_assert((RED_LD * 4) % 16 == 0, "logit rows are read as float4");

__device__ __forceinline__ float sigmoid_f32(float z) { return __frcp_rn(1.0f + __expf(-z)); }

__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// Route one token with one thread.  z: the token's logits in shared memory.
// Scores are computed 32 experts at a time (independent, so their latencies
// overlap); each is then offered to a sorted register top-k list, with a
// single compare against the current k-th value rejecting most of them.
// Scanning experts in index order with a strict '>' keeps the lower index on
// ties.  Then the joint gates (denominator summed over the contributors in
// ascending expert index), the outputs and the pick histogram.
template <int K>
__device__ __forceinline__ void route_token(const Params& p, SmemTail* st, const float* z, int t) {
  const int E = p.n_routed + p.n_shared;
  float* srow = p.scores != nullptr ? p.scores + (size_t)t * E : nullptr;
  float val[K], sc[K];
  int id[K];
#pragma unroll
  for (int q = 0; q < K; ++q) {
    val[q] = -INFINITY;
    sc[q] = 0.0f;
    id[q] = 0x7fffffff;
  }
  for (int c0 = 0; c0 < p.n_routed; c0 += 32) {
    float sv[32], sl[32];
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 z4 = *reinterpret_cast<const float4*>(z + c0 + j);
      const float4 o4 = *reinterpret_cast<const float4*>(st->off + c0 + j);
      const float4 b4 = *reinterpret_cast<const float4*>(st->bias + c0 + j);
      sv[j + 0] = sigmoid_f32(z4.x + o4.x);
      sv[j + 1] = sigmoid_f32(z4.y + o4.y);
      sv[j + 2] = sigmoid_f32(z4.z + o4.z);
      sv[j + 3] = sigmoid_f32(z4.w + o4.w);
      sl[j + 0] = sv[j + 0] + b4.x;
      sl[j + 1] = sv[j + 1] + b4.y;
      sl[j + 2] = sv[j + 2] + b4.z;
      sl[j + 3] = sv[j + 3] + b4.w;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int i = c0 + j;
      if (i < p.n_routed) {
        if (srow) srow[i] = sv[j];
        if (sl[j] > val[K - 1]) {
          val[K - 1] = sl[j];
          sc[K - 1] = sv[j];
          id[K - 1] = i;
#pragma unroll
          for (int q = K - 1; q > 0; --q) {
            if (val[q] > val[q - 1]) {
              float tv = val[q]; val[q] = val[q - 1]; val[q - 1] = tv;
              float ts = sc[q]; sc[q] = sc[q - 1]; sc[q - 1] = ts;
              int ti = id[q]; id[q] = id[q - 1]; id[q - 1] = ti;
            }
          }
        }
      }
    }
  }
  float shv[MOE_MAX_SHARED];
#pragma unroll
  for (int q = 0; q < MOE_MAX_SHARED; ++q) {
    shv[q] = 0.0f;
    if (q < p.n_shared) {
      shv[q] = sigmoid_f32(z[p.n_routed + q]);
      if (srow) srow[p.n_routed + q] = shv[q];
    }
  }
  // the denominator is a sum over the contributor set, in ascending expert index
  float den = 0.0f;
  int prev = -1;
#pragma unroll
  for (int q = 0; q < K; ++q) {
    int best = 0x7fffffff;
    float bs = 0.0f;
#pragma unroll
    for (int r = 0; r < K; ++r)
      if (id[r] > prev && id[r] < best) {
        best = id[r];
        bs = sc[r];
      }
    den += bs;
    prev = best;
  }
#pragma unroll
  for (int q = 0; q < MOE_MAX_SHARED; ++q)
    if (q < p.n_shared) den += shv[q];
  const int G = K + p.n_shared;
  int32_t* ti = p.topk_idx + (size_t)t * K;
  float* gt = p.gates + (size_t)t * G;
#pragma unroll
  for (int q = 0; q < K; ++q) {
    ti[q] = id[q];
    gt[q] = __fmul_rn(__fdiv_rn(sc[q], den), p.gate_scale);
    if (id[q] >= 0 && id[q] < p.n_routed) atomicAdd(&st->hist[id[q]], 1);  // unset only for non-finite scores
  }
#pragma unroll
  for (int q = 0; q < MOE_MAX_SHARED; ++q)
    if (q < p.n_shared) gt[K + q] = __fmul_rn(__fdiv_rn(shv[q], den), p.gate_scale);
}

// Route NT tokens with one warp, their work interleaved so the latencies of the
// NT independent shuffle chains overlap.  z: the first token's logits in shared
// memory (rows ld floats apart); t0: its token index; n_valid <= NT tokens are
// real.  Lane l scores routed experts 8l .. 8l+7 of every token; then k rounds
// of a warp-wide argmax of s + b (a strict '>' scan within a lane, and the
// lower index on equal values across lanes, so ties keep the lower index)
// pick each token's experts in descending order.  Lane n then forms token n's
// joint gates (denominator summed over the contributors in ascending expert
// index) and writes its outputs.
template <int K, int NT, class ST>
__device__ __forceinline__ void route_tokens_warp(const Params& p, ST* st, const float* z, int ld, int t0,
                                                  int n_valid, int lane) {
  const int E = p.n_routed + p.n_shared;
  float s[NT][8], sel[NT][8];
  float4 o4[2], b4[2];
  o4[0] = *reinterpret_cast<const float4*>(st->off + 8 * lane);
  o4[1] = *reinterpret_cast<const float4*>(st->off + 8 * lane + 4);
  b4[0] = *reinterpret_cast<const float4*>(st->bias + 8 * lane);
  b4[1] = *reinterpret_cast<const float4*>(st->bias + 8 * lane + 4);
  const float off[8] = {o4[0].x, o4[0].y, o4[0].z, o4[0].w, o4[1].x, o4[1].y, o4[1].z, o4[1].w};
  const float bia[8] = {b4[0].x, b4[0].y, b4[0].z, b4[0].w, b4[1].x, b4[1].y, b4[1].z, b4[1].w};
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const float4* z4 = reinterpret_cast<const float4*>(z + (size_t)n * ld + 8 * lane);
    const float4 za = z4[0], zb = z4[1];
    const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
    float* srow = (p.scores != nullptr && n < n_valid) ? p.scores + (size_t)(t0 + n) * E : nullptr;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = 8 * lane + j;
      if (i < p.n_routed) {
        s[n][j] = sigmoid_f32(zz[j] + off[j]);
        sel[n][j] = s[n][j] + bia[j];
        if (srow) srow[i] = s[n][j];
      } else {
        s[n][j] = 0.0f;
        sel[n][j] = -INFINITY;
      }
    }
  }
  // shared experts' affinities: lane q < n_shared holds shared expert q of every token
  float sh[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    sh[n] = 0.0f;
    if (lane < p.n_shared) {
      sh[n] = sigmoid_f32(z[(size_t)n * ld + p.n_routed + lane]);
      if (p.scores != nullptr && n < n_valid) p.scores[(size_t)(t0 + n) * E + p.n_routed + lane] = sh[n];
    }
  }
  int id[NT][K];
  float sc[NT][K];
#pragma unroll
  for (int q = 0; q < K; ++q) {
    float bv[NT];
    int bi[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      bv[n] = -INFINITY;
      bi[n] = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (sel[n][j] > bv[n]) {
          bv[n] = sel[n][j];
          bi[n] = 8 * lane + j;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv[n], o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi[n], o);
        if (ov > bv[n] || (ov == bv[n] && oi < bi[n])) {
          bv[n] = ov;
          bi[n] = oi;
        }
      }
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float sw = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (8 * lane + j == bi[n]) {
          sw = s[n][j];
          sel[n][j] = -INFINITY;
        }
      const int owner = (bi[n] >= 0 && bi[n] < 256) ? (bi[n] >> 3) : 0;
      sc[n][q] = __shfl_sync(0xffffffffu, sw, owner);
      id[n][q] = bi[n];
    }
  }
  float shv[NT][MOE_MAX_SHARED];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int q = 0; q < MOE_MAX_SHARED; ++q) shv[n][q] = __shfl_sync(0xffffffffu, sh[n], q);
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    if (lane != n || n >= n_valid) continue;  // lane n finishes token n
    const int t = t0 + n;
    // the denominator is a sum over the contributor set, in ascending expert index
    float den = 0.0f;
    int prev = -1;
#pragma unroll
    for (int q = 0; q < K; ++q) {
      int best = 0x7fffffff;
      float bs = 0.0f;
#pragma unroll
      for (int r = 0; r < K; ++r)
        if (id[n][r] > prev && id[n][r] < best) {
          best = id[n][r];
          bs = sc[n][r];
        }
      den += bs;
      prev = best;
    }
#pragma unroll
    for (int q = 0; q < MOE_MAX_SHARED; ++q)
      if (q < p.n_shared) den += shv[n][q];
    const int G = K + p.n_shared;
    int32_t* ti = p.topk_idx + (size_t)t * K;
    float* gt = p.gates + (size_t)t * G;
#pragma unroll
    for (int q = 0; q < K; ++q) {
      ti[q] = id[n][q];
      gt[q] = __fmul_rn(__fdiv_rn(sc[n][q], den), p.gate_scale);
      if (id[n][q] >= 0 && id[n][q] < p.n_routed) atomicAdd(&st->hist[id[n][q]], 1);  // unset only if non-finite
    }
#pragma unroll
    for (int q = 0; q < MOE_MAX_SHARED; ++q)
      if (q < p.n_shared) gt[K + q] = __fmul_rn(__fdiv_rn(shv[n][q], den), p.gate_scale);
  }
}

template <int K>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    router_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                  const __grid_constant__ CUtensorMap tmB1, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SmemTail* st = reinterpret_cast<SmemTail*>(smem + RING_BYTES);
  auto stageA = [&](int s) { return smem + s * STAGE_BYTES; };
  auto stageB0 = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES; };
  auto stageB1 = [&](int s) { return smem + s * STAGE_BYTES + A_BYTES + B0_BYTES; };
  float* red = reinterpret_cast<float*>(smem);   // [BM][RED_LD] logits (split-K: this CTA's partial)
  float* zsum = red + (size_t)BM * RED_LD;        // [BM/S][RED_LD] reduced rows

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int E = p.n_routed + p.n_shared;
  const bool two = E > B0_ROWS;
  const int S = p.ksplit;
  const uint32_t crank = S > 1 ? cluster_ctarank() : 0u;
  const int m0 = (blockIdx.x / S) * BM;
  const int kb_per = ((p.d + BK - 1) / BK) / S;  // a last partial block is read as zeros past d
  const int kb0 = (int)crank * kb_per;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    mbar_init(&st->tfull, 1);
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    fence_barrier_init();
  }
  for (int i = tid; i < MOE_MAX_ROUTED; i += NUM_THREADS) {
    st->bias[i] = i < p.n_routed ? p.bias[i] : 0.0f;
    st->off[i] = (p.offset != nullptr && i < p.n_routed) ? p.offset[i] : 0.0f;
    st->hist[i] = 0;
  }
  if (warp == 1) tmem_alloc(&st->tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = st->tmem_base;
  volatile int* abort_flag = &st->abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB0);
      if (two) tma_prefetch_desc(&tmB1);
      const uint32_t bytes = (uint32_t)(A_BYTES + B0_BYTES + (two ? B1_BYTES : 0));
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb0 + kb_per; ++kb) {
        if (!mbar_wait(&st->empty[stage], phase ^ 1u, p.timeout_ns, abort_flag, p.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&st->full[stage], bytes);
        tma_load_2d(stageA(stage), &tmA, &st->full[stage], kb * BK, m0);
        tma_load_2d(stageB0(stage), &tmB0, &st->full[stage], kb * BK, 0);
        if (two) tma_load_2d(stageB1(stage), &tmB1, &st->full[stage], kb * BK, B0_ROWS);
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        int zero = 0;
        for (long i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
          mbar_wait(&st->full[i % STAGES], (uint32_t)((i / STAGES) & 1), p.timeout_ns, &zero, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc0 = make_idesc_bf16(BM, B0_ROWS);
      constexpr uint32_t idesc1 = make_idesc_bf16(BM, B1_ROWS);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int kb = 0; kb < kb_per; ++kb) {
        if (!mbar_wait(&st->full[stage], phase, p.timeout_ns, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(stageA(stage));
        const uint32_t b0 = smem_u32(stageB0(stage));
        const uint32_t b1 = smem_u32(stageB1(stage));
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
          mma_bf16_ss(tmem_base, make_desc_sw128(a + k * 32), make_desc_sw128(b0 + k * 32), idesc0, acc);
          if (two)
            mma_bf16_ss(tmem_base + B0_ROWS, make_desc_sw128(a + k * 32), make_desc_sw128(b1 + k * 32), idesc1,
                        acc);
        }
        mma_commit(&st->empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (ok) mma_commit(&st->tfull);
      int zero = 0;
      mma_commit(&st->drain);
      mbar_wait(&st->drain, 0, p.timeout_ns, &zero, p.status);
    }
  } else {
    // ================= epilogue warps: park this CTA's logit tile in shared memory =================
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // this thread's TMEM lane
    const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16);
    if (mbar_wait(&st->tfull, 0, p.timeout_ns, abort_flag, p.status)) {
      tc_fence_after();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the stage ring is idle now
      float* dst = red + (size_t)row * RED_LD;
#pragma unroll 1
      for (int c0 = 0; c0 < B0_ROWS; c0 += 32) {
        float v[32];
        tmem_ld32(taddr + c0, v);
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + c0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
      float v[16];
      if (two) {
        tmem_ld16(taddr + B0_ROWS, v);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.0f;
      }
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4*>(dst + B0_ROWS + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
    }
  }

  if (S == 1) {
    if (warp >= 2) {
      // each thread routes the row it parked (its TMEM lane)
      const int r = (warp & 3) * 32 + lane;
      const int t = m0 + r;
      if (t < p.T) route_token<K>(p, st, red + (size_t)r * RED_LD, t);
    }
  } else {
    tc_fence_before();
    cluster_sync_all();  // every CTA's partial tile is in its shared memory
    if (warp >= 2) {
      const int e = tid - 64;          // 0..127
      const int rows_per = BM / S;     // rows this CTA finishes
      const int r_local = e / S;       // S threads per row
      const int part = e - r_local * S;
      const int row = (int)crank * rows_per + r_local;
      // 1. sum the S partials of this CTA's rows (float4 columns part, part + S, ...), in rank order
      const uint32_t red_local = smem_u32(red + (size_t)row * RED_LD);
      for (int f = part; f < RED_COLS / 4; f += S) {
        float4 q[MAX_SPLIT];
#pragma unroll
        for (int c = 0; c < MAX_SPLIT; ++c)  // all remote loads in flight at once
          if (c < S) q[c] = ld_dsmem_f4(mapa_shared(red_local + f * 16, (uint32_t)c));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int c = 0; c < MAX_SPLIT; ++c) {
          if (c < S) {
            acc.x += q[c].x;
            acc.y += q[c].y;
            acc.z += q[c].z;
            acc.w += q[c].w;
          }
        }
        *reinterpret_cast<float4*>(zsum + (size_t)r_local * RED_LD + 4 * f) = acc;
      }
      named_bar_sync(1, 128);
      // 2. route the rows: with only 128/S of them, 4 tokens per warp pass (all lanes busy)
      const int t_first = m0 + (int)crank * rows_per;
      for (int r = 4 * (warp - 2); r < rows_per; r += 16) {
        const int n_valid = min(4, min(rows_per - r, p.T - (t_first + r)));
        if (n_valid > 0) route_tokens_warp<K, 4>(p, st, zsum + (size_t)r * RED_LD, RED_LD, t_first + r, n_valid, lane);
      }
    }
    cluster_sync_all();  // no CTA leaves while another may still read its partial
  }

  if (warp >= 2) {
    named_bar_sync(1, 128);
    for (int e = tid - 64; e < p.n_routed; e += 128) {
      int c = st->hist[e];
      if (c) atomicAdd(&p.counts[e], c);
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Small batches (T <= SMALL_T_MAX): the tensor-core router's fixed cost (TMEM
// allocation, the TMA pipeline, a 128-row tile for a few tokens) dominates, and
// a few CTAs route every token.  Here the logits are CUDA-core dot products
// spread over many CTAs instead: a cluster of SMALL_CL CTAs takes TB tokens,
// CTA c computes the logits of experts c*EPS .. (c+1)*EPS-1 for them (fp32
// FMAs over 16-byte vectors of x staged in shared memory and of W_r from
// global memory; each lane sums a fixed set of K positions, then a fixed
// shuffle tree, so the result does not depend on timing) and stores them in
// the cluster leader's shared memory; after a cluster barrier the leader routes
// the TB tokens with the warp-level top-k above.
// ---------------------------------------------------------------------------
constexpr int SMALL_T_MAX = 256;
constexpr int SMALL_D_MAX = 2048;  // wider rows: the tensor-core router is faster (measured at d 6144, 7168)
constexpr int SMALL_CL = 8;        // CTAs per cluster: the experts are split into this many slices
constexpr int SMALL_THREADS = 256;
constexpr int SMALL_TB_MAX = 16;
constexpr int SMALL_U = 4;         // experts a warp works on at once
constexpr size_t SMALL_X_BUDGET = 160 * 1024;  // bytes of staged x rows per CTA

struct SmallTail {
  alignas(16) float bias[MOE_MAX_ROUTED];
  alignas(16) float off[MOE_MAX_ROUTED];
  int hist[MOE_MAX_ROUTED];
};

__device__ __forceinline__ void st_dsmem_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Sum TB per-lane partial sums over the warp, scattering the results: at each of
// log2(TB) steps a lane keeps half of its values and adds the partner's copies of
// them (offsets 16, 8, ...), then the last values are summed over the remaining
// lanes.  Lane l ends with the total of token l >> (5 - log2 TB); 2 TB - 1 + ...
// shuffles instead of 5 TB.  The order of the additions is fixed.
template <int TB>
__device__ __forceinline__ float warp_sum_scatter(const float (&acc)[TB], int lane) {
  constexpr int LOG = TB == 1 ? 0 : TB == 2 ? 1 : TB == 4 ? 2 : TB == 8 ? 3 : 4;
  static_assert((1 << LOG) == TB && TB <= 16, "TB: a power of two up to 16");
  float v[TB];
#pragma unroll
  for (int i = 0; i < TB; ++i) v[i] = acc[i];
#pragma unroll
  for (int st = 0; st < LOG; ++st) {
    const int half = TB >> (st + 1);
    const int off = 16 >> st;
    const bool hi = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = hi ? v[i] : v[i + half];
      const float keep = hi ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  float r = v[0];
#pragma unroll
  for (int off = 16 >> LOG; off > 0; off >>= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
  return r;
}

// Dynamic shared memory: x rows [TB][d] bf16, logits [TB][RED_LD] fp32 (the
// leader's are filled by the whole cluster), then the bias / offset / histogram.
template <int TB>
size_t small_smem_bytes(int d) {
  return (size_t)TB * d * 2 + (size_t)TB * RED_LD * 4 + sizeof(SmallTail) + 16;
}

template <int K, int TB>
__global__ void __launch_bounds__(SMALL_THREADS, 1)
    router_small_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
  const int d = p.d;
  uint4* xs = reinterpret_cast<uint4*>(smem);                        // [TB][d/8]
  float* logits = reinterpret_cast<float*>(smem + (size_t)TB * d * 2);  // [TB][RED_LD]
  SmallTail* st = reinterpret_cast<SmallTail*>(smem + (size_t)TB * d * 2 + (size_t)TB * RED_LD * 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t crank = cluster_ctarank();
  const int t0 = (int)(blockIdx.x / SMALL_CL) * TB;
  const int E = p.n_routed + p.n_shared;
  const int eps = (E + SMALL_CL - 1) / SMALL_CL;
  const int e_lo = (int)crank * eps;
  const int e_hi = min(E, e_lo + eps);
  const int nv = d / 8;  // 16-byte vectors per row

  // stage this block's token rows (rows past T are zero) and the routing inputs
  for (int i = tid; i < TB * nv; i += SMALL_THREADS) {
    const int r = i / nv, v = i - r * nv;
    xs[i] = t0 + r < p.T ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + r) * d) + v) : make_uint4(0, 0, 0, 0);
  }
  if (crank == 0) {
    for (int i = tid; i < MOE_MAX_ROUTED; i += SMALL_THREADS) {
      st->bias[i] = i < p.n_routed ? p.bias[i] : 0.0f;
      st->off[i] = (p.offset != nullptr && i < p.n_routed) ? p.offset[i] : 0.0f;
      st->hist[i] = 0;
    }
    for (int i = tid; i < TB * RED_LD; i += SMALL_THREADS) logits[i] = 0.0f;
  }
  __syncthreads();
  cluster_sync_all();  // the leader's logit rows are zeroed before any CTA writes into them

  // logits of this CTA's experts: a warp takes SMALL_U experts at a time (their weight loads in flight
  // together), lane l sums vectors l, l + 32, ... of each
  const uint32_t lead_logits = mapa_shared(smem_u32(logits), 0);
  constexpr int SHIFT = 5 - (TB == 1 ? 0 : TB == 2 ? 1 : TB == 4 ? 2 : TB == 8 ? 3 : 4);
  for (int e0 = e_lo + warp * SMALL_U; e0 < e_hi; e0 += (SMALL_THREADS / 32) * SMALL_U) {
    float acc[SMALL_U][TB];
#pragma unroll
    for (int u = 0; u < SMALL_U; ++u)
#pragma unroll
      for (int t = 0; t < TB; ++t) acc[u][t] = 0.0f;
    for (int v = lane; v < nv; v += 32) {
      float wf[SMALL_U][8];
#pragma unroll
      for (int u = 0; u < SMALL_U; ++u) {
        const int e = min(e0 + u, e_hi - 1);  // past the slice: a valid row, result not stored
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(w + (size_t)e * d) + v), wf[u]);
      }
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        float xf[8];
        bf16x8_to_f32(xs[t * nv + v], xf);
#pragma unroll
        for (int u = 0; u < SMALL_U; ++u)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[u][t] = fmaf(xf[j], wf[u][j], acc[u][t]);
      }
    }
#pragma unroll
    for (int u = 0; u < SMALL_U; ++u) {
      const float v = warp_sum_scatter<TB>(acc[u], lane);
      if (e0 + u < e_hi && (lane & ((1 << SHIFT) - 1)) == 0)
        st_dsmem_f32(lead_logits + (uint32_t)(((lane >> SHIFT) * RED_LD + e0 + u) * 4), v);
    }
  }
  cluster_sync_all();  // every logit of the block is in the leader's shared memory
  if (crank != 0) return;

  // route: warp w takes tokens 2w, 2w + 1 (TB <= 16)
  const int r = 2 * warp;
  const int n_valid = min(2, min(TB - r, p.T - (t0 + r)));
  if (n_valid > 0) route_tokens_warp<K, 2>(p, st, logits + (size_t)r * RED_LD, RED_LD, t0 + r, n_valid, lane);
  __syncthreads();
  for (int e = tid; e < p.n_routed; e += SMALL_THREADS) {
    const int c = st->hist[e];
    if (c) atomicAdd(&p.counts[e], c);
  }
}

// Narrow rows (d <= SINGLE_D_MAX): no cluster at all.  Each CTA takes TB <= 4 tokens and computes
// the logits of every expert itself (W_r is at most 258 x 512 bf16 = 264 KB, read from L2 by every
// CTA), keeps them in its own shared memory and routes its tokens: no cluster barrier, no DSMEM.
constexpr int SINGLE_D_MAX = 512;

// U: experts a warp works on at once.  Each round of a warp is a chain of L2 loads and a butterfly
// reduction, so with narrow rows the latency of the rounds sets the time: more experts a round means fewer
// rounds (the order of every expert's own sum, and so every logit, is the same for any U).
template <int K, int TB, int U = SMALL_U>
__global__ void __launch_bounds__(SMALL_THREADS, 1)
    router_single_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
  const int d = p.d;
  uint4* xs = reinterpret_cast<uint4*>(smem);                           // [TB][d/8]
  float* logits = reinterpret_cast<float*>(smem + (size_t)TB * d * 2);  // [TB][RED_LD]
  SmallTail* st = reinterpret_cast<SmallTail*>(smem + (size_t)TB * d * 2 + (size_t)TB * RED_LD * 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = (int)blockIdx.x * TB;
  const int E = p.n_routed + p.n_shared;
  const int nv = d / 8;
  for (int i = tid; i < TB * nv; i += SMALL_THREADS) {
    const int r = i / nv, v = i - r * nv;
    xs[i] = t0 + r < p.T ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + r) * d) + v) : make_uint4(0, 0, 0, 0);
  }
  for (int i = tid; i < MOE_MAX_ROUTED; i += SMALL_THREADS) {
    st->bias[i] = i < p.n_routed ? p.bias[i] : 0.0f;
    st->off[i] = (p.offset != nullptr && i < p.n_routed) ? p.offset[i] : 0.0f;
    st->hist[i] = 0;
  }
  for (int i = tid; i < TB * RED_LD; i += SMALL_THREADS) logits[i] = 0.0f;
  __syncthreads();
  constexpr int SHIFT = 5 - (TB == 1 ? 0 : TB == 2 ? 1 : 2);
  for (int e0 = warp * U; e0 < E; e0 += (SMALL_THREADS / 32) * U) {
    float acc[U][TB];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int t = 0; t < TB; ++t) acc[u][t] = 0.0f;
    for (int v = lane; v < nv; v += 32) {
      float wf[U][8];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int e = min(e0 + u, E - 1);
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(w + (size_t)e * d) + v), wf[u]);
      }
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        float xf[8];
        bf16x8_to_f32(xs[t * nv + v], xf);
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[u][t] = fmaf(xf[j], wf[u][j], acc[u][t]);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float v = warp_sum_scatter<TB>(acc[u], lane);
      if (e0 + u < E && (lane & ((1 << SHIFT) - 1)) == 0) logits[(lane >> SHIFT) * RED_LD + e0 + u] = v;
    }
  }
  __syncthreads();
  if (warp < TB && t0 + warp < p.T) route_tokens_warp<K, 1>(p, st, logits + (size_t)warp * RED_LD, RED_LD, t0 + warp, 1, lane);
  __syncthreads();
  for (int e = tid; e < p.n_routed; e += SMALL_THREADS) {
    const int c = st->hist[e];
    if (c) atomicAdd(&p.counts[e], c);
  }
}

template <int K, int TB>
int launch_single(const __nv_bfloat16* x, const __nv_bfloat16* w, const Params& p, cudaStream_t s) {
  // 16 experts a round for rows of at most 256 values (one 16-byte load per lane and expert) and up to two
  // tokens a CTA, else 8
  auto kfn = router_single_kernel<K, TB, 8>;
  if constexpr (TB <= 2) {
    if (p.d <= 256) kfn = router_single_kernel<K, TB, 16>;
  }
  const size_t bytes = small_smem_bytes<TB>(p.d);
  int rc = ensure_smem_attr((const void*)kfn, bytes);
  if (rc != MOE_OK) return rc;
  kfn<<<(p.T + TB - 1) / TB, SMALL_THREADS, bytes, s>>>(x, w, p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int K, int TB>
int launch_small(const __nv_bfloat16* x, const __nv_bfloat16* w, const Params& p, cudaStream_t s) {
  auto kfn = router_small_kernel<K, TB>;
  const size_t bytes = small_smem_bytes<TB>(p.d);
  int rc = ensure_smem_attr((const void*)kfn, bytes);
  if (rc != MOE_OK) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(((p.T + TB - 1) / TB) * SMALL_CL), 1, 1);
  cfg.blockDim = dim3(SMALL_THREADS, 1, 1);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = SMALL_CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kfn, x, w, p) != cudaSuccess) return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// MOE_ROUTER_SINGLE=0 keeps narrow rows on the cluster kernel (to test both small-batch kernels).
bool single_allowed() {
  const char* env = getenv("MOE_ROUTER_SINGLE");
  return !(env && env[0] == '0' && env[1] == '\0');
}

// Tokens per cluster: about 128 CTAs in flight for the batch, at most 16 tokens, and the
// staged rows within the shared-memory budget.  0: the small path does not apply.
int small_tb(int T, int d) {
  if (T > SMALL_T_MAX || d > SMALL_D_MAX) return 0;
  int tb = 1;
  while (tb < SMALL_TB_MAX && (long long)((T + 2 * tb - 1) / (2 * tb)) * SMALL_CL >= 128) tb *= 2;
  while (tb > 1 && (size_t)tb * d * 2 > SMALL_X_BUDGET) tb /= 2;
  if ((size_t)tb * d * 2 > SMALL_X_BUDGET) return 0;
  return tb;
}

template <int K>
int launch_small_k(const __nv_bfloat16* x, const __nv_bfloat16* w, const Params& p, int tb, cudaStream_t s) {
  if (p.d <= SINGLE_D_MAX && single_allowed()) {  // tokens per CTA: about 128 CTAs, at most 4
    const int tpc = p.T >= 512 ? 4 : (p.T >= 256 ? 2 : 1);
    if (tpc == 4) return launch_single<K, 4>(x, w, p, s);
    if (tpc == 2) return launch_single<K, 2>(x, w, p, s);
    return launch_single<K, 1>(x, w, p, s);
  }
  switch (tb) {
    case 1: return launch_small<K, 1>(x, w, p, s);
    case 2: return launch_small<K, 2>(x, w, p, s);
    case 4: return launch_small<K, 4>(x, w, p, s);
    case 8: return launch_small<K, 8>(x, w, p, s);
    default: return launch_small<K, 16>(x, w, p, s);
  }
}

template <int K>
int launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const Params& p, int grid,
           cudaStream_t s) {
  auto kfn = router_kernel<K>;
  int rc = ensure_smem_attr((const void*)kfn, SMEM_BYTES);
  if (rc != MOE_OK) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.ksplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kfn, a, b0, b1, p) != cudaSuccess) return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Cluster size sharing one tile: the largest S in {1, 2, 4, 8} that keeps all
// CTAs resident at once (one per SM), divides the K blocks, and leaves each CTA
// at least two of them.
int choose_ksplit(int n_mtiles, int num_kb, int sms) {
  int S = 1;
  while (S < MAX_SPLIT && (long long)n_mtiles * S * 2 <= sms && num_kb % (S * 2) == 0 && num_kb / (S * 2) >= 2)
    S *= 2;
  return S;
}

}  // namespace router
}  // namespace moe

using namespace moe;

extern "C" int moe_router_topk(const moe_bf16* x, const moe_bf16* w_router, const float* bias,
                               const float* logit_offset, int T, int d, int n_routed, int n_shared, int top_k,
                               float route_scale, int32_t* topk_idx, float* gates, int32_t* counts,
                               float* scores_out, void* stream) {
  using namespace moe::router;
  if (!x || !w_router || !bias || !topk_idx || !gates || !counts) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned4(bias) || !aligned4(topk_idx) || !aligned4(gates) ||
      !aligned4(counts) || !aligned4(logit_offset) || !aligned4(scores_out))
    return MOE_ERR_INVALID_ARG;
  if (T < 0 || d <= 0 || n_routed < 1 || n_shared < 0 || top_k < 1) return MOE_ERR_INVALID_ARG;
  if (top_k > MOE_MAX_TOP_K || top_k > n_routed) return MOE_ERR_INVALID_ARG;
  if (!(route_scale > 0.0f) || route_scale > 3.0e38f) return MOE_ERR_INVALID_ARG;  // finite, positive
  if (n_routed > MOE_MAX_ROUTED || n_shared > MOE_MAX_SHARED || n_routed + n_shared > B0_ROWS + B1_ROWS)
    return MOE_ERR_UNSUPPORTED;
  if (d % 8 != 0) return MOE_ERR_UNSUPPORTED;  // 16-byte row pitch for the tensor map
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * n_routed, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (T == 0) return MOE_OK;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;

  // small batches: CUDA-core logits over many CTAs (MOE_ROUTER_SMALL=0 or =1 forces the choice)
  int tb = small_tb(T, d);
  {
    const char* env = getenv("MOE_ROUTER_SMALL");
    if (env && env[0] == '0' && env[1] == '\0') tb = 0;
    if (env && env[0] == '1' && env[1] == '\0' && tb == 0) {
      tb = 1;
      while (tb > 0 && (size_t)tb * d * 2 > SMALL_X_BUDGET) tb = 0;
    }
  }
  if (tb > 0 && n_routed + n_shared <= RED_COLS) {
    Params p{};
    p.bias = bias;
    p.offset = logit_offset;
    p.T = T;
    p.d = d;
    p.n_routed = n_routed;
    p.n_shared = n_shared;
    p.ksplit = 1;
    p.topk_idx = topk_idx;
    p.gates = gates;
    p.gate_scale = route_scale;
    p.counts = counts;
    p.scores = scores_out;
    p.timeout_ns = wait_timeout_ns();
    p.status = status_ptr();
    if (!p.status) return MOE_ERR_CUDA;
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(w_router);
    switch (top_k) {
      case 1: return launch_small_k<1>(xb, wb, p, tb, s);
      case 2: return launch_small_k<2>(xb, wb, p, tb, s);
      case 3: return launch_small_k<3>(xb, wb, p, tb, s);
      case 4: return launch_small_k<4>(xb, wb, p, tb, s);
      case 5: return launch_small_k<5>(xb, wb, p, tb, s);
      case 6: return launch_small_k<6>(xb, wb, p, tb, s);
      case 7: return launch_small_k<7>(xb, wb, p, tb, s);
      default: return launch_small_k<8>(xb, wb, p, tb, s);
    }
  }

  const int E = n_routed + n_shared;
  CUtensorMap tA, tB0, tB1;
  if ((rc = encode_tmap_bf16(&tA, x, 2, (uint64_t)d, (uint64_t)T, 1, BK, BM)) != MOE_OK) return rc;
  if ((rc = encode_tmap_bf16(&tB0, w_router, 2, (uint64_t)d, (uint64_t)E, 1, BK, B0_ROWS)) != MOE_OK) return rc;
  if ((rc = encode_tmap_bf16(&tB1, w_router, 2, (uint64_t)d, (uint64_t)E, 1, BK, B1_ROWS)) != MOE_OK) return rc;

  const int n_mtiles = (T + BM - 1) / BM;
  Params p{};
  p.bias = bias;
  p.offset = logit_offset;
  p.T = T;
  p.d = d;
  p.n_routed = n_routed;
  p.n_shared = n_shared;
  p.ksplit = choose_ksplit(n_mtiles, (d + BK - 1) / BK, sms);
  p.topk_idx = topk_idx;
  p.gates = gates;
  p.gate_scale = route_scale;
  p.counts = counts;
  p.scores = scores_out;
  p.timeout_ns = wait_timeout_ns();
  p.status = status_ptr();
  if (!p.status) return MOE_ERR_CUDA;
  const int grid = n_mtiles * p.ksplit;
  switch (top_k) {
    case 1: return launch<1>(tA, tB0, tB1, p, grid, s);
    case 2: return launch<2>(tA, tB0, tB1, p, grid, s);
    case 3: return launch<3>(tA, tB0, tB1, p, grid, s);
    case 4: return launch<4>(tA, tB0, tB1, p, grid, s);
    case 5: return launch<5>(tA, tB0, tB1, p, grid, s);
    case 6: return launch<6>(tA, tB0, tB1, p, grid, s);
    case 7: return launch<7>(tA, tB0, tB1, p, grid, s);
    default: return launch<8>(tA, tB0, tB1, p, grid, s);
  }
}
