// grouped_ffn.cu -- the expert MLPs y = W2_e gelu(W1_e x) over groups of rows
// ("Inkling, Dissected" §02: an expert is two matmuls with a nonlinearity),
// as two launches of one persistent, warp-specialised tcgen05 grouped GEMM:
//
//   GEMM1:  H[rows of e] = gelu(X[rows of e] . W1_e^T)   (bf16 out, GELU fused)
//   GEMM2:  Y[rows of e] =      H[rows of e] . W2_e^T    (bf16 out)
//
// Per CTA (one per SM, persistent over a static round-robin of 128x256 tiles):
//   warp 0      TMA producer: A (128 x 64) and B (256 x 64) bf16 tiles, 128-byte
//               swizzle, into a 4-stage shared-memory ring (full/empty mbarriers)
//   warp 1      TMEM owner + MMA issuer: tcgen05.mma.cta_group::1.kind::f16,
//               M=128 N=256 K=16, fp32 accumulators in TMEM, two accumulator
//               buffers (512 columns) so the epilogue of tile i overlaps the
//               main loop of tile i+1
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time, activation, bf16
//               rounding, 16-byte stores of each row's 64-byte chunk
// Ragged groups: a tile's A rows run past its group into the next group's rows
// (or past the tensor, where TMA fills zeros); the epilogue writes only the
// group's own rows.  The tile list is built on the device from the group
// offsets, so the host never reads the per-expert counts.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include "moe.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace gffn {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int EPI_GELU = 0;
constexpr int EPI_NONE = 1;

struct Params {
  const int* offsets;  // [n_groups + 1] or null (every group sees rows 0..n_rows-1)
  int n_groups;
  int n_rows;          // rows of A for offsets mode; rows per group in identity mode
  int a_group_stride;  // identity mode: A row base of group g = g * a_group_stride
  int c_group_stride;  // identity mode: C row base of group g = g * c_group_stride
  int c_row_limit;     // rows of C (writes at or past it are skipped)
  int N;               // output columns
  int K;               // reduction length
  int n_tiles_n;
  __nv_bfloat16* C;
  int ldc;
  uint64_t timeout_ns;
  unsigned int* status;
};

struct SmemTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int off[MOE_MAX_GROUPS + 1];
  int prefix[MOE_MAX_GROUPS + 1];
};

constexpr size_t SMEM_BYTES = 1024 /* alignment slack */ + (size_t)STAGES * STAGE_BYTES + sizeof(SmemTail);

struct TileInfo {
  int g, m, nt;
};

__device__ __forceinline__ TileInfo tile_info(int tile, const int* prefix, int n_groups, int n_tiles_n) {
  TileInfo ti;
  int mt = tile / n_tiles_n;
  ti.nt = tile - mt * n_tiles_n;
  int lo = 0, hi = n_groups;  // largest g with prefix[g] <= mt
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= mt)
      lo = mid;
    else
      hi = mid;
  }
  ti.g = lo;
  ti.m = mt - prefix[lo];
  return ti;
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smemA = smem;
  uint8_t* smemB = smem + STAGES * A_BYTES;
  SmemTail* st = reinterpret_cast<SmemTail*>(smem + STAGES * STAGE_BYTES);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const bool identity = (p.offsets == nullptr);

  // ---- setup: barriers, group table, m-tile prefix ----
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&st->tfull[a], 1);
      mbar_init(&st->tempty[a], 128);
    }
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    fence_barrier_init();
  }
  if (!identity) {
    for (int i = tid; i <= p.n_groups; i += NUM_THREADS) {
      int v = p.offsets[i];
      st->off[i] = v < 0 ? 0 : (v > p.n_rows ? p.n_rows : v);
    }
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.n_groups; base += 32) {
      int g = base + lane;
      int cnt = 0;
      if (g < p.n_groups) {
        int rows = identity ? p.n_rows : st->off[g + 1] - st->off[g];
        cnt = rows > 0 ? (rows + BM - 1) / BM : 0;
      }
      int v = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (g < p.n_groups) st->prefix[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) st->prefix[0] = 0;
  }
  __syncthreads();
  const int total_tiles = st->prefix[p.n_groups] * p.n_tiles_n;
  if ((int)blockIdx.x >= total_tiles) return;  // uniform across the CTA, before TMEM is taken

  if (warp == 1) tmem_alloc(&st->tmem_base, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = st->tmem_base;
  const int num_kb = (p.K + BK - 1) / BK;
  volatile int* abort_flag = &st->abort_flag;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        TileInfo ti = tile_info(tile, st->prefix, p.n_groups, p.n_tiles_n);
        int a_row = (identity ? ti.g * p.a_group_stride : st->off[ti.g]) + ti.m * BM;
        int n0 = ti.nt * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&st->empty[stage], phase ^ 1u, p.timeout_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&st->full[stage], STAGE_BYTES);
          tma_load_2d(smemA + stage * A_BYTES, &tmA, &st->full[stage], kb * BK, a_row);
          tma_load_3d(smemB + stage * B_BYTES, &tmB, &st->full[stage], kb * BK, n0, ti.g);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // wind down: let the copies already issued land before the CTA exits
        int zero = 0;
        for (long i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
          mbar_wait(&st->full[i % STAGES], (uint32_t)((i / STAGES) & 1), p.timeout_ns, &zero, p.status);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&st->tempty[acc], acc_phase ^ 1u, p.timeout_ns, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&st->full[stage], phase, p.timeout_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smemA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(smemB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            mma_bf16_ss(d_tmem, make_desc_sw128(a_addr + k * 32), make_desc_sw128(b_addr + k * 32), idesc,
                        (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit(&st->empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&st->tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // no MMA may still be running when TMEM is released
      int zero = 0;
      mma_commit(&st->drain);
      mbar_wait(&st->drain, 0, p.timeout_ns, &zero, p.status);
    }
  } else {
    // ================= epilogue (warps 2..5) =================
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      TileInfo ti = tile_info(tile, st->prefix, p.n_groups, p.n_tiles_n);
      int rows_g = identity ? p.n_rows : st->off[ti.g + 1] - st->off[ti.g];
      int c_base = identity ? ti.g * p.c_group_stride : st->off[ti.g];
      int r = ti.m * BM + row_in_tile;
      int c_row = c_base + r;
      bool valid = (r < rows_g) && (c_row < p.c_row_limit);
      if (!mbar_wait(&st->tfull[acc], acc_phase, p.timeout_ns, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      __nv_bfloat16* crow = p.C + (size_t)c_row * p.ldc;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        const int col0 = ti.nt * BN + ch * 32;
        if (col0 >= p.N) break;  // same for the whole warp
        float v[32];
        tmem_ld32(taddr + ch * 32, v);
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a = v[2 * i], b = v[2 * i + 1];
            if (EPI == EPI_GELU) {
              a = gelu_tanh_f32(a);
              b = gelu_tanh_f32(b);
            }
            pk[i] = pack_bf16x2(a, b);
          }
          uint4* dst = reinterpret_cast<uint4*>(crow + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&st->tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
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
// CTA-pair variant: a cluster of 2 CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256).  CTA rank r holds A rows
// r*128 .. r*128+127 of the tile and B rows (output columns) r*128 ..
// r*128+127 in its own shared memory, and receives accumulator rows r*128 ..
// in its own TMEM.  Each CTA's producer loads its halves; every load signals
// the leader's (rank 0) full barrier, whose producer expects both halves'
// bytes.  The leader's single MMA thread issues for the pair and commits to
// both CTAs' empty / accumulator-full barriers; both CTAs' epilogue warps
// release the accumulator on the leader's barrier.  Per CTA and K step this
// halves the B operand's shared-memory traffic of the 1-CTA kernel.
// ---------------------------------------------------------------------------
constexpr int P_BM = 256;                      // tile rows per pair
constexpr int P_HALF = 128;                    // rows (of A and of B) per CTA
constexpr int P_STAGES = 6;
constexpr int P_A_BYTES = P_HALF * BK * 2;     // 16 KB
constexpr int P_B_BYTES = P_HALF * BK * 2;     // 16 KB
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;

struct SmemTailPair {
  uint64_t full[P_STAGES];
  uint64_t empty[P_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int off[MOE_MAX_GROUPS + 1];
  int prefix[MOE_MAX_GROUPS + 1];
};

constexpr size_t P_SMEM_BYTES = 1024 + (size_t)P_STAGES * P_STAGE_BYTES + sizeof(SmemTailPair);

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smemA = smem;
  uint8_t* smemB = smem + P_STAGES * P_A_BYTES;
  SmemTailPair* st = reinterpret_cast<SmemTailPair*>(smem + P_STAGES * P_STAGE_BYTES);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const bool identity = (p.offsets == nullptr);

  if (tid == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&st->tfull[a], 1);
      mbar_init(&st->tempty[a], 8);  // 4 epilogue warps x 2 CTAs
    }
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    fence_barrier_init();
  }
  if (!identity) {
    for (int i = tid; i <= p.n_groups; i += NUM_THREADS) {
      int v = p.offsets[i];
      st->off[i] = v < 0 ? 0 : (v > p.n_rows ? p.n_rows : v);
    }
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.n_groups; base += 32) {
      int g = base + lane;
      int cnt = 0;
      if (g < p.n_groups) {
        int rows = identity ? p.n_rows : st->off[g + 1] - st->off[g];
        cnt = rows > 0 ? (rows + P_BM - 1) / P_BM : 0;
      }
      int v = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (g < p.n_groups) st->prefix[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) st->prefix[0] = 0;
  }
  __syncthreads();
  const int total_tiles = st->prefix[p.n_groups] * p.n_tiles_n;
  if (pair >= total_tiles) return;  // both CTAs of the pair leave together, before any cluster traffic

  if (warp == 1) tmem_alloc_pair(&st->tmem_base, TMEM_COLS);
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM taken in both
  tc_fence_after();
  const uint32_t tmem_base = st->tmem_base;
  const int num_kb = (p.K + BK - 1) / BK;
  volatile int* abort_flag = &st->abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        TileInfo ti = tile_info(tile, st->prefix, p.n_groups, p.n_tiles_n);
        int a_row = (identity ? ti.g * p.a_group_stride : st->off[ti.g]) + ti.m * P_BM + (int)rank * P_HALF;
        int b_row = ti.nt * BN + (int)rank * P_HALF;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&st->empty[stage], phase ^ 1u, p.timeout_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(&st->full[stage], 2 * P_STAGE_BYTES);
          tma_load_2d_pair(smemA + stage * P_A_BYTES, &tmA, &st->full[stage], kb * BK, a_row);
          tma_load_3d_pair(smemB + stage * P_B_BYTES, &tmB, &st->full[stage], kb * BK, b_row, ti.g);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = make_idesc_bf16(P_BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        if (!mbar_wait(&st->tempty[acc], acc_phase ^ 1u, p.timeout_ns, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&st->full[stage], phase, p.timeout_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smemA + stage * P_A_BYTES);
          const uint32_t b_addr = smem_u32(smemB + stage * P_B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            mma_bf16_ss_pair(d_tmem, make_desc_sw128(a_addr + k * 32), make_desc_sw128(b_addr + k * 32), idesc,
                             (kb | k) != 0 ? 1u : 0u);
          }
          mma_commit_pair(&st->empty[stage], 0x3);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair(&st->tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      int zero = 0;
      mma_commit_pair(&st->drain, 0x1);
      mbar_wait(&st->drain, 0, p.timeout_ns, &zero, p.status);
    }
  } else {
    const int quarter = warp & 3;
    const int row_in_tile = (int)rank * P_HALF + quarter * 32 + lane;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&st->tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&st->tempty[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      TileInfo ti = tile_info(tile, st->prefix, p.n_groups, p.n_tiles_n);
      int rows_g = identity ? p.n_rows : st->off[ti.g + 1] - st->off[ti.g];
      int c_base = identity ? ti.g * p.c_group_stride : st->off[ti.g];
      int r = ti.m * P_BM + row_in_tile;
      int c_row = c_base + r;
      bool valid = (r < rows_g) && (c_row < p.c_row_limit);
      if (!mbar_wait(&st->tfull[acc], acc_phase, p.timeout_ns, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BN);
      __nv_bfloat16* crow = p.C + (size_t)c_row * p.ldc;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        const int col0 = ti.nt * BN + ch * 32;
        if (col0 >= p.N) break;
        float v[32];
        tmem_ld32(taddr + ch * 32, v);
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a = v[2 * i], b = v[2 * i + 1];
            if (EPI == EPI_GELU) {
              a = gelu_tanh_f32(a);
              b = gelu_tanh_f32(b);
            }
            pk[i] = pack_bf16x2(a, b);
          }
          uint4* dst = reinterpret_cast<uint4*>(crow + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  cluster_sync_all();  // every MMA of the pair has landed and both CTAs are done with each other's memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

template <int EPI>
int launch_pair(const CUtensorMap& tmA, const CUtensorMap& tmB, const Params& p, int grid, cudaStream_t stream) {
  auto kfn = grouped_gemm_pair_kernel<EPI>;
  int rc = ensure_smem_attr((const void*)kfn, P_SMEM_BYTES);
  if (rc != MOE_OK) return rc;
  kfn<<<grid, NUM_THREADS, P_SMEM_BYTES, stream>>>(tmA, tmB, p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

template <int EPI>
int launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const Params& p, int grid, cudaStream_t stream) {
  auto kfn = grouped_gemm_kernel<EPI>;
  int rc = ensure_smem_attr((const void*)kfn, SMEM_BYTES);
  if (rc != MOE_OK) return rc;
  kfn<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(tmA, tmB, p);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace gffn
}  // namespace moe

using namespace moe;

extern "C" int moe_grouped_ffn(const moe_bf16* rows, const int32_t* offsets, int n_groups, int n_rows,
                               int expert_base, const moe_bf16* w1, const moe_bf16* w2, int d, int d_ff,
                               int activation, moe_bf16* h_scratch, moe_bf16* y, void* stream) {
  using namespace moe::gffn;
  if (n_groups < 0 || n_rows < 0 || expert_base < 0 || d <= 0 || d_ff <= 0) return MOE_ERR_INVALID_ARG;
  if (activation != MOE_ACT_GELU_TANH) return MOE_ERR_INVALID_ARG;
  if (!aligned16(rows) || !aligned16(w1) || !aligned16(w2) || !aligned16(h_scratch) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  if (!rows || !w1 || !w2 || !h_scratch || !y) return MOE_ERR_INVALID_ARG;
  if (d % 64 != 0 || d_ff % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (n_groups > MOE_MAX_GROUPS) return MOE_ERR_UNSUPPORTED;
  if (n_rows == 0 || n_groups == 0) return MOE_OK;
  const bool identity = (offsets == nullptr);
  if (!identity && !aligned4(offsets)) return MOE_ERR_INVALID_ARG;
  const long long h_rows = identity ? (long long)n_groups * n_rows : n_rows;
  if (h_rows > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;

  cudaStream_t s = (cudaStream_t)stream;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;

  const __nv_bfloat16* w1e = reinterpret_cast<const __nv_bfloat16*>(w1) + (size_t)expert_base * d_ff * d;
  const __nv_bfloat16* w2e = reinterpret_cast<const __nv_bfloat16*>(w2) + (size_t)expert_base * d * d_ff;

  // Kernel variant.  CTA pairs (cta_group::2, 256 x 256 tiles) halve each CTA's shared-memory
  // operand traffic and win when groups are large (compute-bound); with few rows per group the
  // work is weight streaming and single CTAs (128 x 256 tiles, more weight bytes in flight per
  // SM) win.  MOE_GEMM_CTA=1 or =2 forces one of them.
  const char* env = getenv("MOE_GEMM_CTA");
  const long long rows_per_group = identity ? n_rows : n_rows / n_groups;
  bool pair = rows_per_group >= 256;
  if (env && env[0] == '1' && env[1] == '\0') pair = false;
  if (env && env[0] == '2' && env[1] == '\0') pair = true;
  const uint32_t b_box = pair ? (uint32_t)P_HALF : (uint32_t)BN;
  const int tile_m = pair ? P_BM : BM;

  CUtensorMap tA1, tB1, tA2, tB2;
  // GEMM1: A = rows [n_rows, d], B = W1 [n_groups, d_ff, d]
  if ((rc = encode_tmap_bf16(&tA1, rows, 2, (uint64_t)d, (uint64_t)n_rows, 1, BK, BM)) != MOE_OK) return rc;
  if ((rc = encode_tmap_bf16(&tB1, w1e, 3, (uint64_t)d, (uint64_t)d_ff, (uint64_t)n_groups, BK, b_box)) != MOE_OK)
    return rc;
  // GEMM2: A = H [h_rows, d_ff], B = W2 [n_groups, d, d_ff]
  if ((rc = encode_tmap_bf16(&tA2, h_scratch, 2, (uint64_t)d_ff, (uint64_t)h_rows, 1, BK, BM)) != MOE_OK)
    return rc;
  if ((rc = encode_tmap_bf16(&tB2, w2e, 3, (uint64_t)d_ff, (uint64_t)d, (uint64_t)n_groups, BK, b_box)) != MOE_OK)
    return rc;

  // upper bound on m-tiles: every group may add one partial tile
  long long mtiles = identity ? (long long)n_groups * ((n_rows + tile_m - 1) / tile_m)
                              : (n_rows + tile_m - 1) / tile_m + n_groups;
  auto grid_for = [&](long long tiles) -> int {
    if (pair) {
      long long pairs = tiles < sms / 2 ? tiles : sms / 2;
      return (int)(2 * pairs);
    }
    return (int)(tiles < sms ? tiles : sms);
  };

  Params p1{};
  p1.offsets = offsets;
  p1.n_groups = n_groups;
  p1.n_rows = n_rows;
  p1.a_group_stride = 0;
  p1.c_group_stride = n_rows;
  p1.c_row_limit = (int)h_rows;
  p1.N = d_ff;
  p1.K = d;
  p1.n_tiles_n = (d_ff + BN - 1) / BN;
  p1.C = reinterpret_cast<__nv_bfloat16*>(h_scratch);
  p1.ldc = d_ff;
  p1.timeout_ns = wait_timeout_ns();
  p1.status = status_ptr();
  if (!p1.status) return MOE_ERR_CUDA;
  const int grid1 = grid_for(mtiles * p1.n_tiles_n);
  rc = pair ? launch_pair<EPI_GELU>(tA1, tB1, p1, grid1, s) : launch<EPI_GELU>(tA1, tB1, p1, grid1, s);
  if (rc != MOE_OK) return rc;

  Params p2 = p1;
  p2.a_group_stride = n_rows;
  p2.c_group_stride = n_rows;
  p2.c_row_limit = (int)h_rows;
  p2.N = d;
  p2.K = d_ff;
  p2.n_tiles_n = (d + BN - 1) / BN;
  p2.C = reinterpret_cast<__nv_bfloat16*>(y);
  p2.ldc = d;
  const int grid2 = grid_for(mtiles * p2.n_tiles_n);
  return pair ? launch_pair<EPI_NONE>(tA2, tB2, p2, grid2, s) : launch<EPI_NONE>(tA2, tB2, p2, grid2, s);
}
