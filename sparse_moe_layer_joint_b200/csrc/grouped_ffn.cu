// grouped_ffn.cu -- the expert MLPs y = W2_e gelu(W1_e x) over groups of rows
// ("Inkling, Dissected" §02: an expert is two matmuls with a nonlinearity), as
// two launches of one persistent, warp-specialised tcgen05 grouped GEMM:
//
//   GEMM1:  H[rows of e] = gelu(X[rows of e] . W1_e^T)   (bf16 out, GELU fused)
//   GEMM2:  Y[rows of e] =      H[rows of e] . W2_e^T    (bf16 out)
//
// Groups.  A launch covers G_r "routed" groups, whose rows are given by device
// offsets (the dispatch layout), followed by G_s "shared" groups that each see
// the same `shared_rows` rows (every token).  Group g uses expert g of the
// weight tensors it is given, so one launch can run the 256 routed and the 2
// shared experts of the layer together.  The tile list, (group, row tile,
// column tile) with the column index fastest, is built on the device from the
// offsets, so the host never reads the per-expert counts.
//
// Per CTA (persistent, static round-robin over tiles):
//   warp 0      TMA producer into a shared-memory ring of A and B tiles
//               (128-byte swizzle, full/empty mbarriers); in gathering launches
//               the routed A rows come from the token rows through the row
//               indices, one tile::gather4 load (four rows) per lane and stage
//   warp 1      TMEM owner + MMA issuer (one thread): tcgen05.mma kind::f16,
//               bf16 in, fp32 accumulators in TMEM: two 256-column
//               accumulator buffers so the epilogue of tile i overlaps the
//               main loop of tile i+1 (one 512-column buffer for WIDE tiles)
//   warps 2-5   epilogue (2-9 for WIDE tiles): tcgen05.ld, activation, bf16,
//               16-byte stores of each row's 64-byte chunks
// Variants:
//   PAIR = false  one CTA per 128 x 256 tile (4-stage ring of 48 KB)
//   PAIR = true   a cluster of two CTAs per 256 x 256 tile with
//                 tcgen05.mma.cta_group::2 (M = 256): CTA rank r holds A rows
//                 r*128.. and B rows (output columns) r*128.. in its own
//                 shared memory and accumulator rows r*128.. in its own TMEM;
//                 both CTAs' loads signal the leader's full barrier, the
//                 leader's MMA thread issues for the pair and commits to both
//                 CTAs' barriers, both epilogues release the accumulator on
//                 the leader.  Per CTA this halves the B operand's shared-
//                 memory traffic (6-stage ring of 32 KB).
//   WIDE          pair tiles of 256 x 512 accumulator columns (see Cfg): 25% fewer
//                 L2 bytes per FLOP and one accumulator, which the epilogue hands
//                 back as soon as it holds its share as packed bf16 registers
//                 (the stores then overlap the next tile's MMAs); SwiGLU tiles
//                 hold 256 gate and the 256 matching up columns; the default for
//                 pair launches (MOE_GEMM_WIDE=0: 256 x 256).
//   half tiles    (pairs, GELU and plain epilogues, groups of at most 1024 rows
//                 on average) a group's last row tile with at most 128 rows runs
//                 as an M = 128 pair MMA: 64 rows a CTA, whose 64 x 256 result
//                 TMEM holds folded (lanes 0-63 the first 128 columns, lanes
//                 64-127 the other 128), at half the MMA work.
// Ragged groups: a tile's A rows may run past its group (into the next
// group's rows, or past the tensor where TMA fills zeros); the epilogue writes
// only the group's own rows.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <type_traits>

#include "moe.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace gffn {

constexpr int BN = 256;  // output columns per tile
constexpr int BK = 64;   // reduction depth per stage (one 128-byte swizzle atom)
constexpr uint32_t TMEM_COLS = 512;
constexpr int EPI_GELU = 0;
constexpr int EPI_NONE = 1;
// Gated first GEMM of SwiGLU experts: a tile's 256 accumulator columns are 128 gate
// columns (weight rows 128*nt ..) then the 128 matching up columns (rows b_up_row +
// 128*nt ..), and the epilogue writes silu(gate) * up into 128 output columns.
constexpr int EPI_SWIGLU = 2;
constexpr int SWIGLU_OUT = BN / 2;

// WIDE (pairs only): a tile is 256 x 512, two 256-column halves that share the A stage; each CTA
// holds 128 A rows and 2 x 128 weight rows per stage, so a K step moves 48 KB per CTA for twice
// the MMA work of a 256 x 256 tile (32 KB): 25% fewer L2 -> shared-memory bytes per FLOP.  Its
// 512-column accumulator fills TMEM, so there is one accumulator, read by eight epilogue warps (two
// per TMEM lane quarter, one per column half) into packed bf16 registers; the next tile's MMAs start
// once every warp holds its share, while the warps store it.
template <bool PAIR, int ST, bool WIDE = false>
struct Cfg {
  static_assert(!WIDE || PAIR, "wide tiles are pair tiles");
  static constexpr int NH = WIDE ? 2 : 1;          // 256-column halves per tile
  static constexpr int TILE_N = BN * NH;           // output columns per tile
  static constexpr int TILE_M = PAIR ? 256 : 128;  // rows per tile (per pair, or per CTA)
  static constexpr int A_ROWS = 128;               // A rows held by one CTA
  static constexpr int B_HALF_ROWS = PAIR ? 128 : 256;  // weight rows of one column half held by one CTA
  static constexpr int B_ROWS = B_HALF_ROWS * NH;  // B rows (output columns) held by one CTA
  static constexpr int STAGES = ST;
  static constexpr int A_BYTES = A_ROWS * BK * 2;
  static constexpr int B_HALF_BYTES = B_HALF_ROWS * BK * 2;
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_WARPS = 4 * NH;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int ACC_BUFS = WIDE ? 1 : 2;   // accumulators of 256 * NH columns in TMEM
  static constexpr uint32_t TX_BYTES = (PAIR ? 2 : 1) * STAGE_BYTES;  // bytes landing on the (leader's) full barrier
  static_assert(A_ROWS == 4 * 32, "one gather4 load per producer lane covers the CTA's A rows");
};

struct Params {
  const int* offsets;  // [G_r + 1] routed group row offsets (device); unused when G_r == 0
  const int* gather_rows;  // non-null: routed A rows are gathered through map A0 (one-row boxes),
                           // row r of group g = gather_rows[off[g] + r]
  int gather_limit;        // gathered row indices are clamped to [0, gather_limit)
  int G_r;             // routed groups
  int G_s;             // shared groups
  int routed_rows;     // offsets are clamped to [0, routed_rows]
  int shared_rows;     // rows of every shared group
  int a_sh_map;        // A tensor map of shared groups: 0 = tmA0 (as routed), 1 = tmA1
  int a_sh_base, a_sh_stride;  // A row of shared group s, row r: a_sh_base + s*a_sh_stride + r
  __nv_bfloat16* C0;           // routed output: row off[g] + r
  int c0_limit;
  __nv_bfloat16* C1;           // shared output: row c1_base + s*c1_stride + r
  int c1_base, c1_stride, c1_limit;
  int N;  // output columns
  int K;  // reduction length
  int b_up_row;  // EPI_SWIGLU: first weight row of the up projection (= d_ff)
  int n_tiles_n;
  int ldc;
  int prefetch_kb;   // > 0: also prefetch the tiles this many K blocks ahead into L2 (TMA prefetch)
  int n_major_rows;  // groups of at most this many row tiles run column-tile-major (0: none)
  int tail_mode;     // TAIL_ALL: every row of every group; TAIL_WHOLE: only each group's whole blocks of
                     // tail_unit rows; TAIL_ONLY: only the rows past them (two launches cover a group)
  int tail_unit;
  int hints;  // L2 policies: HINT_B_KEEP weight tiles evict_last, HINT_C_STREAM outputs evict_first,
              // HINT_A_STREAM A tiles evict_first
  int half_tiles;  // pair kernels, GELU / plain epilogues, tiled A loads: a group's last row tile with at
                   // most 128 rows runs as an M = 128 pair MMA (64 rows a CTA) at half the MMA work
  uint64_t timeout_ns;
  unsigned int* status;
};

constexpr int TAIL_ALL = 0;
constexpr int TAIL_WHOLE = 1;
constexpr int TAIL_ONLY = 2;

constexpr int HINT_B_KEEP = 1;
constexpr int HINT_C_STREAM = 2;
constexpr int HINT_A_STREAM = 4;

struct GroupTables {
  int off[MOE_MAX_GROUPS + 1];
  int prefix[MOE_MAX_GROUPS + 1];  // prefix[g] = row tiles of groups < g
};

template <int ST>
struct SmemTail {
  uint64_t full[ST];
  uint64_t empty[ST];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  GroupTables gt;
};

template <bool PAIR, int ST, bool WIDE = false>
constexpr size_t smem_bytes() {
  return 1024 /* alignment slack */ + (size_t)ST * Cfg<PAIR, ST, WIDE>::STAGE_BYTES + sizeof(SmemTail<ST>);
}

struct Group {
  int rows;
  int a_map;
  int a_base;
  int c_sel;
  int c_base;
};

__device__ __forceinline__ Group group_info(const Params& p, const GroupTables& gt, int g) {
  Group G;
  if (g < p.G_r) {
    G.rows = gt.off[g + 1] - gt.off[g];
    G.a_map = 0;
    G.a_base = gt.off[g];
    G.c_sel = 0;
    G.c_base = gt.off[g];
  } else {
    const int s = g - p.G_r;
    G.rows = p.shared_rows;
    G.a_map = p.a_sh_map;
    G.a_base = p.a_sh_base + s * p.a_sh_stride;
    G.c_sel = 1;
    G.c_base = p.c1_base + s * p.c1_stride;
  }
  if (p.tail_mode == TAIL_ONLY) {  // the rows past the group's last whole tail_unit-row block
    const int start = (G.rows / p.tail_unit) * p.tail_unit;
    G.rows -= start;
    G.a_base += start;
    G.c_base += start;
  }
  return G;
}

// Row tiles a group contributes to a launch (see Params::tail_mode).
template <int TILE_M>
__device__ __forceinline__ int group_row_tiles(const Params& p, int rows) {
  if (rows <= 0) return 0;
  if (p.tail_mode == TAIL_ALL) return (rows + TILE_M - 1) / TILE_M;
  if (p.tail_mode == TAIL_WHOLE) return (rows / p.tail_unit) * (p.tail_unit / TILE_M);
  rows -= (rows / p.tail_unit) * p.tail_unit;  // TAIL_ONLY
  return (rows + TILE_M - 1) / TILE_M;
}

struct TileInfo {
  int g, m, nt;
};

// Whether a tile runs as a half (M = 128) pair tile: its group's rows end within its first 128.
__device__ __forceinline__ bool half_tile(const Params& p, const Group& gr, const TileInfo& ti) {
  return p.half_tiles != 0 && gr.rows - ti.m * 256 <= 128;
}

// A group's tiles are the tile numbers [prefix[g] * n_tiles_n, prefix[g + 1] * n_tiles_n).  Within a
// group they run row-tile-major (the column tiles of one row block together) or, for groups of at most
// n_major_rows row tiles, column-tile-major (every row block of one weight tile together: each weight
// tile is read from DRAM once while the group's few A blocks stay in L2).
__device__ __forceinline__ TileInfo tile_info(int tile, const int* prefix, int n_groups, int n_tiles_n,
                                              int n_major_rows) {
  TileInfo ti;
  const int mt = tile / n_tiles_n;
  int lo = 0, hi = n_groups;  // largest g with prefix[g] <= mt (never an empty group)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= mt)
      lo = mid;
    else
      hi = mid;
  }
  ti.g = lo;
  const int rows_g = prefix[lo + 1] - prefix[lo];  // row tiles of the group
  if (rows_g <= n_major_rows) {
    const int l = tile - prefix[lo] * n_tiles_n;
    ti.nt = l / rows_g;
    ti.m = l - ti.nt * rows_g;
  } else {
    ti.nt = tile - mt * n_tiles_n;
    ti.m = mt - prefix[lo];
  }
  return ti;
}

// Load the routed offsets and build the row-tile prefix over all groups.
template <int TILE_M, int THREADS>
__device__ __forceinline__ void build_tables(const Params& p, GroupTables& gt, int tid, int warp, int lane) {
  for (int i = tid; i <= p.G_r && p.G_r > 0; i += THREADS) {
    int v = p.offsets[i];
    gt.off[i] = v < 0 ? 0 : (v > p.routed_rows ? p.routed_rows : v);
  }
  __syncthreads();
  const int G = p.G_r + p.G_s;
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      int g = base + lane;
      int cnt = 0;
      if (g < G) {
        int rows = g < p.G_r ? gt.off[g + 1] - gt.off[g] : p.shared_rows;
        cnt = group_row_tiles<TILE_M>(p, rows);
      }
      int v = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      if (g < G) gt.prefix[g + 1] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
    if (lane == 0) gt.prefix[0] = 0;
  }
  __syncthreads();
}

template <int EPI, bool PAIR, int ST, bool WIDE>
__global__ void __launch_bounds__(Cfg<PAIR, ST, WIDE>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmB, const Params p) {
  using C = Cfg<PAIR, ST, WIDE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smemA = smem;
  uint8_t* smemB = smem + C::STAGES * C::A_BYTES;
  SmemTail<ST>* st = reinterpret_cast<SmemTail<ST>*>(smem + C::STAGES * C::STAGE_BYTES);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // pair or CTA index
  const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&st->tfull[a], 1);
      mbar_init(&st->tempty[a], (PAIR ? 2 : 1) * C::EPI_WARPS);  // one arrival per epilogue warp (of both CTAs)
    }
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    fence_barrier_init();
  }
  build_tables<C::TILE_M, C::THREADS>(p, st->gt, tid, warp, lane);
  const int G = p.G_r + p.G_s;
  const int total_tiles = st->gt.prefix[G] * p.n_tiles_n;
  if (unit >= total_tiles) return;  // uniform across the CTA (and the pair), before TMEM is taken

  if (warp == 1) {
    if (PAIR)
      tmem_alloc_pair(&st->tmem_base, TMEM_COLS);
    else
      tmem_alloc(&st->tmem_base, TMEM_COLS);
  }
  tc_fence_before();
  if (PAIR)
    cluster_sync_all();  // both CTAs' barriers initialised and TMEM taken before any cross-CTA traffic
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = st->tmem_base;
  const int num_kb = (p.K + BK - 1) / BK;
  volatile int* abort_flag = &st->abort_flag;

  if (warp == 0) {
    // ================= producer =================
    // Tiles arrive by TMA.  Tiled loads are issued by lane 0.  In gathering launches the routed
    // groups' A rows are instead gathered from the source rows through the row indices with
    // tile::gather4 loads, one per lane and stage: lane l brings rows 4l .. 4l+3 of the CTA's
    // 128-row A tile, so the whole warp runs the loop.
    const bool gathering = p.gather_rows != nullptr;
    if (lane == 0) {
      tma_prefetch_desc(&tmA0);
      if (p.G_s > 0 && p.a_sh_map == 1) tma_prefetch_desc(&tmA1);
      tma_prefetch_desc(&tmB);
    }
    int stage = 0;
    uint32_t phase = 0;
    long issued = 0;
    bool ok = true;
    const bool active = gathering || lane == 0;  // without gathers, lane 0 alone produces
    const uint64_t pol_last = l2_policy_evict_last();
    const uint64_t pol_first = l2_policy_evict_first();
    for (int tile = unit; active && tile < total_tiles && ok; tile += n_units) {
      const TileInfo ti = tile_info(tile, st->gt.prefix, G, p.n_tiles_n, p.n_major_rows);
      const Group gr = group_info(p, st->gt, ti.g);
      const CUtensorMap* am = gr.a_map ? &tmA1 : &tmA0;
      const bool half = half_tile(p, gr, ti);
      // a half tile's CTA loads its usual 128-row box from its 64-row offset and uses the first 64 rows
      const int a_row = gr.a_base + ti.m * C::TILE_M + (int)rank * (half ? C::A_ROWS / 2 : C::A_ROWS);
      // weight rows of this CTA's share of the tile's 256 columns; for SwiGLU the first 128
      // columns are gate rows and the other 128 the matching up rows
      // (a wide tile's second half: b_row + 256)
      // (SwiGLU, wide: the first half's rows are gate rows, the second half's the matching up rows, so a
      // tile computes 256 outputs; SwiGLU on 256-column pairs: one CTA loads gate rows, the other up rows)
      const int b_row = EPI == EPI_SWIGLU ? (C::NH == 2 ? ti.nt * BN + (int)rank * C::B_HALF_ROWS
                                                        : (rank == 0u ? ti.nt * SWIGLU_OUT : p.b_up_row + ti.nt * SWIGLU_OUT))
                                          : ti.nt * C::TILE_N + (int)rank * C::B_HALF_ROWS;
      const int b_half_step = EPI == EPI_SWIGLU ? p.b_up_row : BN;  // weight rows between the two halves
      const bool gather = gathering && ti.g < p.G_r;
      int src[4] = {0, 0, 0, 0};  // this lane's four source rows (rows past the group: row 0, masked later)
      if (gather) {
        const int r0 = ti.m * C::TILE_M + (int)rank * C::A_ROWS + 4 * lane;  // row within the group
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (r0 + i < gr.rows) {
            const int v = __ldg(p.gather_rows + gr.a_base + r0 + i);
            src[i] = v < 0 ? 0 : (v >= p.gather_limit ? p.gather_limit - 1 : v);
          }
        }
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        if (lane == 0) ok = mbar_wait(&st->empty[stage], phase ^ 1u, p.timeout_ns, abort_flag, p.status);
        if (gathering) ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (lane == 0 && leader) mbar_arrive_expect_tx(&st->full[stage], C::TX_BYTES);
        uint8_t* a_dst = smemA + stage * C::A_BYTES;
        if (gather) {
          __syncwarp();
          uint8_t* dst = a_dst + lane * 4 * (BK * 2);
          if (PAIR)
            tma_gather4_pair(dst, &tmA0, &st->full[stage], kb * BK, src[0], src[1], src[2], src[3]);
          else
            tma_gather4(dst, &tmA0, &st->full[stage], kb * BK, src[0], src[1], src[2], src[3]);
        }
        if (lane == 0 && p.prefetch_kb > 0 && kb + p.prefetch_kb < num_kb) {
          // the K block prefetch_kb ahead goes to L2 now, so its DRAM latency overlaps this stage
          const int kp = (kb + p.prefetch_kb) * BK;
          if (!gather) tma_prefetch_l2_2d(am, kp, a_row);
#pragma unroll
          for (int h = 0; h < C::NH; ++h) {
            if (EPI == EPI_SWIGLU && !PAIR && h == 0) tma_prefetch_l2_3d(&tmB, kp, p.b_up_row + ti.nt * SWIGLU_OUT, ti.g);
            tma_prefetch_l2_3d(&tmB, kp, b_row + h * b_half_step, ti.g);
          }
        }
        if (lane == 0) {
          if (PAIR) {
            if (!gather) {
              if (p.hints & HINT_A_STREAM)
                tma_load_2d_pair_hint(a_dst, am, &st->full[stage], kb * BK, a_row, pol_first);
              else
                tma_load_2d_pair(a_dst, am, &st->full[stage], kb * BK, a_row);
            }
#pragma unroll
            for (int h = 0; h < C::NH; ++h) {
              uint8_t* b_dst = smemB + stage * C::B_BYTES + h * C::B_HALF_BYTES;
              if (p.hints & HINT_B_KEEP)
                tma_load_3d_pair_hint(b_dst, &tmB, &st->full[stage], kb * BK, b_row + h * b_half_step, ti.g,
                                      pol_last);
              else
                tma_load_3d_pair(b_dst, &tmB, &st->full[stage], kb * BK, b_row + h * b_half_step, ti.g);
            }
          } else {
            if (!gather) tma_load_2d(a_dst, am, &st->full[stage], kb * BK, a_row);
            if (EPI == EPI_SWIGLU) {  // two 128-row boxes: gate rows, then up rows
              uint8_t* b_dst = smemB + stage * C::B_BYTES;
              tma_load_3d(b_dst, &tmB, &st->full[stage], kb * BK, b_row, ti.g);
              tma_load_3d(b_dst + C::B_BYTES / 2, &tmB, &st->full[stage], kb * BK, p.b_up_row + ti.nt * SWIGLU_OUT,
                          ti.g);
            } else {
              tma_load_3d(smemB + stage * C::B_BYTES, &tmB, &st->full[stage], kb * BK, b_row, ti.g);
            }
          }
        }
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!ok && !PAIR && lane == 0) {
      // wind down: let the copies already issued land before the CTA exits
      int zero = 0;
      for (long i = issued > C::STAGES ? issued - C::STAGES : 0; i < issued; ++i)
        mbar_wait(&st->full[i % C::STAGES], (uint32_t)((i / C::STAGES) & 1), p.timeout_ns, &zero, p.status);
    }
  } else if (warp == 1) {
    // ================= MMA issuer (the pair's leader) =================
    if (lane == 0 && leader) {
      constexpr uint32_t idesc_full = make_idesc_bf16(C::TILE_M, BN);  // one MMA per 256-column half
      constexpr uint32_t idesc_half = make_idesc_bf16(C::TILE_M / 2, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = unit; tile < total_tiles && ok; tile += n_units) {
        const TileInfo ti = tile_info(tile, st->gt.prefix, G, p.n_tiles_n, p.n_major_rows);
        const bool half = half_tile(p, group_info(p, st->gt, ti.g), ti);
        // an M = 128 pair MMA folds each CTA's 64 x 256 result into 128 TMEM columns: lanes 0-63 hold
        // columns 0-127, lanes 64-127 columns 128-255
        const uint32_t idesc = half ? idesc_half : idesc_full;
        const uint32_t h_cols = half ? BN / 2 : BN;
        if (!mbar_wait(&st->tempty[acc], acc_phase ^ 1u, p.timeout_ns, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * C::TILE_N);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&st->full[stage], phase, p.timeout_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smemA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(smemB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = make_desc_sw128(a_addr + k * 32);
#pragma unroll
            for (int h = 0; h < C::NH; ++h) {
              const uint64_t bd = make_desc_sw128(b_addr + h * C::B_HALF_BYTES + k * 32);
              if (PAIR)
                mma_bf16_ss_pair(d_tmem + h * h_cols, ad, bd, idesc, (kb | k) != 0 ? 1u : 0u);
              else
                mma_bf16_ss(d_tmem + h * BN, ad, bd, idesc_full, (kb | k) != 0 ? 1u : 0u);
            }
          }
          if (PAIR)
            mma_commit_pair(&st->empty[stage], 0x3);
          else
            mma_commit(&st->empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (PAIR)
          mma_commit_pair(&st->tfull[acc], 0x3);
        else
          mma_commit(&st->tfull[acc]);
        if (++acc == C::ACC_BUFS) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // no MMA may still be running when TMEM is released
      int zero = 0;
      if (PAIR)
        mma_commit_pair(&st->drain, 0x1);
      else
        mma_commit(&st->drain);
      mbar_wait(&st->drain, 0, p.timeout_ns, &zero, p.status);
    }
  } else {
    // ================= epilogue (warps 2 .. 2 + EPI_WARPS - 1) =================
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = (warp - 2) >> 2;  // the 256-column half of the tile this warp drains
    const int row_in_tile = (int)rank * C::A_ROWS + quarter * 32 + lane;
    const uint32_t tempty0 = PAIR ? mapa_shared(smem_u32(&st->tempty[0]), 0) : 0u;
    const uint32_t tempty1 = PAIR ? mapa_shared(smem_u32(&st->tempty[1]), 0) : 0u;
    int acc = 0;
    uint32_t acc_phase = 0;
    const bool c_stream = (p.hints & HINT_C_STREAM) != 0;
    const uint64_t pol_c = l2_policy_evict_first();
    auto store16 = [&](uint4* dst, const uint32_t* pk) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        if (c_stream)
          st_global_v4_hint(dst + q, v, pol_c);
        else
          dst[q] = v;
      }
    };
    for (int tile = unit; tile < total_tiles; tile += n_units) {
      const TileInfo ti = tile_info(tile, st->gt.prefix, G, p.n_tiles_n, p.n_major_rows);
      const Group gr = group_info(p, st->gt, ti.g);
      // a half tile (M = 128 pair MMA): this CTA's 64 rows, lanes 0-63 holding the first 128 of an MMA's
      // 256 columns and lanes 64-127 the other 128, in 128 TMEM columns per MMA
      const bool htile = PAIR && half_tile(p, gr, ti);
      const int r = ti.m * C::TILE_M + (htile ? (int)rank * 64 + (quarter & 1) * 32 + lane : row_in_tile);
      const int col_base = ti.nt * C::TILE_N + half * BN + (htile ? (quarter >> 1) * (BN / 2) : 0);
      const int n_ch = htile ? BN / 64 : BN / 32;  // 32-column chunks this warp drains
      const int c_row = gr.c_base + r;
      __nv_bfloat16* cbase = gr.c_sel ? p.C1 : p.C0;
      const int climit = gr.c_sel ? p.c1_limit : p.c0_limit;
      const bool valid = (r < gr.rows) && (c_row < climit);
      if (!mbar_wait(&st->tfull[acc], acc_phase, p.timeout_ns, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * C::TILE_N + half * (htile ? BN / 2 : BN));
      __nv_bfloat16* crow = cbase + (size_t)c_row * p.ldc;
      if (C::ACC_BUFS == 1 && EPI == EPI_SWIGLU) {
        // wide SwiGLU tile: accumulator columns 0-255 hold the gate and 256-511 the matching up columns of
        // the tile's 256 outputs; this warp forms outputs half * 128 .. + 127 as packed bf16 registers, hands
        // the accumulator back, then stores
        constexpr int NCH = SWIGLU_OUT / 32;
        uint32_t pk[NCH * 16];
        const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * SWIGLU_OUT);
#pragma unroll
        for (int c16 = 0; c16 < 2 * NCH; ++c16) {  // 16 outputs at a time (register pressure)
          float g[16], u[16];
          tmem_ld16(tbase + c16 * 16, g);
          tmem_ld16(tbase + BN + c16 * 16, u);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[c16 * 8 + i] = pack_bf16x2(silu_f32(g[2 * i]) * u[2 * i], silu_f32(g[2 * i + 1]) * u[2 * i + 1]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR)
            mbar_arrive_cluster(tempty0);
          else
            mbar_arrive(&st->tempty[0]);
        }
        acc_phase ^= 1u;
        if (valid) {
#pragma unroll
          for (int ch = 0; ch < NCH; ++ch) {
            const int col0 = ti.nt * BN + half * SWIGLU_OUT + ch * 32;
            if (col0 < p.N) store16(reinterpret_cast<uint4*>(crow + col0), pk + ch * 16);
          }
        }
        continue;
      }
      if (C::ACC_BUFS == 1 && EPI != EPI_SWIGLU) {
        // one accumulator (wide tiles): convert this warp's whole share into packed bf16 registers, hand
        // the accumulator back to the MMA, and only then store, so the next tile's MMAs overlap the stores
        // (a half tile's share is half as wide; each width has its own fully unrolled copy)
        auto drain = [&](auto n_chunks) {
          constexpr int NCH = decltype(n_chunks)::value;
          uint32_t pk[NCH * 16];
#pragma unroll
          for (int c16 = 0; c16 < 2 * NCH; ++c16) {  // 16 columns at a time (register pressure)
            float v[16];
            tmem_ld16(taddr + c16 * 16, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float a = v[2 * i], b = v[2 * i + 1];
              if (EPI == EPI_GELU) {
                a = gelu_tanh_f32(a);
                b = gelu_tanh_f32(b);
              }
              pk[c16 * 8 + i] = pack_bf16x2(a, b);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (PAIR)
              mbar_arrive_cluster(tempty0);
            else
              mbar_arrive(&st->tempty[0]);
          }
          if (valid) {
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
              const int col0 = col_base + ch * 32;
              if (col0 < p.N) store16(reinterpret_cast<uint4*>(crow + col0), pk + ch * 16);
            }
          }
        };
        if (htile)
          drain(std::integral_constant<int, BN / 64>{});
        else
          drain(std::integral_constant<int, BN / 32>{});
        acc_phase ^= 1u;
        continue;
      }
      if (EPI == EPI_SWIGLU) {
#pragma unroll 1
        for (int ch = 0; ch < SWIGLU_OUT / 32; ++ch) {
          const int col0 = ti.nt * SWIGLU_OUT + ch * 32;
          if (col0 >= p.N) break;  // same for the whole warp
          float g[32], u[32];
          tmem_ld32(taddr + ch * 32, g);
          tmem_ld32(taddr + SWIGLU_OUT + ch * 32, u);
          if (valid) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(silu_f32(g[2 * i]) * u[2 * i], silu_f32(g[2 * i + 1]) * u[2 * i + 1]);
            store16(reinterpret_cast<uint4*>(crow + col0), pk);
          }
        }
      }
#pragma unroll 1
      for (int ch = 0; ch < (EPI == EPI_SWIGLU ? 0 : n_ch); ++ch) {
        const int col0 = col_base + ch * 32;
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
          store16(reinterpret_cast<uint4*>(crow + col0), pk);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR)
          mbar_arrive_cluster(acc == 0 ? tempty0 : tempty1);
        else
          mbar_arrive(&st->tempty[acc]);
      }
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before();
  if (PAIR)
    cluster_sync_all();  // every MMA of the pair has landed; both CTAs are done with each other's memory
  else
    __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else
      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int EPI, bool PAIR, int ST, bool WIDE = false>
int launch_one(const CUtensorMap& a0, const CUtensorMap& a1, const CUtensorMap& b, const Params& p, int grid,
               cudaStream_t stream) {
  auto kfn = grouped_gemm_kernel<EPI, PAIR, ST, WIDE>;
  constexpr size_t bytes = smem_bytes<PAIR, ST, WIDE>();
  constexpr int NUM_THREADS = Cfg<PAIR, ST, WIDE>::THREADS;
  static_assert(bytes <= 232448, "shared memory per CTA");
  int rc = ensure_smem_attr((const void*)kfn, bytes);
  if (rc != MOE_OK) return rc;
  if (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kfn, a0, a1, b, p) != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    kfn<<<grid, NUM_THREADS, bytes, stream>>>(a0, a1, b, p);
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Everything one GEMM launch needs from the host.
struct GemmSpec {
  const void* a0;
  uint64_t a0_rows;
  uint32_t a0_box_rows;  // 128 for tiled A loads, 1 for row gathers
  const void* a1;  // may be null (then a0's map is passed twice)
  uint64_t a1_rows;
  const void* b;   // weights of the launch's group 0: [G, b_rows, K]
  uint64_t b_rows; // weight rows per group (0: N)
  Params p;
};

// Kernel variant.  CTA pairs (cta_group::2; 256 x 512 tiles by default, see wide_for) halve each CTA's
// shared-memory operand traffic and win when groups are large (compute-bound); with few rows per group the
// work is weight streaming and single CTAs (128 x 256 tiles, more weight bytes in flight per SM) win.
// MOE_GEMM_CTA=1 or =2 forces one of them.
bool choose_pair(long long rows, int groups) {
  bool pair = groups > 0 && rows / groups >= 256;
  const char* env = getenv("MOE_GEMM_CTA");
  if (env && env[0] == '1' && env[1] == '\0') pair = false;
  if (env && env[0] == '2' && env[1] == '\0') pair = true;
  return pair;
}

// Pipeline depth of the pair kernel (stages of 64-deep K slices in flight per CTA).  Deeper pipelines
// hide more load latency and win on short launches.  Launches of several TFLOP run for milliseconds under
// the board's power cap; there shallower ones win: with less prefetch the pairs that share A rows or
// weight tiles stay closer together in K, so more of their loads hit L2.  At 65536 tokens, d 7168,
// d_ff 2048 the first GEMM reads about 21 GB from DRAM with four stages of 256 x 256 tiles against about
// 50 GB with six, and with 256 x 512 tiles (whose stages hold twice the MMA work) 19 GB with three
// against 43 GB with four.  256 x 256 tiles: 6 short, 4 long; 256 x 512 tiles: 4 short, 3 long.
// MOE_GEMM_STAGES="s1,s2" (each 3 .. 6; 3 for wide tiles only) forces the depth of GEMM1, GEMM2.
constexpr double LONG_LAUNCH_FLOP = 4e12;

int stages_for(bool pair, bool wide, int which, double flop) {
  if (!pair) return 4;
  const bool long_launch = flop >= LONG_LAUNCH_FLOP;
  int st = wide ? (long_launch ? 3 : 4) : (long_launch ? 4 : 6);
  const char* env = getenv("MOE_GEMM_STAGES");
  if (env && env[0] && env[1] == ',' && env[2] && env[3] == '\0') {
    const char c = which == 1 ? env[0] : env[2];
    if (c == '3') st = 3;  // wide tiles only (others take 4)
    if (c == '4') st = 4;
    if (c == '5') st = 5;
    if (c == '6') st = 6;
  }
  return st;
}

// Groups of at most this many row tiles run column-tile-major; MOE_GEMM_NMAJOR=<rows> overrides (0: all
// row-tile-major).
int n_major_rows_for() {
  int r = 0;
  const char* env = getenv("MOE_GEMM_NMAJOR");
  if (env && env[0]) r = atoi(env);
  return r < 0 ? 0 : r;
}

// L2 prefetch distance in K blocks (0: off).  MOE_GEMM_PREFETCH=<blocks> overrides.
int prefetch_for() {
  int r = 0;
  const char* env = getenv("MOE_GEMM_PREFETCH");
  if (env && env[0]) r = atoi(env);
  return r < 0 ? 0 : (r > 64 ? 64 : r);
}

// L2 policies of a launch (HINT_* bits).  MOE_GEMM_HINTS=<0..7> overrides.
int hints_for() {
  int h = 0;
  const char* env = getenv("MOE_GEMM_HINTS");
  if (env && env[0] >= '0' && env[0] <= '7' && env[1] == '\0') h = env[0] - '0';
  return h;
}

// Wide pair tiles: 256 x 512 (GELU and plain epilogues; measured 7-10% faster than 256 x 256 at the
// prefill, skewed and slice sizes), or 256 x 256 outputs from 256 gate and 256 up accumulator columns
// (SwiGLU).  MOE_GEMM_WIDE=0 or =1 forces them off or on.
bool wide_for(bool pair, int epi) {
  bool wide = true;
  const char* env = getenv("MOE_GEMM_WIDE");
  if (env && env[0] == '1' && env[1] == '\0') wide = true;
  if (env && env[0] == '0' && env[1] == '\0') wide = false;
  (void)epi;
  return wide && pair;
}

// Half (M = 128) pair tiles for groups' last row tiles of at most 128 rows: pair launches with the GELU
// or plain epilogue and tiled A loads, where groups average at most 1024 rows.  A group's last 256-row
// tile is on average half padding, so they save up to half of that: measured 3.5% on the expert pair at
// the skewed workload (about 500 rows a group, 20% padding).  With long groups the saving is small and
// the shorter tiles pull the CTA pairs that share A blocks and weight tiles apart in K: at the prefill
// size (about 2000 rows a group) GEMM1 then read 34 GB from DRAM instead of 18 and the pair ran 4%
// slower.  MOE_GEMM_HALF=1 / =0 forces them on / off.
bool half_tiles_for(bool pair, int epi, const Params& p) {
  const long long groups = (long long)p.G_r + p.G_s;
  const long long rows = (long long)p.routed_rows * (p.G_r > 0 ? 1 : 0) + (long long)p.G_s * p.shared_rows;
  bool on = groups > 0 && rows <= 1024LL * groups;
  const char* env = getenv("MOE_GEMM_HALF");
  if (env && env[0] == '0' && env[1] == '\0') on = false;
  if (env && env[0] == '1' && env[1] == '\0') on = true;
  return on && pair && epi != EPI_SWIGLU && p.gather_rows == nullptr && p.tail_mode == TAIL_ALL;
}

template <int EPI>
int run_gemm(const GemmSpec& g, bool pair, int stages, int sms, long long tiles_upper, cudaStream_t s) {
  // rows per weight box: a pair CTA loads 128 (per column half); a single CTA 256, or 2 x 128 (gate,
  // up) for SwiGLU
  const uint32_t b_box = (pair || EPI == EPI_SWIGLU) ? (uint32_t)Cfg<true, 4>::B_HALF_ROWS
                                                     : (uint32_t)Cfg<false, 4>::B_HALF_ROWS;
  const bool wide = wide_for(pair, EPI);
  Params p = g.p;
  if (wide)  // 512 output columns a tile; SwiGLU: 256 outputs (256 gate + 256 up accumulator columns)
    p.n_tiles_n = EPI == EPI_SWIGLU ? (p.N + BN - 1) / BN
                                    : (p.N + Cfg<true, 4, true>::TILE_N - 1) / Cfg<true, 4, true>::TILE_N;
  p.half_tiles = half_tiles_for(pair, EPI, p) ? 1 : 0;
  CUtensorMap a0, a1, b;
  int rc;
  const uint64_t K = (uint64_t)g.p.K, N = g.b_rows ? g.b_rows : (uint64_t)g.p.N;
  if ((rc = encode_tmap_bf16(&a0, g.a0, 2, K, g.a0_rows, 1, BK, g.a0_box_rows ? g.a0_box_rows : 128)) != MOE_OK)
    return rc;
  if (g.a1) {
    if ((rc = encode_tmap_bf16(&a1, g.a1, 2, K, g.a1_rows, 1, BK, 128)) != MOE_OK) return rc;
  } else {
    a1 = a0;
  }
  if ((rc = encode_tmap_bf16(&b, g.b, 3, K, N, (uint64_t)(g.p.G_r + g.p.G_s), BK, b_box)) != MOE_OK) return rc;
  long long units = tiles_upper * p.n_tiles_n;
  if (pair) {
    long long pairs = units < sms / 2 ? units : sms / 2;
    if (wide) {
      if (stages == 3) return launch_one<EPI, true, 3, true>(a0, a1, b, p, (int)(2 * pairs), s);
      return launch_one<EPI, true, 4, true>(a0, a1, b, p, (int)(2 * pairs), s);
    }
    if (stages == 6) return launch_one<EPI, true, 6>(a0, a1, b, p, (int)(2 * pairs), s);
    if (stages == 5) return launch_one<EPI, true, 5>(a0, a1, b, p, (int)(2 * pairs), s);
    return launch_one<EPI, true, 4>(a0, a1, b, p, (int)(2 * pairs), s);
  }
  return launch_one<EPI, false, 4>(a0, a1, b, p, (int)(units < sms ? units : sms), s);
}

// Pair launches with each group's last rows split off: the CTA pairs take every group's whole
// 256-row blocks and single CTAs (128-row tiles) the rows past them, so a group's last block is
// padded to 128 rows instead of 256.  MOE_GEMM_TAILS=1 or =0 forces it on or off.
bool tails_for(bool pair) {
  bool on = false;
  const char* env = getenv("MOE_GEMM_TAILS");
  if (env && env[0] == '1' && env[1] == '\0') on = true;
  if (env && env[0] == '0' && env[1] == '\0') on = false;
  return on && pair;
}

template <int EPI>
int run_split(const GemmSpec& g, bool pair, int stages, int sms, long long tiles_upper, cudaStream_t s) {
  if (!tails_for(pair)) return run_gemm<EPI>(g, pair, stages, sms, tiles_upper, s);
  GemmSpec whole = g;
  whole.p.tail_mode = TAIL_WHOLE;
  whole.p.tail_unit = Cfg<true, 4>::TILE_M;
  int rc = run_gemm<EPI>(whole, true, stages, sms, tiles_upper, s);
  if (rc != MOE_OK) return rc;
  GemmSpec tail = g;
  tail.p.tail_mode = TAIL_ONLY;
  tail.p.tail_unit = Cfg<true, 4>::TILE_M;
  const long long groups = (long long)g.p.G_r + g.p.G_s;
  return run_gemm<EPI>(tail, false, 4, sms, groups * (Cfg<true, 4>::TILE_M / Cfg<false, 4>::TILE_M), s);
}

}  // namespace gffn
}  // namespace moe

using namespace moe;
using namespace moe::gffn;

extern "C" int moe_grouped_ffn(const moe_bf16* rows, const int32_t* offsets, int n_groups, int n_rows,
                               int expert_base, const moe_bf16* w1, const moe_bf16* w2, int d, int d_ff,
                               int activation, moe_bf16* h_scratch, moe_bf16* y, void* stream) {
  if (n_groups < 0 || n_rows < 0 || expert_base < 0 || d <= 0 || d_ff <= 0) return MOE_ERR_INVALID_ARG;
  if (activation != MOE_ACT_GELU_TANH && activation != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  const bool swiglu = activation == MOE_ACT_SWIGLU;
  const int w1_rows = swiglu ? 2 * d_ff : d_ff;  // SwiGLU: gate rows, then up rows
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
  unsigned int* status = status_ptr();
  if (!status) return MOE_ERR_CUDA;

  const bool pair = choose_pair(h_rows, n_groups);
  const int tile_m = pair ? Cfg<true, 4>::TILE_M : Cfg<false, 4>::TILE_M;
  const long long tiles_upper = identity ? (long long)n_groups * ((n_rows + tile_m - 1) / tile_m)
                                         : (n_rows + tile_m - 1) / tile_m + n_groups;

  Params p{};
  p.offsets = offsets;
  p.G_r = identity ? 0 : n_groups;
  p.G_s = identity ? n_groups : 0;
  p.routed_rows = n_rows;
  p.shared_rows = n_rows;
  p.a_sh_map = 0;
  p.timeout_ns = wait_timeout_ns();
  p.status = status;
  p.hints = hints_for();
  p.n_major_rows = n_major_rows_for();
  p.prefetch_kb = prefetch_for();

  GemmSpec g1{};
  g1.a0 = rows;
  g1.a0_rows = (uint64_t)n_rows;
  g1.b = reinterpret_cast<const __nv_bfloat16*>(w1) + (size_t)expert_base * w1_rows * d;
  g1.b_rows = (uint64_t)w1_rows;
  g1.p = p;
  g1.p.a_sh_base = 0;
  g1.p.a_sh_stride = 0;  // every shared group reads rows 0..n_rows-1
  g1.p.C0 = g1.p.C1 = reinterpret_cast<__nv_bfloat16*>(h_scratch);
  g1.p.c0_limit = g1.p.c1_limit = (int)h_rows;
  g1.p.c1_base = 0;
  g1.p.c1_stride = n_rows;
  g1.p.N = d_ff;
  g1.p.K = d;
  g1.p.n_tiles_n = swiglu ? (d_ff + SWIGLU_OUT - 1) / SWIGLU_OUT : (d_ff + BN - 1) / BN;
  g1.p.b_up_row = d_ff;
  g1.p.ldc = d_ff;
  const double flop = 2.0 * (double)h_rows * d * d_ff;  // GEMM2; GEMM1 has w1_rows / d_ff times as many
  rc = swiglu ? run_split<EPI_SWIGLU>(g1, pair, stages_for(pair, wide_for(pair, EPI_SWIGLU), 1, 2.0 * flop), sms, tiles_upper, s)
              : run_split<EPI_GELU>(g1, pair, stages_for(pair, wide_for(pair, EPI_GELU), 1, flop), sms, tiles_upper, s);
  if (rc != MOE_OK) return rc;

  GemmSpec g2{};
  g2.a0 = h_scratch;
  g2.a0_rows = (uint64_t)h_rows;
  g2.b = reinterpret_cast<const __nv_bfloat16*>(w2) + (size_t)expert_base * d * d_ff;
  g2.p = p;
  g2.p.a_sh_base = 0;
  g2.p.a_sh_stride = n_rows;
  g2.p.C0 = g2.p.C1 = reinterpret_cast<__nv_bfloat16*>(y);
  g2.p.c0_limit = g2.p.c1_limit = (int)h_rows;
  g2.p.c1_base = 0;
  g2.p.c1_stride = n_rows;
  g2.p.N = d;
  g2.p.K = d_ff;
  g2.p.n_tiles_n = (d + BN - 1) / BN;
  g2.p.ldc = d;
  return run_split<EPI_NONE>(g2, pair, stages_for(pair, wide_for(pair, EPI_NONE), 2, flop), sms, tiles_upper, s);
}

extern "C" int moe_experts_ffn(const moe_bf16* x, const moe_bf16* x_perm, const int32_t* row_token,
                               const int32_t* offsets, int T, int n_routed, int n_shared, int top_k,
                               const moe_bf16* w1, const moe_bf16* w2, int d, int d_ff, int activation,
                               moe_bf16* h_scratch, moe_bf16* y_perm, moe_bf16* y_shared, void* stream) {
  if (T < 0 || n_routed < 0 || n_shared < 0 || top_k < 1 || d <= 0 || d_ff <= 0) return MOE_ERR_INVALID_ARG;
  if (activation != MOE_ACT_GELU_TANH && activation != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  const bool swiglu = activation == MOE_ACT_SWIGLU;
  const int w1_rows = swiglu ? 2 * d_ff : d_ff;  // SwiGLU: gate rows, then up rows
  if (n_routed + n_shared > MOE_MAX_GROUPS) return MOE_ERR_UNSUPPORTED;
  if (d % 64 != 0 || d_ff % 64 != 0) return MOE_ERR_UNSUPPORTED;
  if (!w1 || !w2 || !h_scratch || !aligned16(w1) || !aligned16(w2) || !aligned16(h_scratch))
    return MOE_ERR_INVALID_ARG;
  const bool gather = (x_perm == nullptr);  // routed rows gathered from x through row_token
  if (n_routed > 0 && (!offsets || !y_perm || !aligned16(x_perm) || !aligned4(offsets) || !aligned16(y_perm)))
    return MOE_ERR_INVALID_ARG;
  if (n_routed > 0 && gather && (!x || !row_token || !aligned16(x) || !aligned4(row_token)))
    return MOE_ERR_INVALID_ARG;
  if (n_shared > 0 && (!x || !y_shared || !aligned16(x) || !aligned16(y_shared))) return MOE_ERR_INVALID_ARG;
  const long long R = (long long)T * top_k;
  const long long h_rows = R + (long long)n_shared * T;
  if (h_rows > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (T == 0 || n_routed + n_shared == 0) return MOE_OK;

  cudaStream_t s = (cudaStream_t)stream;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;
  unsigned int* status = status_ptr();
  if (!status) return MOE_ERR_CUDA;

  const int G = n_routed + n_shared;
  const bool pair = choose_pair(h_rows, G);
  const int tile_m = pair ? Cfg<true, 4>::TILE_M : Cfg<false, 4>::TILE_M;
  const long long tiles_upper =
      (R + tile_m - 1) / tile_m + n_routed + (long long)n_shared * ((T + tile_m - 1) / tile_m);

  Params p{};
  p.offsets = offsets;
  p.G_r = n_routed;
  p.G_s = n_shared;
  p.routed_rows = (int)R;
  p.shared_rows = T;
  p.timeout_ns = wait_timeout_ns();
  p.status = status;
  p.hints = hints_for();
  p.n_major_rows = n_major_rows_for();
  p.prefetch_kb = prefetch_for();

  // GEMM1: routed rows from x_perm, or gathered from x through row_token (map 0), shared rows from x
  // (map 1); H = [routed rows | shared s rows]
  GemmSpec g1{};
  const bool routed_gather = n_routed > 0 && gather;
  g1.a0 = (n_routed > 0 && !gather) ? (const void*)x_perm : (const void*)x;
  g1.a0_rows = (n_routed > 0 && !gather) ? (uint64_t)R : (uint64_t)T;
  g1.a0_box_rows = routed_gather ? 1u : 128u;  // gather4 loads take a tensor map whose box is one row
  g1.a1 = n_shared > 0 ? (const void*)x : nullptr;
  g1.a1_rows = (uint64_t)T;
  g1.b = w1;
  g1.b_rows = (uint64_t)w1_rows;
  g1.p = p;
  g1.p.gather_rows = routed_gather ? row_token : nullptr;
  g1.p.gather_limit = T;
  g1.p.a_sh_map = (n_routed > 0 || n_shared == 0) ? 1 : 0;
  g1.p.a_sh_base = 0;
  g1.p.a_sh_stride = 0;
  g1.p.C0 = g1.p.C1 = reinterpret_cast<__nv_bfloat16*>(h_scratch);
  g1.p.c0_limit = (int)R;
  g1.p.c1_base = (int)R;
  g1.p.c1_stride = T;
  g1.p.c1_limit = (int)h_rows;
  g1.p.N = d_ff;
  g1.p.K = d;
  g1.p.n_tiles_n = swiglu ? (d_ff + SWIGLU_OUT - 1) / SWIGLU_OUT : (d_ff + BN - 1) / BN;
  g1.p.b_up_row = d_ff;
  g1.p.ldc = d_ff;
  const double flop = 2.0 * (double)h_rows * d * d_ff;  // GEMM2; GEMM1 has w1_rows / d_ff times as many
  rc = swiglu ? run_split<EPI_SWIGLU>(g1, pair, stages_for(pair, wide_for(pair, EPI_SWIGLU), 1, 2.0 * flop), sms, tiles_upper, s)
              : run_split<EPI_GELU>(g1, pair, stages_for(pair, wide_for(pair, EPI_GELU), 1, flop), sms, tiles_upper, s);
  if (rc != MOE_OK) return rc;

  // GEMM2: all A rows from H (map 0); routed outputs to y_perm, shared outputs to y_shared
  GemmSpec g2{};
  g2.a0 = h_scratch;
  g2.a0_rows = (uint64_t)h_rows;
  g2.b = w2;
  g2.p = p;
  g2.p.a_sh_map = 0;
  g2.p.a_sh_base = (int)R;
  g2.p.a_sh_stride = T;
  g2.p.C0 = reinterpret_cast<__nv_bfloat16*>(y_perm);
  g2.p.c0_limit = (int)R;
  g2.p.C1 = reinterpret_cast<__nv_bfloat16*>(y_shared);
  g2.p.c1_base = 0;
  g2.p.c1_stride = T;
  g2.p.c1_limit = n_shared * T;
  g2.p.N = d;
  g2.p.K = d_ff;
  g2.p.n_tiles_n = (d + BN - 1) / BN;
  g2.p.ldc = d;
  return run_split<EPI_NONE>(g2, pair, stages_for(pair, wide_for(pair, EPI_NONE), 2, flop), sms, tiles_upper, s);
}
