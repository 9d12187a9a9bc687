// nvfp4.cu -- the routed experts in NVFP4 (W4A4): FP4 (E2M1) weights and
// activations in blocks of 16 values, each block with an FP8 (E4M3) scale, on
// the tcgen05 block-scaled tensor-core path ("Under the hood", "Quantization:
// BF16 vs NVFP4": FP4 weights and activations, group size 16, FP8 scale
// metadata, dynamic block scales, for Blackwell FP4 tensor cores).
//
// Recipe (every conversion rounds to nearest, ties to even, and saturates):
//   weights      one fp32 scale per matrix, g = amax|W| / (6 * 448); per block
//                s = E4M3(fl(amax_b / 6) / g); codes E2M1(fl(w * fl(1 / fl(s * g))))
//   activations  per block s = E4M3(fl(amax_b / 6)); codes E2M1(fl(x * fl(1 / s)))
// A block whose scale rounds to zero has all codes zero.
//
// Layouts (device memory, all caller-owned):
//   codes        [rows, K/2] bytes, K-major; byte j of a row holds values 2j
//                (bits 0-3) and 2j+1 (bits 4-7)
//   scales       atom-tiled: atoms of 128 rows x 64 values (4 scales a row),
//                512 bytes, the atoms of one 128-row block consecutive along K;
//                inside an atom the scale of (row r, block b) is at byte
//                (r % 32) * 16 + (r % 128 / 32) * 4 + b % 4 -- one 32 x 16-byte
//                block that tcgen05.cp copies to TMEM as the MMA reads it
//   routed rows  each expert's rows start at a multiple of 128 ("padded"
//                offsets), so every 128-row tile owns whole scale atoms
//
// Kernels:
//   weight_amax / weight_quant / weight_scale   weights, once
//   dispatch_quant   x rows quantized once per token and written to the padded
//                    rows of its k experts (the FP4 dispatch)
//   fp4_gemm_kernel<EPI, TN, PAIR>   persistent grouped GEMM, one CTA per 128 x 256
//                    tile (128 x 128 where N is not a multiple of 256; or, as an
//                    option, a CTA pair per 256 x TN tile):
//                    warp 0 loads code tiles (TMA, 128-byte swizzle) and scale
//                    atoms (bulk copies), warp 1 copies the scales to TMEM
//                    (tcgen05.cp) and issues tcgen05.mma kind::mxf4nvf4 with
//                    block16 scales, warps 2-9 drain the accumulator: x the
//                    weight matrix's g, then GELU and FP4 re-quantization
//                    (GEMM1) or bf16 (GEMM2)
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace fp4 {

constexpr int ATOM_ROWS = 128;
constexpr int ATOM_K = 64;
constexpr int ATOM_BYTES = 512;
constexpr float E2M1_MAX = 6.0f;
constexpr float E4M3_MAX = 448.0f;

// Byte offset of the scale of (row r, 16-value block b) in the atom-tiled
// layout of a matrix with K values per row.
__host__ __device__ __forceinline__ size_t sf_offset(long long r, int b, int K) {
  const long long atoms_k = K / ATOM_K;
  return (size_t)(((r / ATOM_ROWS) * atoms_k + (b >> 2)) * ATOM_BYTES + (r & 31) * 16 + ((r & 127) >> 5) * 4 +
                  (b & 3));
}

// Nearest E2M1 value (ties to the even code), saturating at +-6; no negative zero.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  const float m = fabsf(v);
  uint32_t c = m <= 0.25f ? 0u
               : m < 0.75f ? 1u
               : m <= 1.25f ? 2u
               : m < 1.75f ? 3u
               : m <= 2.5f ? 4u
               : m < 3.5f ? 5u
               : m <= 5.0f ? 6u
                           : 7u;
  if (c != 0u && v < 0.0f) c |= 8u;
  return c;
}

__device__ __forceinline__ uint32_t e4m3_code(float s) {  // s >= 0
  return (uint32_t)__nv_cvt_float_to_fp8(s, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  return e == 0u ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// 16 values with one scale (already chosen): packed codes, 4 bits each, value i at bits 4i of word i/8.
// A code is the E2M1 rounding of the value over its scale, the quotient correctly rounded to fp32
// (a product with the scale's reciprocal would land past an exact tie, e.g. 1.25 * 0.9375 / 0.9375).
__device__ __forceinline__ uint2 pack16(const float* v, float denom) {
  uint32_t w[2] = {0u, 0u};
  if (denom > 0.0f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i >> 3] |= e2m1_code(__fdiv_rn(v[i], denom)) << (4 * (i & 7));
  }
  return make_uint2(w[0], w[1]);
}

// The same code, E2M1(fl32(v / s)), for a scale s > 0 that is an E4M3 value, decided without the
// division.  Rounding is monotone, so fl32(q) against an E2M1 midpoint t is a test on q itself: every
// midpoint has an even last mantissa bit, so a quotient halfway between t and a neighbour rounds to t,
//   fl32(q) <= t  <=>  q <= t + h      fl32(q) < t  <=>  q < t - h      (h: half the fp32 spacing at t),
// and with q = |v| / s these read |v| - t s <= h s and |v| - t s < -h s.  h s is exact (a power of two
// times s), and the fma rounds |v| - t s once; wherever that difference is within a few of its own
// spacings of h s, |v| and t s are within a factor of two of each other, so it is exact (Sterbenz) and
// the comparison decides as over the reals.  (Checked against the rounded quotient for every positive
// E4M3 scale at and around each midpoint.)  A NaN gives code 7, as the division form does.
__device__ __forceinline__ uint32_t e2m1_code_of_quotient(float v, float s) {
  const float a = fabsf(v);
  const int n = (int)(fmaf(-0.25f, s, a) <= 0x1p-26f * s) + (int)(fmaf(-0.75f, s, a) < -0x1p-25f * s) +
                (int)(fmaf(-1.25f, s, a) <= 0x1p-24f * s) + (int)(fmaf(-1.75f, s, a) < -0x1p-24f * s) +
                (int)(fmaf(-2.5f, s, a) <= 0x1p-23f * s) + (int)(fmaf(-3.5f, s, a) < -0x1p-23f * s) +
                (int)(fmaf(-5.0f, s, a) <= 0x1p-22f * s);
  uint32_t c = 7u - (uint32_t)n;  // the midpoints fl32(q) has passed
  if (c != 0u && v < 0.0f) c |= 8u;
  return c;
}

// Activation block: dynamic scale, no tensor scale.
__device__ __forceinline__ uint2 quant16_act(const float* v, uint32_t& sf) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  sf = e4m3_code(__fdiv_rn(amax, E2M1_MAX));
  const float s = e4m3_value(sf);
  uint32_t w[2] = {0u, 0u};
  if (s > 0.0f) {
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i >> 3] |= e2m1_code_of_quotient(v[i], s) << (4 * (i & 7));
  }
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ void bf16x8_to_float(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// GELU, tanh form, written through the identity (1 + tanh z) / 2 = 1 / (1 + e^-2z):
// u / (1 + e^(-2 k0 (u + k1 u^3))).  No cancellation near 0, one exp and one
// approximate division, so the result is within a few fp32 ulps -- it decides FP4
// codes, so it must stay close to the exact value (the tanh.approx of the bf16 path
// would move ~0.1% of codes).  For very negative u the denominator overflows and
// the quotient is -0.
__device__ __forceinline__ float gelu_tanh_accurate(float u) {
  const float k0x2 = 1.5957691216057308f;  // 2 sqrt(2/pi)
  const float k1 = 0.044715f;
  const float z = k0x2 * fmaf(k1 * u, u * u, u);
  return __fdividef(u, 1.0f + __expf(-z));
}

// ---------------------------------------------------------------------------
// weights
// ---------------------------------------------------------------------------
__global__ void weight_amax_kernel(const uint4* __restrict__ w, long long vec_per_matrix,
                                   unsigned int* __restrict__ amax_bits) {
  const int g = blockIdx.y;
  const uint4* src = w + (size_t)g * vec_per_matrix;
  float m = 0.0f;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < vec_per_matrix;
       i += (long long)gridDim.x * blockDim.x) {
    float f[8];
    bf16x8_to_float(__ldg(src + i), f);
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(f[j]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + g, __float_as_uint(m));  // m >= 0: bits order as values
}

// One thread per 16-value block of one row of one matrix.
__global__ void weight_quant_kernel(const uint4* __restrict__ w, int G, int N, int K,
                                    const unsigned int* __restrict__ amax_bits, uint8_t* __restrict__ q,
                                    uint8_t* __restrict__ sf) {
  const int nb = K / 16;
  const long long units = (long long)G * N * nb;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const int b = (int)(u % nb);
    const long long rowg = u / nb;  // g * N + n
    const int g = (int)(rowg / N);
    const int n = (int)(rowg - (long long)g * N);
    const float gs = __fdiv_rn(__uint_as_float(amax_bits[g]), E2M1_MAX * E4M3_MAX);
    float v[16];
    const uint4* src = w + rowg * (K / 8) + 2 * b;
    bf16x8_to_float(__ldg(src), v);
    bf16x8_to_float(__ldg(src + 1), v + 8);
    uint32_t s = 0u;
    float denom = 0.0f;
    if (gs > 0.0f) {
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
      s = e4m3_code(__fdiv_rn(__fdiv_rn(amax, E2M1_MAX), gs));
      denom = __fmul_rn(e4m3_value(s), gs);
    }
    *reinterpret_cast<uint2*>(q + rowg * (K / 2) + 8 * b) = pack16(v, denom);
    sf[(size_t)g * N * nb + sf_offset(n, b, K)] = (uint8_t)s;
  }
}

__global__ void weight_scale_kernel(unsigned int* amax_bits_to_scale, int G) {
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  if (g < G) {
    const float s = __fdiv_rn(__uint_as_float(amax_bits_to_scale[g]), E2M1_MAX * E4M3_MAX);
    amax_bits_to_scale[g] = __float_as_uint(s);
  }
}

// ---------------------------------------------------------------------------
// dispatch: quantize each token's x once, write it to its k padded rows
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) dispatch_quant_kernel(const uint4* __restrict__ x,
                                                             const int32_t* __restrict__ topk_idx,
                                                             const int32_t* __restrict__ token_row,
                                                             const int32_t* __restrict__ offsets, int T, int d,
                                                             int n_routed, int k, long long rows_cap,
                                                             uint8_t* __restrict__ xq, uint8_t* __restrict__ xsf,
                                                             int32_t* __restrict__ token_row_pad,
                                                             int32_t* __restrict__ offsets_pad) {
  __shared__ int off[MOE_MAX_ROUTED + 1], offp[MOE_MAX_ROUTED + 1];
  __shared__ int wsum[8];
  // padded offsets: every expert's rows start at a multiple of 128
  {
    const int e = threadIdx.x;
    int n = 0;
    if (e < n_routed) {
      off[e] = offsets[e];
      n = offsets[e + 1] - offsets[e];
      n = n < 0 ? 0 : n;
    }
    if (e == n_routed - 1) off[n_routed] = offsets[n_routed];
    int v = (n + ATOM_ROWS - 1) / ATOM_ROWS * ATOM_ROWS;
    const int own = v;
    const int lane = e & 31, w = e >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    if (lane == 31) wsum[w] = v;
    __syncthreads();
    int before = 0;
    for (int i = 0; i < w; ++i) before += wsum[i];
    if (e < n_routed) offp[e] = before + v - own;
    if (e == n_routed - 1) offp[n_routed] = before + v;
    __syncthreads();
    if (blockIdx.x == 0 && e < n_routed) offsets_pad[e] = offp[e];
    if (blockIdx.x == 0 && e == 0) offsets_pad[n_routed] = offp[n_routed];  // n_routed may equal the block size
  }
  const int nb = d / 16;
  const long long units = (long long)T * nb;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(u / nb);
    const int b = (int)(u - (long long)t * nb);
    float v[16];
    const uint4* src = x + (size_t)t * (d / 8) + 2 * b;
    bf16x8_to_float(__ldg(src), v);
    bf16x8_to_float(__ldg(src + 1), v + 8);
    uint32_t s;
    const uint2 packed = quant16_act(v, s);
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(topk_idx + (size_t)t * k + j);
      const int r = __ldg(token_row + (size_t)t * k + j);
      long long rp = -1;
      if (e >= 0 && e < n_routed && r >= off[e] && r < off[e + 1]) rp = (long long)r - off[e] + offp[e];
      if (rp >= rows_cap) rp = -1;
      if (b == 0) token_row_pad[(size_t)t * k + j] = (int32_t)rp;
      if (rp < 0) continue;
      *reinterpret_cast<uint2*>(xq + rp * (d / 2) + 8 * b) = packed;
      xsf[sf_offset(rp, b, d)] = (uint8_t)s;
    }
  }
}

// ---------------------------------------------------------------------------
// grouped GEMM on NVFP4 operands
// ---------------------------------------------------------------------------
constexpr int EPI_WARPS = 8;     // two per TMEM lane quarter, one per half of the tile's output columns
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;  // producer warp, MMA warp, epilogue warps
constexpr int TM = 128;           // rows per CTA
constexpr int ROW_BYTES = 128;    // code bytes per row per stage: 256 values
constexpr int KV_STAGE = 256;     // values along K per stage
constexpr int A_BYTES = TM * ROW_BYTES;
constexpr int SF_BYTES = (KV_STAGE / ATOM_K) * ATOM_BYTES;  // 4 atoms = 2 KB per 128 rows per stage
constexpr int SF_ROW = 256;       // scale atoms seen as rows of 256 bytes by the pair's TMA loads
constexpr uint32_t TMEM_COLS = 512;

// Tile shapes.
//   TN = 256 (default where N allows): twice the MMA work per stage of TN = 128; two 256-column
//     accumulators would leave no TMEM for the scales, so one accumulator, which the epilogue hands back
//     as soon as it has read it, and four 54 KB stages.
//   TN = 128: one CTA per 128 x 128 tile, two accumulators, six 36 KB stages.
//   PAIR: a cluster of two CTAs per 256 x TN tile with tcgen05.mma.cta_group::2.  CTA rank r holds A rows
//     r*128.. and weight rows r*TN/2.. of the tile (SwiGLU: rank 0 the 128 gate rows, rank 1 the 128
//     matching up rows), its A rows' scales and the scales of all TN weight rows (the MMA reads SFB from
//     both CTAs' TMEM).  256 x 256: 38 KB per stage per CTA for the MMA work of a 54 KB single-CTA stage,
//     five stages, one accumulator; 256 x 128: 28 KB for that of a 36 KB stage, seven stages, two.
template <int TN_, bool PAIR_ = false>
struct FCfg {
  static constexpr int TN = TN_;
  static constexpr bool PAIR = PAIR_;
  static_assert(TN == 128 || TN == 256, "tile widths");
  static constexpr int TILE_M = PAIR ? 2 * TM : TM;  // rows per tile (per pair, or per CTA)
  static constexpr int B_ROWS = PAIR ? TN / 2 : TN;   // weight rows one CTA holds
  static constexpr int ACC_BUFS = TN == 256 ? 1 : 2;
  static constexpr int STAGES = PAIR ? (TN == 256 ? 5 : 7) : (TN == 256 ? 4 : 6);
  static constexpr int B_BYTES = B_ROWS * ROW_BYTES;
  static constexpr int SFB_BYTES = (TN / ATOM_ROWS) * SF_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SF_BYTES + SFB_BYTES;
  static constexpr uint32_t STAGE_TX = (uint32_t)STAGE_BYTES * (PAIR ? 2u : 1u);  // on the (leader's) barrier
  // A stage's scales in the columns past the accumulators: 16 for A (4 K-chunks x 4), then TN/8 for the
  // weights (4 K-chunks x TN/32).  Every stage reuses them: tcgen05 operations issued by one thread run in
  // order, so a stage's copies land after the previous stage's MMAs have read them.  (Rotating buffers,
  // one a stage, measured no faster.)
  static constexpr uint32_t SFA_COL = (uint32_t)(ACC_BUFS * TN);
  static constexpr uint32_t SFB_COL = SFA_COL + 16;
  static_assert(SFB_COL + TN / 8 <= TMEM_COLS, "TMEM columns");
};
constexpr int EPI_GELU_FP4 = 0;   // GEMM1: x g1, GELU, FP4 out (the next GEMM's A)
constexpr int EPI_BF16 = 1;       // GEMM2: x g2, bf16 out
constexpr int EPI_SWIGLU_FP4 = 2; // GEMM1 of SwiGLU experts (256-wide tiles: 128 gate + the 128 matching up
                                  // columns), silu(g1 gate) * (g1 up), FP4 out

struct Params {
  const int* offsets_pad;  // [G + 1] group row starts, multiples of 128
  int G;
  long long rows_cap;      // rows of A / of the outputs
  const uint8_t* a_sf;     // atom-tiled scales of A [rows_cap, K]
  const uint8_t* b_sf;     // atom-tiled scales of the weights, per group b_sf_stride bytes
  long long b_sf_stride;
  const float* gscale;     // [G] weight tensor scales
  int N, K, n_tiles_n;    // N: output columns
  int b_up_row;            // EPI_SWIGLU_FP4: first weight row of the up projection (= N)
  uint8_t* out_q;          // EPI_GELU_FP4: codes [rows_cap, N/2] and atom-tiled scales
  uint8_t* out_sf;
  __nv_bfloat16* out;      // EPI_BF16: [rows_cap, N], or [out_rows, N] through offsets_out
  const int* offsets_out;  // nullable: the groups' real rows (offsets_out[e+1] - offsets_out[e] of them); with
                           // EPI_BF16 group e's row i goes to row offsets_out[e] + i.  Rows past a group's
                           // real count are neither loaded nor (FP4 epilogues) written
  long long out_rows;
  uint64_t timeout_ns;
  unsigned int* status;
};

struct Tables {
  int off[MOE_MAX_ROUTED + 1];
  int prefix[MOE_MAX_ROUTED + 1];  // row tiles of groups < g
  int off_out[MOE_MAX_ROUTED + 1];
};

template <int STAGES>
struct SmemTail {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  Tables t;
};

template <int TN, bool PAIR = false>
constexpr size_t smem_bytes() {
  using C = FCfg<TN, PAIR>;
  return 1024 + (size_t)C::STAGES * C::STAGE_BYTES + sizeof(SmemTail<C::STAGES>);
}
static_assert(smem_bytes<128>() <= 232448 && smem_bytes<256>() <= 232448 && smem_bytes<128, true>() <= 232448 &&
                  smem_bytes<256, true>() <= 232448,
              "shared memory per CTA");

// tmA / tmA32: A codes in 128-row / 32-row boxes; tmB: weight codes, boxes of FCfg::B_ROWS rows (128 for
// SwiGLU); tmSA / tmSB (pair tiles only): the A / weight scale atoms as rows of 256 bytes, 8-row boxes.
template <int EPI, int TN, bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA32,
                    const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmSA,
                    const __grid_constant__ CUtensorMap tmSB, const Params p) {
  using C = FCfg<TN, PAIR>;
  static_assert(EPI != EPI_SWIGLU_FP4 || TN == 256, "SwiGLU tiles hold gate and up columns side by side");
  constexpr int OUT_W = EPI == EPI_SWIGLU_FP4 ? TN / 2 : TN;  // output columns per tile
  constexpr int STAGES = C::STAGES;
  constexpr int B_BYTES = C::B_BYTES;
  constexpr int SFB_BYTES = C::SFB_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sSFA = sB + STAGES * B_BYTES;
  uint8_t* sSFB = sSFA + STAGES * SF_BYTES;
  SmemTail<STAGES>* st = reinterpret_cast<SmemTail<STAGES>*>(sSFB + STAGES * SFB_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // pair or CTA index
  const int n_units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&st->full[s], 1);
      mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&st->tfull[a], 1);
      mbar_init(&st->tempty[a], EPI_WARPS * (PAIR ? 2 : 1));  // one arrival per epilogue warp (of both CTAs)
    }
    mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    fence_barrier_init();
  }
  // group tables: clamped padded offsets and the row-tile prefix
  for (int i = tid; i <= p.G; i += NUM_THREADS) {
    long long v = p.offsets_pad[i];
    v = v < 0 ? 0 : (v > p.rows_cap ? p.rows_cap : v);
    st->t.off[i] = (int)v;
    if (p.offsets_out != nullptr) {
      long long o = p.offsets_out[i];
      st->t.off_out[i] = (int)(o < 0 ? 0 : (o > p.out_rows ? p.out_rows : o));
    }
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int g = 0; g < p.G; ++g) {
      st->t.prefix[g] = run;
      const int rows = st->t.off[g + 1] - st->t.off[g];
      run += rows > 0 ? (rows + C::TILE_M - 1) / C::TILE_M : 0;
    }
    st->t.prefix[p.G] = run;
  }
  __syncthreads();
  const int total_tiles = st->t.prefix[p.G] * p.n_tiles_n;
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
  const int num_kb = p.K / KV_STAGE;
  const int atoms_k = p.K / ATOM_K;
  volatile int* abort_flag = &st->abort_flag;

  auto tile_of = [&](int tile, int& g, int& m, int& nt) {
    const int mt = tile / p.n_tiles_n;
    nt = tile - mt * p.n_tiles_n;
    int lo = 0, hi = p.G;  // largest g with prefix[g] <= mt
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (st->t.prefix[mid] <= mt)
        lo = mid;
      else
        hi = mid;
    }
    g = lo;
    m = mt - st->t.prefix[lo];
  };

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      if (PAIR) {
        tma_prefetch_desc(&tmSA);
        tma_prefetch_desc(&tmSB);
      } else {
        tma_prefetch_desc(&tmA32);
      }
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int tile = unit; tile < total_tiles && ok; tile += n_units) {
        int g, m, nt;
        tile_of(tile, g, m, nt);
        const int a_row = st->t.off[g] + m * C::TILE_M + (int)rank * TM;
        const int n0 = nt * OUT_W;  // first output column; for SwiGLU also the first gate row
        // A rows to load: the group's real rows in this tile, in 32-row boxes (few-row groups at small
        // T would otherwise fill three quarters of every A stage with padding)
        int a_boxes = 4;
        if (!PAIR && p.offsets_out != nullptr) {
          const int real = st->t.off_out[g + 1] - st->t.off_out[g] - m * TM;
          a_boxes = real >= TM ? 4 : (real <= 0 ? 1 : (real + 31) / 32);
        }
        const uint32_t tx = C::STAGE_TX - (uint32_t)(4 - a_boxes) * (A_BYTES / 4);
        const uint8_t* sfa = p.a_sf + ((size_t)(a_row / ATOM_ROWS) * atoms_k) * ATOM_BYTES;
        const uint8_t* sfb_g = p.b_sf + (size_t)g * p.b_sf_stride;
        // pair tiles: the scale atoms' rows of 256 bytes (every offset below is a multiple of 2 KB)
        const int sfa_row = (int)(((long long)(a_row / ATOM_ROWS) * atoms_k * ATOM_BYTES) / SF_ROW);
        const int sfb_row =
            (int)(((long long)g * p.b_sf_stride + (long long)(n0 / ATOM_ROWS) * atoms_k * ATOM_BYTES) / SF_ROW);
        const int sfb_up_row = (int)(((long long)g * p.b_sf_stride +
                                      (long long)((p.b_up_row + n0) / ATOM_ROWS) * atoms_k * ATOM_BYTES) /
                                     SF_ROW);
        for (int kb = 0; kb < num_kb; ++kb) {
          ok = mbar_wait(&st->empty[stage], phase ^ 1u, p.timeout_ns, abort_flag, p.status);
          if (!ok) break;
          uint64_t* bar = &st->full[stage];
          if (PAIR) {
            // both CTAs' copies complete on the leader's barrier, which expects the pair's bytes
            if (leader) mbar_arrive_expect_tx(bar, C::STAGE_TX);
            const int b_row = EPI == EPI_SWIGLU_FP4 ? (rank == 0u ? n0 : p.b_up_row + n0) : n0 + (int)rank * C::B_ROWS;
            tma_load_2d_pair(sA + stage * A_BYTES, &tmA, bar, kb * ROW_BYTES, a_row);
            tma_load_3d_pair(sB + stage * B_BYTES, &tmB, bar, kb * ROW_BYTES, b_row, g);
            tma_load_2d_pair(sSFA + stage * SF_BYTES, &tmSA, bar, 0, sfa_row + kb * (SF_BYTES / SF_ROW));
#pragma unroll
            for (int rb = 0; rb < TN / ATOM_ROWS; ++rb) {  // the weight rows' 128-row blocks, in every CTA
              const int blk_row = rb == 0 ? sfb_row : (EPI == EPI_SWIGLU_FP4 ? sfb_up_row : sfb_row + atoms_k * 2);
              tma_load_2d_pair(sSFB + stage * SFB_BYTES + rb * SF_BYTES, &tmSB, bar, 0,
                               blk_row + kb * (SF_BYTES / SF_ROW));
            }
          } else {
            mbar_arrive_expect_tx(bar, tx);
            if (a_boxes == 4) {
              tma_load_2d(sA + stage * A_BYTES, &tmA, bar, kb * ROW_BYTES, a_row);
            } else {
              for (int i = 0; i < a_boxes; ++i)
                tma_load_2d(sA + stage * A_BYTES + i * (A_BYTES / 4), &tmA32, bar, kb * ROW_BYTES, a_row + 32 * i);
            }
            if (EPI == EPI_SWIGLU_FP4) {  // gate rows, then the matching up rows (128-row boxes)
              tma_load_3d(sB + stage * B_BYTES, &tmB, bar, kb * ROW_BYTES, n0, g);
              tma_load_3d(sB + stage * B_BYTES + B_BYTES / 2, &tmB, bar, kb * ROW_BYTES, p.b_up_row + n0, g);
            } else {
              tma_load_3d(sB + stage * B_BYTES, &tmB, bar, kb * ROW_BYTES, n0, g);
            }
            bulk_load(sSFA + stage * SF_BYTES, sfa + (size_t)kb * SF_BYTES, SF_BYTES, bar);
#pragma unroll
            for (int rb = 0; rb < TN / ATOM_ROWS; ++rb) {  // the weight rows' 128-row blocks
              const int blk =
                  (EPI == EPI_SWIGLU_FP4 && rb == 1) ? (p.b_up_row + n0) / ATOM_ROWS : n0 / ATOM_ROWS + rb;
              bulk_load(sSFB + stage * SFB_BYTES + rb * SF_BYTES,
                        sfb_g + ((size_t)blk * atoms_k) * ATOM_BYTES + (size_t)kb * SF_BYTES, SF_BYTES, bar);
            }
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && !PAIR) {
        // wind down: let the copies already issued land before the CTA exits
        int zero = 0;
        for (long i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
          mbar_wait(&st->full[i % STAGES], (uint32_t)((i / STAGES) & 1), p.timeout_ns, &zero, p.status);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = make_idesc_nvf4(C::TILE_M, TN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = unit; tile < total_tiles && ok; tile += n_units) {
        if (!mbar_wait(&st->tempty[acc], acc_phase ^ 1u, p.timeout_ns, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&st->full[stage], phase, p.timeout_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
          const uint32_t sfa_addr = smem_u32(sSFA + stage * SF_BYTES);
          const uint32_t sfb_addr = smem_u32(sSFB + stage * SFB_BYTES);
          const uint32_t sfa_col = tmem_base + C::SFA_COL, sfb_col = tmem_base + C::SFB_COL;
          // K-chunk j's scales: A's 128 rows in 4 columns; the weights' TN rows in TN/32 columns, 4 per
          // 128-row block (the layout the MMA reads: row r at lane r % 32, column r / 32)
#pragma unroll
          for (int j = 0; j < KV_STAGE / ATOM_K; ++j) {
            if (PAIR)
              tmem_cp_sf_pair(sfa_col + 4 * j, make_desc_sf(sfa_addr + j * ATOM_BYTES));
            else
              tmem_cp_sf(sfa_col + 4 * j, make_desc_sf(sfa_addr + j * ATOM_BYTES));
#pragma unroll
            for (int rb = 0; rb < TN / ATOM_ROWS; ++rb) {
              const uint64_t d = make_desc_sf(sfb_addr + rb * SF_BYTES + j * ATOM_BYTES);
              if (PAIR)
                tmem_cp_sf_pair(sfb_col + (TN / 32) * j + 4 * rb, d);
              else
                tmem_cp_sf(sfb_col + (TN / 32) * j + 4 * rb, d);
            }
          }
#pragma unroll
          for (int j = 0; j < KV_STAGE / ATOM_K; ++j) {
            const uint64_t ad = make_desc_sw128(a_addr + j * 32), bd = make_desc_sw128(b_addr + j * 32);
            const uint32_t sfa_t = sfa_col + 4 * j, sfb_t = sfb_col + (TN / 32) * j;
            if (PAIR)
              mma_nvf4_ss_pair(d_tmem, ad, bd, idesc, sfa_t, sfb_t, (kb | j) != 0 ? 1u : 0u);
            else
              mma_nvf4_ss(d_tmem, ad, bd, idesc, sfa_t, sfb_t, (kb | j) != 0 ? 1u : 0u);
          }
          if (PAIR)
            mma_commit_pair(&st->empty[stage], 0x3);
          else
            mma_commit(&st->empty[stage]);
          if (++stage == STAGES) {
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
    // epilogue, EPI_WARPS warps: warp w reads TMEM lanes 32 * (w % 4) .. +31 (one tile row per thread)
    // and drains the column half (w - 2) / 4 of the tile's outputs.  It reads its whole share of the
    // accumulator, hands the accumulator back to the MMA, and only then computes and stores: the next
    // tile's MMAs overlap the math and the stores, and the hand-back never waits for stores to land.
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int W = OUT_W / 2;                            // output columns per warp
    constexpr int NV = EPI == EPI_SWIGLU_FP4 ? 2 * W : W;  // accumulator columns per thread (gate, up)
    const uint32_t tempty0 = PAIR ? mapa_shared(smem_u32(&st->tempty[0]), 0) : 0u;
    const uint32_t tempty1 = PAIR ? mapa_shared(smem_u32(&st->tempty[1]), 0) : 0u;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = unit; tile < total_tiles; tile += n_units) {
      int g, m, nt;
      tile_of(tile, g, m, nt);
      const int in_group = m * C::TILE_M + (int)rank * TM + quarter * 32 + lane;  // row within the group
      const long long r = (long long)st->t.off[g] + in_group;
      // a pair tile's second half may run past the group's padded rows (into the next group's)
      bool valid = r < p.rows_cap && in_group < st->t.off[g + 1] - st->t.off[g];
      long long r_out = r;  // output row
      if (p.offsets_out != nullptr) {
        // only the groups' real rows are meaningful (and, with EPI_BF16, written to the unpadded rows)
        const int real = st->t.off_out[g + 1] - st->t.off_out[g];
        if (EPI == EPI_BF16) {
          r_out = (long long)st->t.off_out[g] + in_group;
          valid = in_group < real && r_out < p.out_rows;
        } else {
          valid = valid && in_group < real;
        }
      }
      const float gs = __ldg(p.gscale + g);
      if (!mbar_wait(&st->tfull[acc], acc_phase, p.timeout_ns, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * TN);
      float v[NV];
      if (EPI == EPI_SWIGLU_FP4) {
        tmem_ld64(taddr + half * W, v);              // gate columns
        tmem_ld64(taddr + OUT_W + half * W, v + W);  // the matching up columns
      } else {
#pragma unroll
        for (int c = 0; c < W; c += 64) tmem_ld64(taddr + half * W + c, v + c);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // the peer's hand-back orders no memory writes, so it need not wait for this warp's stores of
        // the previous tile to land (a releasing arrive there cost 8% on a prefill-shaped slice)
        if (PAIR)
          mbar_arrive_cluster_relaxed(acc == 0 ? tempty0 : tempty1);
        else
          mbar_arrive(&st->tempty[acc]);
      }
      if (++acc == C::ACC_BUFS) {
        acc = 0;
        acc_phase ^= 1u;
      }
      if (!valid) continue;
#pragma unroll
      for (int ch = 0; ch < W / 32; ++ch) {
        const int col0 = nt * OUT_W + half * W + ch * 32;
        if (col0 >= p.N) break;  // same for the whole warp
        float* x = v + ch * 32;
        if (EPI == EPI_SWIGLU_FP4) {
          const float* u = v + W + ch * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float gate = __fmul_rn(x[i], gs);
            x[i] = __fmul_rn(__fdividef(gate, 1.0f + __expf(-gate)), __fmul_rn(u[i], gs));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = __fmul_rn(x[i], gs);
          if (EPI == EPI_GELU_FP4) {
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = gelu_tanh_accurate(x[i]);
          }
        }
        if (EPI != EPI_BF16) {
          uint32_t s0, s1;
          const uint2 q0 = quant16_act(x, s0);
          const uint2 q1 = quant16_act(x + 16, s1);
          *reinterpret_cast<uint4*>(p.out_q + r * (p.N / 2) + col0 / 2) = make_uint4(q0.x, q0.y, q1.x, q1.y);
          const size_t so = sf_offset(r, col0 / 16, p.N);  // the two blocks share an atom line (b even)
          p.out_sf[so] = (uint8_t)s0;
          p.out_sf[so + 1] = (uint8_t)s1;
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
          uint4* dst = reinterpret_cast<uint4*>(p.out + r_out * p.N + col0);
#pragma unroll
          for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
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

template <int EPI, int TN, bool PAIR = false>
int launch_fp4(const CUtensorMap& ta, const CUtensorMap& ta32, const CUtensorMap& tb, const CUtensorMap& tsa,
               const CUtensorMap& tsb, const Params& p, int grid, cudaStream_t s) {
  auto kfn = fp4_gemm_kernel<EPI, TN, PAIR>;
  constexpr size_t bytes = smem_bytes<TN, PAIR>();
  const int rc = ensure_smem_attr((const void*)kfn, bytes);
  if (rc != MOE_OK) return rc;
  if (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = bytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kfn, ta, ta32, tb, tsa, tsb, p) != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    kfn<<<grid, NUM_THREADS, bytes, s>>>(ta, ta32, tb, tsa, tsb, p);
  }
  return MOE_OK;
}

// Pair tiles (256 x TN), an option for groups long enough to fill them (MOE_FP4_PAIR=1; =0 or unset: off).
// They move 30% fewer bytes per MMA into each SM than single-CTA tiles of the same width but were measured
// no faster on a prefill-shaped slice (256 x 256 pairs 1.04 ms against 1.03 ms per GEMM pair for 128 x 256
// single-CTA tiles; 256 x 128 pairs 1.53 against 1.49 for 128 x 128).
bool fp4_pair_for(long long rows_cap, int n_groups) {
  bool on = false;
  (void)rows_cap;
  (void)n_groups;
  if (const char* env = getenv("MOE_FP4_PAIR")) {
    if (env[0] == '1' && env[1] == '\0') on = true;
    if (env[0] == '0' && env[1] == '\0') on = false;
  }
  return on;
}

}  // namespace fp4
}  // namespace moe

using namespace moe;
using namespace moe::fp4;

extern "C" int moe_nvfp4_quantize_weights(const moe_bf16* w, int G, int N, int K, uint8_t* q, uint8_t* sf,
                                          float* gscale, void* stream) {
  if (!w || !q || !sf || !gscale || G < 0 || N < 0 || K < 0) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(q) || !aligned16(sf) || !aligned4(gscale)) return MOE_ERR_INVALID_ARG;
  if (N % ATOM_ROWS != 0 || K % KV_STAGE != 0) return MOE_ERR_UNSUPPORTED;
  if (G == 0 || N == 0 || K == 0) return MOE_OK;
  cudaStream_t s = (cudaStream_t)stream;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;
  unsigned int* amax = reinterpret_cast<unsigned int*>(gscale);  // amax first, then the scale, in place
  if (cudaMemsetAsync(amax, 0, sizeof(float) * G, s) != cudaSuccess) return MOE_ERR_CUDA;
  const long long vec = (long long)N * K / 8;
  const int bx = (int)((vec + 256 * 8 - 1) / (256 * 8) < 64 ? (vec + 256 * 8 - 1) / (256 * 8) : 64);
  weight_amax_kernel<<<dim3(bx, G), 256, 0, s>>>(reinterpret_cast<const uint4*>(w), vec, amax);
  const long long units = (long long)G * N * (K / 16);
  const int grid = (int)(units / 256 + 1 < (long long)sms * 16 ? units / 256 + 1 : (long long)sms * 16);
  weight_quant_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(w), G, N, K, amax, q, sf);
  weight_scale_kernel<<<(G + 255) / 256, 256, 0, s>>>(amax, G);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" long long moe_nvfp4_rows_capacity(int T, int n_routed, int top_k) {
  if (T < 0 || n_routed < 1 || top_k < 1) return 0;
  const long long r = (long long)T * top_k + (long long)n_routed * (ATOM_ROWS - 1);
  return (r + ATOM_ROWS - 1) / ATOM_ROWS * ATOM_ROWS;
}

extern "C" int moe_nvfp4_dispatch(const moe_bf16* x, const int32_t* topk_idx, const int32_t* token_row,
                                  const int32_t* offsets, int T, int d, int n_routed, int top_k, uint8_t* xq,
                                  uint8_t* xsf, int32_t* token_row_pad, int32_t* offsets_pad, void* stream) {
  if (!x || !topk_idx || !token_row || !offsets || !xq || !xsf || !token_row_pad || !offsets_pad)
    return MOE_ERR_INVALID_ARG;
  if (T < 0 || d <= 0 || n_routed < 1 || n_routed > MOE_MAX_ROUTED || top_k < 1 || top_k > MOE_MAX_TOP_K)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(xsf) || !aligned4(topk_idx) || !aligned4(token_row) ||
      !aligned4(offsets) || !aligned4(token_row_pad) || !aligned4(offsets_pad))
    return MOE_ERR_INVALID_ARG;
  if (d % KV_STAGE != 0) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;
  const long long units = (long long)T * (d / 16);
  long long grid = (units + 255) / 256;
  if (grid > (long long)sms * 8) grid = (long long)sms * 8;
  if (grid < 1) grid = 1;  // the offsets are written even with no tokens
  dispatch_quant_kernel<<<(int)grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(x), topk_idx, token_row, offsets,
                                                 T, d, n_routed, top_k, moe_nvfp4_rows_capacity(T, n_routed, top_k),
                                                 xq, xsf, token_row_pad, offsets_pad);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

extern "C" int moe_nvfp4_grouped_gemm(const uint8_t* aq, const uint8_t* asf, const int32_t* offsets_pad,
                                      int n_groups, long long rows_cap, const uint8_t* wq, const uint8_t* wsf,
                                      const float* gscale, int N, int K, int epilogue, uint8_t* out_q,
                                      uint8_t* out_sf, moe_bf16* out, const int32_t* offsets_out,
                                      long long out_rows, void* stream) {
  if (!aq || !asf || !offsets_pad || !wq || !wsf || !gscale || n_groups < 0 || rows_cap < 0 || N <= 0 || K <= 0)
    return MOE_ERR_INVALID_ARG;
  if (n_groups > MOE_MAX_ROUTED) return MOE_ERR_UNSUPPORTED;
  if (epilogue != MOE_NVFP4_EPI_GELU_FP4 && epilogue != MOE_NVFP4_EPI_BF16 && epilogue != MOE_NVFP4_EPI_SWIGLU_FP4)
    return MOE_ERR_INVALID_ARG;
  const bool fp4_out = epilogue != MOE_NVFP4_EPI_BF16;
  const bool swiglu = epilogue == MOE_NVFP4_EPI_SWIGLU_FP4;
  if (fp4_out && (!out_q || !out_sf || !aligned16(out_q))) return MOE_ERR_INVALID_ARG;
  if (epilogue == MOE_NVFP4_EPI_BF16 && (!out || !aligned16(out))) return MOE_ERR_INVALID_ARG;
  if (offsets_out != nullptr && (!aligned4(offsets_out) || out_rows < 0 || out_rows > 0x7fffffffLL))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(aq) || !aligned16(asf) || !aligned16(wq) || !aligned16(wsf) || !aligned4(gscale) ||
      !aligned4(offsets_pad))
    return MOE_ERR_INVALID_ARG;
  if (N % 128 != 0 || K % KV_STAGE != 0 || rows_cap % ATOM_ROWS != 0) return MOE_ERR_UNSUPPORTED;
  // tile width: 256 where N allows (twice the MMA work per stage and 25% fewer bytes per MMA than 128; with
  // the epilogue handing the accumulator back before its math, measured faster at every size: 1.03 against
  // 1.49 ms on a prefill-shaped slice, 4.86 against 4.23 TB/s at decode); MOE_FP4_TN=128 or =256 forces one
  int tn = N % 256 == 0 ? 256 : 128;
  if (const char* env = getenv("MOE_FP4_TN")) {
    if (env[0] == '1' && env[1] == '2' && env[2] == '8' && env[3] == '\0') tn = 128;
    if (env[0] == '2' && env[1] == '5' && env[2] == '6' && env[3] == '\0' && N % 256 == 0) tn = 256;
  }
  if (swiglu) tn = 256;  // 128 gate + 128 up columns a tile
  const uint64_t b_rows = swiglu ? 2ull * N : (uint64_t)N;  // weight rows per group
  if (rows_cap > 0x7fffffffLL) return MOE_ERR_UNSUPPORTED;
  if (n_groups == 0 || rows_cap == 0) return MOE_OK;
  cudaStream_t s = (cudaStream_t)stream;
  int dev, sms;
  int rc = device_info(&dev, &sms);
  if (rc != MOE_OK) return rc;
  unsigned int* status = status_ptr();
  if (!status) return MOE_ERR_CUDA;
  const bool pair = fp4_pair_for(rows_cap, n_groups);
  CUtensorMap ta, ta32, tb, tsa, tsb;
  if ((rc = encode_tmap_u8(&ta, aq, 2, (uint64_t)K / 2, (uint64_t)rows_cap, 1, ROW_BYTES, TM)) != MOE_OK) return rc;
  if ((rc = encode_tmap_u8(&ta32, aq, 2, (uint64_t)K / 2, (uint64_t)rows_cap, 1, ROW_BYTES, 32)) != MOE_OK) return rc;
  const uint32_t b_box = swiglu ? 128u : (uint32_t)(pair ? tn / 2 : tn);  // weight rows a CTA loads per box
  if ((rc = encode_tmap_u8(&tb, wq, 3, (uint64_t)K / 2, b_rows, (uint64_t)n_groups, ROW_BYTES, b_box)) != MOE_OK)
    return rc;
  if (pair) {  // the scale atoms as rows of 256 bytes: 8 rows (2 KB) per operand and stage
    const uint64_t a_sf_bytes = (uint64_t)rows_cap * (K / 16), b_sf_bytes = (uint64_t)n_groups * b_rows * (K / 16);
    if ((rc = encode_tmap_u8_plain(&tsa, asf, SF_ROW, a_sf_bytes / SF_ROW, SF_ROW, SF_BYTES / SF_ROW)) != MOE_OK)
      return rc;
    if ((rc = encode_tmap_u8_plain(&tsb, wsf, SF_ROW, b_sf_bytes / SF_ROW, SF_ROW, SF_BYTES / SF_ROW)) != MOE_OK)
      return rc;
  } else {
    tsa = tsb = ta;  // not read
  }
  Params p{};
  p.offsets_pad = offsets_pad;
  p.G = n_groups;
  p.rows_cap = rows_cap;
  p.a_sf = asf;
  p.b_sf = wsf;
  p.b_sf_stride = (long long)b_rows * (K / 16);
  p.gscale = gscale;
  p.N = N;
  p.K = K;
  p.n_tiles_n = swiglu ? N / 128 : N / tn;
  p.b_up_row = N;
  p.out_q = out_q;
  p.out_sf = out_sf;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.offsets_out = offsets_out;
  p.out_rows = out_rows;
  p.timeout_ns = wait_timeout_ns();
  p.status = status;
  if (pair) {
    // every group may end in a partial 256-row tile
    const long long tiles_upper = (rows_cap / FCfg<128, true>::TILE_M + n_groups) * p.n_tiles_n;
    const int grid = (int)(2 * (tiles_upper < sms / 2 ? tiles_upper : sms / 2));
    if (swiglu)
      rc = launch_fp4<EPI_SWIGLU_FP4, 256, true>(ta, ta32, tb, tsa, tsb, p, grid, s);
    else if (epilogue == MOE_NVFP4_EPI_GELU_FP4)
      rc = tn == 256 ? launch_fp4<EPI_GELU_FP4, 256, true>(ta, ta32, tb, tsa, tsb, p, grid, s)
                     : launch_fp4<EPI_GELU_FP4, 128, true>(ta, ta32, tb, tsa, tsb, p, grid, s);
    else
      rc = tn == 256 ? launch_fp4<EPI_BF16, 256, true>(ta, ta32, tb, tsa, tsb, p, grid, s)
                     : launch_fp4<EPI_BF16, 128, true>(ta, ta32, tb, tsa, tsb, p, grid, s);
    if (rc != MOE_OK) return rc;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  const long long tiles_upper = (rows_cap / TM) * p.n_tiles_n;
  const int grid = (int)(tiles_upper < sms ? tiles_upper : sms);
  if (swiglu)
    rc = launch_fp4<EPI_SWIGLU_FP4, 256>(ta, ta32, tb, tsa, tsb, p, grid, s);
  else if (epilogue == MOE_NVFP4_EPI_GELU_FP4)
    rc = tn == 256 ? launch_fp4<EPI_GELU_FP4, 256>(ta, ta32, tb, tsa, tsb, p, grid, s)
                   : launch_fp4<EPI_GELU_FP4, 128>(ta, ta32, tb, tsa, tsb, p, grid, s);
  else
    rc = tn == 256 ? launch_fp4<EPI_BF16, 256>(ta, ta32, tb, tsa, tsb, p, grid, s)
                   : launch_fp4<EPI_BF16, 128>(ta, ta32, tb, tsa, tsb, p, grid, s);
  if (rc != MOE_OK) return rc;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
