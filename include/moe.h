/*
 * moe.h -- C ABI of libmoe: the forward hot path of one sparse MoE layer
 * (256 routed experts, top-6, plus 2 shared experts normalised jointly) and
 * its auxiliary-loss-free bias update, as hand-written CUDA kernels for
 * NVIDIA B200 (sm_100a).
 *
 * The layer is the one of "Inkling, Dissected" (engineermaxxing.com),
 * §02 "Anatomy of one MoE layer" and §02b "Sigmoid, not softmax":
 *     s_i = sigmoid(x . w_i)                       for all routed + shared experts
 *     kept = top-k over routed i of (s_i + b_i)    (the bias steers selection only)
 *     g_i  = s_i / sum_{j in kept U shared} s_j    (one joint normalisation)
 *     out  = sum_{i in kept U shared} g_i * E_i(x),  E_i(x) = W2_i gelu(W1_i x)
 * followed by §02e "The aux-loss-free bias":
 *     b_i <- b_i + gamma * sign(Lbar - L_i),  L_i = tokens that picked i,
 *     Lbar = (total selections) / n_routed.
 * "Under the hood" (huggingface.co blog), "The routing strategy", adds that the
 * shared experts join the normalisation but are never top-k candidates.
 *
 * Beyond that core path the library also covers: hard expert capacities with
 * token dropping and per-batch balance statistics (§02d, §02g:
 * moe_permute_capped, moe_load_stats); the released configuration's SwiGLU
 * experts and routing-weight scale ("Under the hood", "MoE: the expert
 * configuration", "The routing strategy": MOE_ACT_SWIGLU, route_scale);
 * NVFP4 W4A4 routed experts on the block-scaled tensor cores ("Under the hood",
 * "Quantization: BF16 vs NVFP4": moe_nvfp4_*); and expert parallelism with the
 * exchange done by the dispatch and combine kernels through peer pointers
 * (§02d's all-to-all schedule: moe_ep_*, with CUDA IPC mappings moe_ipc_*).
 *
 * Conventions for every call
 * --------------------------
 *  - All tensor pointers are DEVICE pointers to caller-owned memory, row-major,
 *    16-byte aligned.  The library allocates nothing and keeps no pointer after
 *    a call returns.
 *  - bf16 tensors are passed as moe_bf16 (the 16-bit pattern).
 *  - Every call is asynchronous on the given cudaStream_t (passed as void*;
 *    NULL = legacy default stream).  No call synchronises the host.
 *  - Return value: MOE_OK or a negative MOE_ERR_* code.  Argument errors are
 *    detected on the host before anything is launched; nothing is launched
 *    when a call fails validation.  Calls never abort, exit or trap.
 *  - Errors found on the device (a bounded wait that ran out, an expert index
 *    out of range, inconsistent counts) set bits in a per-device status word
 *    that moe_get_status() reads and clears.
 *  - T = 0 (no tokens) is valid: the call does nothing except what it states
 *    (moe_router_topk still zeroes counts).
 *  - Host-only calls (no stream, nothing launched): moe_permute_scratch_bytes,
 *    moe_nvfp4_rows_capacity, moe_capacity_for, moe_status_string,
 *    moe_set_wait_timeout_ns and the moe_ipc_* mappings.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16;

/* return codes */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1) /* null / misaligned pointer, bad size or k   */
#define MOE_ERR_UNSUPPORTED (-2) /* shape outside what the kernels handle      */
#define MOE_ERR_CUDA (-3)        /* a CUDA runtime/driver call failed          */
#define MOE_ERR_TIMEOUT (-4)     /* reported by moe_get_status: a device wait ran out */
#define MOE_ERR_DEVICE (-5)      /* reported by moe_get_status: other device-side error */
#define MOE_ERR_SCRATCH (-6)     /* scratch buffer smaller than required       */

/* device status bits (moe_get_status) */
#define MOE_STATUS_TIMEOUT 0x1u        /* a bounded mbarrier wait gave up          */
#define MOE_STATUS_BAD_EXPERT 0x2u     /* permute saw an expert id outside [0,n)   */
#define MOE_STATUS_COUNT_MISMATCH 0x4u /* permute's counts differ from topk_idx    */
#define MOE_STATUS_RECV_OVERFLOW 0x8u  /* expert-parallel dispatch/combine: a row's place
                                          in the owner's receive buffer is outside it */

/* expert nonlinearity */
#define MOE_ACT_GELU_TANH 0 /* gelu(u) = u/2 (1 + tanh(sqrt(2/pi)(u + 0.044715 u^3))) */
#define MOE_ACT_SWIGLU 1    /* h = silu(Wg x) * (Wu x), silu(u) = u / (1 + e^-u); W1 = [Wg; Wu] */

/* limits */
#define MOE_MAX_TOP_K 8
#define MOE_MAX_ROUTED 256
#define MOE_MAX_SHARED 8
#define MOE_MAX_GROUPS 1024
#define MOE_EP_MAX_WORLD 64 /* ranks of an expert-parallel group */

/*
 * moe_router_topk -- router scores, biased top-k, joint gates, load counts.
 * "Inkling, Dissected" §02b (router formula and per-token sketch); "Under the
 * hood", "The routing strategy", steps 1-4; loads L_i of §02e.
 *
 *   x          [T, d] bf16          hidden states
 *   w_router   [n_routed + n_shared, d] bf16; rows 0..n_routed-1 routed,
 *              the next n_shared rows the shared experts
 *   bias       [n_routed] fp32      balancing bias b (selection only)
 *   logit_offset [n_routed] fp32 or NULL: added to the routed logits before the
 *              sigmoid (a workload input for skewed routing, not part of the method)
 *   route_scale finite, > 0: the jointly normalised weights are multiplied by it
 *              ("Under the hood", "The routing strategy", step 5: route_scale 8
 *              times the learned global_scale; pass the product).  1: gates sum to 1
 *   topk_idx   [T, top_k] int32 out: kept routed experts, descending s_i + b_i,
 *              ties to the lower index
 *   gates      [T, top_k + n_shared] fp32 out: g of the kept experts in topk
 *              order, then the shared experts in index order; per token they sum
 *              to route_scale (each is fl32(fl32(s / sum) * route_scale))
 *   counts     [n_routed] int32 out: L_i; zeroed by this call, then accumulated
 *   scores_out [T, n_routed + n_shared] fp32 or NULL: s_i for debugging
 * Logits are accumulated in fp32 from bf16 products (tcgen05 tensor cores);
 * s, s + b and the gates are fp32.
 * Limits: d % 8 == 0 (widths that are not a multiple of 64 are read as zeros
 * past d), 1 <= top_k <= min(MOE_MAX_TOP_K, n_routed),
 * n_routed <= 256, n_shared <= 8, n_routed + n_shared <= 272.
 */
int moe_router_topk(const moe_bf16* x, const moe_bf16* w_router, const float* bias, const float* logit_offset,
                    int T, int d, int n_routed, int n_shared, int top_k, float route_scale, int32_t* topk_idx,
                    float* gates, int32_t* counts, float* scores_out, void* stream);

/*
 * moe_permute -- dispatch: group the T*top_k (token, slot) pairs by expert.
 * "Inkling, Dissected" §02 (every token goes to exactly its top-k routed
 * experts; dispatch precedes the experts) and §02d (tokens are queued per expert).
 *
 *   x          [T, d] bf16
 *   topk_idx   [T, top_k] int32 (from moe_router_topk)
 *   counts     [n_routed] int32 or NULL: if given, checked against topk_idx
 *              (MOE_STATUS_COUNT_MISMATCH on the device if they differ); the
 *              layout is always derived from topk_idx itself
 *   offsets    [n_routed + 1] int32 out: rows of expert e are offsets[e] .. offsets[e+1]-1
 *   x_perm     [T*top_k, d] bf16 out: row r = x[row_token[r]]; may be NULL (then x
 *              may be NULL too): only the index outputs are produced, for
 *              moe_experts_ffn to gather the rows itself
 *   row_token  [T*top_k] int32 out
 *   token_row  [T, top_k] int32 out: the row each (token, slot) went to
 *   scratch    device buffer of at least moe_permute_scratch_bytes(T, n_routed)
 *              bytes, caller-owned, contents need not be initialised
 * Within an expert, rows are in increasing token order (deterministic).
 * Limits: d % 8 == 0, n_routed <= 256, 1 <= top_k <= 8.
 */
size_t moe_permute_scratch_bytes(int T, int n_routed);
int moe_permute(const moe_bf16* x, const int32_t* topk_idx, const int32_t* counts, int T, int d, int n_routed,
                int top_k, int32_t* offsets, moe_bf16* x_perm, int32_t* row_token, int32_t* token_row, void* scratch,
                size_t scratch_bytes, void* stream);

/*
 * moe_permute_capped -- moe_permute with a hard expert capacity.
 * "Inkling, Dissected" §02d: every expert can process at most a fixed number
 * of tokens per batch; when more tokens select it, the overflow is dropped and
 * those tokens get nothing from that expert (the layer output is made of what
 * remains).  §02g: the capacity is 1.25x the ideal load k*T/n_routed.
 *
 * Arguments as moe_permute, plus
 *   capacity   >= 0: rows each expert serves.  An expert's queue is filled in
 *              token order; the (t, j) pair whose place in the queue of expert
 *              topk_idx[t, j] is capacity or later is dropped: token_row[t, j]
 *              = -1, no row is made for it (moe_combine then skips it, so the
 *              token's other gates stay as they are).
 *   offsets    rows of expert e are offsets[e] .. offsets[e+1]-1, with
 *              offsets[e+1] - offsets[e] = min(L_e, capacity); rows past
 *              offsets[n_routed] of x_perm and row_token are not written.
 *   counts     (if given) still the demand L_e, dropped picks included.
 * capacity >= max L_e gives exactly moe_permute's result.  Negative capacity:
 * MOE_ERR_INVALID_ARG.  The capacity in tokens is the caller's to choose (the
 * Python layer takes floor(factor * k*T / n_routed)).
 */
int moe_permute_capped(const moe_bf16* x, const int32_t* topk_idx, const int32_t* counts, int T, int d,
                       int n_routed, int top_k, int capacity, int32_t* offsets, moe_bf16* x_perm,
                       int32_t* row_token, int32_t* token_row, void* scratch, size_t scratch_bytes, void* stream);

/*
 * moe_permute_noalloc -- moe_permute for callers that cannot allocate device
 * memory.  No counterpart in the paper: it exists for the library's users, not
 * the method.
 *
 * Some callers have no way to obtain a scratch buffer: a plugin running inside
 * a host application that owns every device allocation and lends it none, a
 * process that reserved all of HBM for its own pool at start-up, or a latency
 * loop that must not call cudaMalloc/cudaFree (they can synchronise the
 * device).  This entry point takes the same arguments as moe_permute minus the
 * scratch buffer and gives identical results; its scratch lives in a fixed
 * device array inside libmoe of MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES (1 MiB),
 * which every GPU that loads the library holds until the process exits.
 *  - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *  - Limit: moe_permute_scratch_bytes(T, n_routed) must not exceed 1 MiB
 *    (with 256 routed experts: T <= 130816 tokens); larger calls return
 *    MOE_ERR_SCRATCH and launch nothing.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents; nothing in it needs clearing, because each call writes every
 *    part it reads.  Calls whose kernels overlap on the GPU (for instance on
 *    two streams without ordering between them) race on the array: order them.
 * Inputs and outputs are caller-owned device buffers exactly as for moe_permute.
 */
#define MOE_PERMUTE_NOALLOC_MAX_SCRATCH_BYTES (1 << 20)
int moe_permute_noalloc(const moe_bf16* x, const int32_t* topk_idx, const int32_t* counts, int T, int d,
                        int n_routed, int top_k, int32_t* offsets, moe_bf16* x_perm, int32_t* row_token,
                        int32_t* token_row, void* stream);

/*
 * moe_grouped_ffn -- the expert MLPs, y = W2_e gelu(W1_e x), for groups of rows.
 * "Inkling, Dissected" §02: an expert is two matrix multiplies with a
 * nonlinearity between them (GELU, tanh form, here).  With MOE_ACT_SWIGLU the
 * expert is the gated one of the released configuration ("Under the hood",
 * "MoE: the expert configuration": SwiGLU experts), y = W2_e (silu(Wg_e x) *
 * (Wu_e x)), three matrices.
 *
 *   rows       [n_rows, d] bf16 input rows
 *   offsets    [n_groups + 1] int32 or NULL.
 *              Non-NULL: group g is rows offsets[g] .. offsets[g+1]-1 (device
 *              values, e.g. from moe_permute), expert expert_base + g; h_scratch
 *              is [n_rows, d_ff] and y is [n_rows, d].
 *              NULL: every group sees all n_rows rows (the shared experts);
 *              h_scratch is [n_groups, n_rows, d_ff] and y is [n_groups, n_rows, d].
 *   w1         [*, d_ff, d] bf16 all experts' first matrices (K-major); for
 *              MOE_ACT_SWIGLU [*, 2*d_ff, d]: rows 0..d_ff-1 the gate projection
 *              Wg, rows d_ff..2*d_ff-1 the up projection Wu
 *   w2         [*, d, d_ff] bf16 all experts' second matrices (K-major)
 *   expert_base index of the first expert used (group g uses expert_base + g)
 *   activation MOE_ACT_GELU_TANH or MOE_ACT_SWIGLU
 *   h_scratch  bf16 hidden activations (caller-owned), written then read
 * Tensor cores (tcgen05, bf16 in, fp32 accumulate); h is rounded to bf16
 * between the two matmuls; y is bf16.
 * Limits: d % 64 == 0, d_ff % 64 == 0, n_groups <= MOE_MAX_GROUPS.
 */
int moe_grouped_ffn(const moe_bf16* rows, const int32_t* offsets, int n_groups, int n_rows, int expert_base,
                    const moe_bf16* w1, const moe_bf16* w2, int d, int d_ff, int activation, moe_bf16* h_scratch,
                    moe_bf16* y, void* stream);

/*
 * moe_experts_ffn -- every expert of the layer in one pair of launches: the
 * n_routed routed experts on their dispatched rows and the n_shared shared
 * experts on all T tokens ("Inkling, Dissected" §02: each token goes to its 6
 * routed experts and to both shared experts; an expert is two matmuls with a
 * nonlinearity).  The same grouped GEMM as moe_grouped_ffn, with the shared
 * experts' tiles scheduled in the same persistent launches as the routed ones.
 *
 *   x          [T, d] bf16 (the shared experts' input, and the routed experts' when
 *              x_perm is NULL)
 *   x_perm     [T*top_k, d] bf16 (from moe_permute) or NULL: then the routed rows
 *              are gathered from x through row_token by the GEMM's own loads
 *              (TMA tile::gather4, four rows an instruction), and moe_permute
 *              need not copy rows (on B200 this is slower than copied rows:
 *              the gathers bound the TMA unit)
 *   row_token  [T*top_k] int32 (from moe_permute); used when x_perm is NULL
 *   offsets    [n_routed + 1] int32 (from moe_permute)
 *   w1, w2     [n_routed + n_shared, d_ff, d] and [n_routed + n_shared, d, d_ff]
 *              bf16: routed experts first, then the shared experts; for
 *              MOE_ACT_SWIGLU w1 is [n_routed + n_shared, 2*d_ff, d] (gate rows,
 *              then up rows), as for moe_grouped_ffn
 *   activation MOE_ACT_GELU_TANH or MOE_ACT_SWIGLU
 *   h_scratch  [T*top_k + n_shared*T, d_ff] bf16 (caller-owned)
 *   y_perm     [T*top_k, d] bf16 out (routed, dispatch order)
 *   y_shared   [n_shared, T, d] bf16 out
 * Limits: d % 64 == 0, d_ff % 64 == 0, n_routed + n_shared <= MOE_MAX_GROUPS.
 */
int moe_experts_ffn(const moe_bf16* x, const moe_bf16* x_perm, const int32_t* row_token, const int32_t* offsets,
                    int T, int n_routed, int n_shared, int top_k, const moe_bf16* w1, const moe_bf16* w2, int d,
                    int d_ff, int activation, moe_bf16* h_scratch, moe_bf16* y_perm, moe_bf16* y_shared,
                    void* stream);

/*
 * NVFP4 routed experts (W4A4).  "Under the hood", "Quantization: BF16 vs NVFP4":
 * the released NVFP4 checkpoint stores FP4 weights and activations in groups of
 * 16 values, each with an FP8 scale ("group_size": 16, dynamic block scales),
 * for Blackwell's FP4 tensor cores.  The router and the shared experts stay
 * bf16.  Recipe (round to nearest even, saturating, in fp32):
 *   weights      g = amax|W| / (6 * 448) per matrix; block scale
 *                s = E4M3(fl(amax_b / 6) / g); codes E2M1(w / fl(s * g))
 *   activations  s = E4M3(fl(amax_b / 6)) per block; codes E2M1(x / s)
 * Each quotient (w / fl(s * g), x / s) is correctly rounded to fp32 before its
 * E2M1 rounding, so an exact midpoint takes the even code.  A block whose scale
 * is 0 has codes 0.  E2M1 codes have no negative zero.
 *
 * Layouts:
 *   codes   [rows, K/2] bytes, K-major; byte j of a row packs values 2j (bits
 *           0-3) and 2j+1 (bits 4-7); E2M1 sign in bit 3
 *   scales  atom-tiled, rows * K/16 bytes: 512-byte atoms of 128 rows x 64
 *           values, the atoms of one 128-row block consecutive along K; the
 *           scale of (row r, block b) is at byte
 *             ((r/128) * (K/64) + b/4) * 512 + (r%32) * 16 + (r%128/32) * 4 + b%4
 *   routed rows for the FP4 path: expert e's rows start at offsets_pad[e], a
 *           multiple of 128 (offsets_pad[e+1] - offsets_pad[e] = the expert's
 *           rows rounded up to 128); the rows of all experts fit in
 *           moe_nvfp4_rows_capacity(T, n_routed, top_k) rows.
 */
#define MOE_NVFP4_EPI_GELU_FP4 0 /* out = FP4(gelu(g * acc)): codes + scales (the next GEMM's A) */
#define MOE_NVFP4_EPI_BF16 1     /* out = bf16(g * acc) */
#define MOE_NVFP4_EPI_SWIGLU_FP4 2 /* SwiGLU GEMM1: weights [n_groups, 2N, K] (gate rows, then up rows);
                                      out = FP4(silu(g * acc_gate) * (g * acc_up)), N output columns */

/*
 * moe_nvfp4_quantize_weights -- quantize G weight matrices [G, N, K] bf16 (K-major)
 *   q       [G, N, K/2] bytes out; sf [G, N*K/16] bytes out (per matrix, atom-tiled)
 *   gscale  [G] fp32 out: each matrix's tensor scale g (the call also uses it as
 *           scratch for the matrices' amax before writing g)
 * Limits: N % 128 == 0, K % 256 == 0.  Run once per weight set.
 */
int moe_nvfp4_quantize_weights(const moe_bf16* w, int G, int N, int K, uint8_t* q, uint8_t* sf, float* gscale,
                               void* stream);

/* Rows (a multiple of 128) that the padded routed rows of one batch can need. */
long long moe_nvfp4_rows_capacity(int T, int n_routed, int top_k);

/*
 * moe_nvfp4_dispatch -- the FP4 dispatch: each token's x row is quantized once
 * (activation recipe) and written to the padded rows of its routed experts.
 *   x          [T, d] bf16; topk_idx [T, top_k]; token_row [T, top_k] and
 *              offsets [n_routed + 1] from moe_permute (or moe_permute_capped;
 *              a token_row of -1 stays -1)
 *   xq         [rows_cap, d/2] bytes out, xsf [rows_cap * d/16] bytes out
 *              (rows_cap = moe_nvfp4_rows_capacity(T, n_routed, top_k)); rows
 *              between experts (padding) are not written
 *   token_row_pad [T, top_k] int32 out: the padded row of each (token, slot)
 *   offsets_pad   [n_routed + 1] int32 out
 * Limits: d % 256 == 0, n_routed <= 256, 1 <= top_k <= 8.
 */
int moe_nvfp4_dispatch(const moe_bf16* x, const int32_t* topk_idx, const int32_t* token_row, const int32_t* offsets,
                       int T, int d, int n_routed, int top_k, uint8_t* xq, uint8_t* xsf, int32_t* token_row_pad,
                       int32_t* offsets_pad, void* stream);

/*
 * moe_nvfp4_grouped_gemm -- out = g_e * (A_e x W_e^T) for every group e on FP4
 * operands with block scales (tcgen05.mma kind::mxf4nvf4, block16 scales, fp32
 * accumulation).  Group e: rows offsets_pad[e] .. offsets_pad[e+1]-1 of A,
 * weight matrix e.
 *   aq, asf    A codes [rows_cap, K/2] and scales (atom-tiled, K values a row)
 *   wq, wsf, gscale   from moe_nvfp4_quantize_weights ([n_groups, N, K])
 *   epilogue   MOE_NVFP4_EPI_SWIGLU_FP4: as GELU_FP4 for a SwiGLU expert's first
 *              GEMM: wq / wsf / gscale quantize [n_groups, 2N, K] (gate rows, then
 *              up rows, one matrix per group), out = FP4(silu(gate) * up), N columns;
 *              MOE_NVFP4_EPI_GELU_FP4: out_q [rows_cap, N/2] and out_sf
 *              (atom-tiled, N values a row) get FP4(gelu(.)) -- the expert's
 *              hidden layer, ready as the second GEMM's A;
 *              MOE_NVFP4_EPI_BF16: out [rows_cap, N] bf16 at the padded rows,
 *              or, with offsets_out (e.g. moe_permute's offsets), group e's
 *              i-th row to row offsets_out[e] + i of out [out_rows, N] for
 *              i < offsets_out[e+1] - offsets_out[e] (padding rows dropped): the
 *              y_perm layout moe_combine reads with moe_permute's token_row
 *   offsets_out [n_groups + 1] int32 or NULL; values clamped to [0, out_rows].
 *              With either epilogue it also gives each group's real row count:
 *              rows past it are padding; they are not loaded and, with the FP4
 *              epilogues, not written, which saves most of the A traffic and the
 *              epilogue work when groups have few rows (decode)
 * Without offsets_out padding rows are computed and written like any row (their
 * FP4 outputs are not meaningful).
 * Limits: N % 128 == 0, K % 256 == 0, rows_cap % 128 == 0, n_groups <= 256.
 */
int moe_nvfp4_grouped_gemm(const uint8_t* aq, const uint8_t* asf, const int32_t* offsets_pad, int n_groups,
                           long long rows_cap, const uint8_t* wq, const uint8_t* wsf, const float* gscale, int N,
                           int K, int epilogue, uint8_t* out_q, uint8_t* out_sf, moe_bf16* out,
                           const int32_t* offsets_out, long long out_rows, void* stream);

/*
 * moe_combine -- gate-weighted sum of the contributors, back in token order.
 * "Inkling, Dissected" §02 (the layer output is the weighted sum of the 8
 * contributing experts) and §02b sketch (out += g_k * e_k(x)).
 *
 *   y_perm     [T*top_k, d] bf16 routed expert outputs in dispatch order
 *   token_row  [T, top_k] int32 (from moe_permute or moe_permute_capped); an
 *              entry of -1 (a dropped assignment) contributes nothing
 *   gates      [T, top_k + n_shared] fp32 (from moe_router_topk)
 *   y_shared   [n_shared, T, d] bf16 or NULL (then n_shared must be 0)
 *   out        [T, d] bf16: out[t] = sum_j g[t,j] y_perm[token_row[t,j]]
 *              + sum_s g[t,top_k+s] y_shared[s,t], accumulated in fp32
 * Limits: d % 8 == 0, 1 <= top_k <= 8, n_shared <= 8.
 */
int moe_combine(const moe_bf16* y_perm, const int32_t* token_row, const float* gates, const moe_bf16* y_shared,
                int T, int d, int top_k, int n_shared, moe_bf16* out, void* stream);

/*
 * moe_bias_update -- the aux-loss-free balancing controller, in place.
 * "Inkling, Dissected" §02e: b_i <- b_i + gamma * sign(Lbar - L_i).
 * Lbar = top_k * T / n_routed; the sign is taken in integers as
 * sign(top_k*T - n_routed*counts[i]) (sign(0) = 0), and b_i is updated in fp32:
 * b_i = fl32(b_i + fl32(gamma) * sign).  Runs after the forward, for the next batch.
 *   counts [n_routed] int32, bias [n_routed] fp32 (in/out).
 */
int moe_bias_update(const int32_t* counts, int n_routed, int T, int top_k, float gamma, float* bias, void* stream);

/*
 * moe_load_stats -- the balance of one batch, from the loads alone.
 * "Inkling, Dissected" §02g (the Router Balance Lab measures MaxVio, the
 * hottest expert's load over the ideal minus one, and the share of expert
 * slots dropped) and §02d (what overflows a capacity is dropped).
 *   counts   [n_routed] int32: L_i (from moe_router_topk), the demand of the
 *            batch of T tokens with top_k choices each
 *   capacity >= 0 (tokens per expert; INT_MAX when no capacity applies)
 *   stats    [2] int32 out (device): stats[0] = max_i L_i,
 *            stats[1] = sum_i max(0, L_i - capacity), the dropped assignments
 *   metrics  [2] fp32 out (device) or NULL: metrics[0] = MaxVio =
 *            max_i L_i * n_routed / (top_k * T) - 1, metrics[1] = drop rate =
 *            stats[1] / (top_k * T); each quotient is formed in fp64 from the
 *            exact integers and rounded once to fp32 (both 0 when T = 0).
 * Limits: n_routed <= 256.  Errors: MOE_ERR_INVALID_ARG (null counts or stats,
 * a pointer not 4-byte aligned, capacity < 0, T < 0, top_k < 1).
 */
int moe_load_stats(const int32_t* counts, int n_routed, int T, int top_k, int capacity, int32_t* stats,
                   float* metrics, void* stream);

/*
 * moe_capacity_for -- the expert capacity of "Inkling, Dissected" §02d ("1.25x
 * the ideal load", the setting §02g's lab uses): floor(factor * top_k * T /
 * n_routed) tokens, with factor = factor_num / factor_den given exactly (1.25 as
 * 5/4), so no binary rounding of the factor moves the result.  Rounding down
 * keeps the capacity at or below the stated multiple of the ideal load.
 * Returns the capacity (clamped to INT_MAX), or MOE_ERR_INVALID_ARG for
 * factor_num < 0, factor_den < 1, T < 0, top_k < 1 or n_routed < 1.  Host only,
 * no device work.
 */
long long moe_capacity_for(long long factor_num, long long factor_den, int T, int top_k, int n_routed);

/* Human-readable text for a MOE_* return code. */
const char* moe_status_string(int code);

/*
 * Expert parallelism over peer memory.  "Inkling, Dissected" §02d: the experts
 * live on different GPUs and every token's rows travel to its experts' GPUs and
 * back (the all-to-all schedule that bounds an expert's capacity).  Rank q of a
 * group of W ranks owns the routed experts [q*E/W, (q+1)*E/W) (E = n_routed, W
 * dividing E) and keeps, in its own device memory, a receive buffer recv_x
 * [recv_rows, d] and an output buffer recv_y [recv_rows, d] (bf16).  Its rows are
 * grouped by its experts and, within an expert, by source rank, so the owner runs
 * one moe_grouped_ffn over all of them (groups recv_offsets, expert_base 0, its
 * experts' weights).  A step on rank r:
 *   1. moe_router_topk, moe_permute (x_perm may be NULL) on its T tokens;
 *   2. the caller all-gathers the per-expert counts: counts_all [W, E] int32;
 *   3. moe_ep_plan -> send_base [E] (where this rank's rows of expert e start in
 *      the owner's buffer) and recv_offsets [E/W + 1] (the groups of this rank's
 *      buffer);
 *   4. moe_ep_dispatch: every routed (token, slot) row is stored straight into its
 *      owner's recv_x at send_base[e] + (its place among this rank's rows of e);
 *   5. the caller orders the ranks (a collective or barrier: every rank's
 *      dispatch is complete before any owner reads), the owner runs
 *      moe_grouped_ffn(recv_x, recv_offsets, E/W, recv_rows, 0, ...) -> recv_y,
 *      then the caller orders the ranks again;
 *   6. moe_ep_combine gathers each token's outputs from the owners' recv_y and
 *      adds the shared experts' rows, in the order and arithmetic of moe_combine
 *      (one rank gives results bit-identical to moe_combine);
 *   7. the bias update with the counts summed over the ranks and the whole batch's
 *      token count.
 * recv_x / recv_y are arrays of W device pointers, in device memory (8-byte
 * aligned), entry q addressing rank q's buffer: this rank's own, and the peers'
 * as mapped into this process (moe_ipc_open, or any peer-accessible mapping).
 * Rows whose place falls outside [0, recv_rows) are skipped and set
 * MOE_STATUS_RECV_OVERFLOW; an expert id outside [0, E) sets
 * MOE_STATUS_BAD_EXPERT.  Errors: MOE_ERR_INVALID_ARG (null or misaligned
 * pointers, W not dividing E, W > MOE_EP_MAX_WORLD, rank outside [0, W)),
 * MOE_ERR_UNSUPPORTED (d % 8 != 0).  Asynchronous on the stream; allocates nothing.
 */
int moe_ep_plan(const int32_t* counts_all, int rank, int world, int n_routed, int32_t* send_base,
                int32_t* recv_offsets, void* stream);
int moe_ep_dispatch(const moe_bf16* x, const int32_t* topk_idx, const int32_t* token_row, const int32_t* offsets,
                    const int32_t* send_base, int T, int d, int n_routed, int top_k, int world,
                    moe_bf16* const* recv_x, long long recv_rows, void* stream);
int moe_ep_combine(const moe_bf16* const* recv_y, const int32_t* topk_idx, const int32_t* token_row,
                   const int32_t* offsets, const int32_t* send_base, const float* gates, const moe_bf16* y_shared,
                   int T, int d, int n_routed, int top_k, int n_shared, int world, long long recv_rows,
                   moe_bf16* out, void* stream);

/*
 * Peer mappings of device buffers between processes (CUDA IPC), for the
 * expert-parallel buffers above.  moe_ipc_get_handle writes the handle of the
 * device allocation that holds dev_ptr into moe_ipc_handle_bytes() bytes of host
 * memory, and dev_ptr's byte offset in that allocation into *offset (both to be
 * sent to the other ranks: a pointer from a caching allocator is often inside a
 * larger allocation).  moe_ipc_open maps a peer's handle into this process (peer
 * access enabled on demand) and returns the mapped allocation's address plus
 * offset; moe_ipc_close unmaps the allocation that holds a pointer moe_ipc_open
 * returned.  A handle cannot be opened in the process that made it.  Host calls;
 * errors: MOE_ERR_INVALID_ARG (null pointers), MOE_ERR_CUDA (the runtime refused).
 */
int moe_ipc_handle_bytes(void);
int moe_ipc_get_handle(const void* dev_ptr, void* handle, unsigned long long* offset);
int moe_ipc_open(const void* handle, unsigned long long offset, void** dev_ptr);
int moe_ipc_close(void* dev_ptr);

/*
 * moe_get_status -- synchronise `stream`, then read and clear this device's
 * status word (MOE_STATUS_* bits) into *device_status.  Returns MOE_OK,
 * MOE_ERR_TIMEOUT if the timeout bit was set, MOE_ERR_DEVICE if another bit
 * was set, or MOE_ERR_CUDA.
 */
int moe_get_status(void* stream, int* device_status);

/*
 * moe_set_wait_timeout_ns -- limit, in nanoseconds, on every device-side wait
 * of the kernels launched afterwards (default 2e9).  A wait that runs out sets
 * MOE_STATUS_TIMEOUT and its kernel winds down and returns.
 */
int moe_set_wait_timeout_ns(uint64_t ns);

/*
 * moe_debug_bounded_wait -- launch one CTA that waits on a shared-memory
 * barrier which nothing ever completes, through the same bounded wait the
 * GEMM kernels use; it must give up after timeout_ns and set
 * MOE_STATUS_TIMEOUT.  For testing the failure path without faulting a GPU.
 */
int moe_debug_bounded_wait(uint64_t timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
