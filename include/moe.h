/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts FFN layer
 * forward: router -> softmax top-k -> permutation by expert -> grouped
 * gated-MLP GEMMs (gate/up, SwiGLU, down) -> weighted combine, in bf16 and in
 * fine-grained FP8.
 *
 * Passages the operations follow (titles of the pages they come from):
 *   [R]  "Mixture of Experts (MoE): a practical explanation of how expert
 *        models work" (lira-now.com), section 5 "How the Router (Top-k
 *        Routing) works step by step" and its pseudocode; section 13's toy
 *        layer.
 *   [X]  "Experts backends" (HF Transformers docs), the backend table
 *        (`eager`, `grouped_mm`, `deepgemm_megamoe` rows), "Switching at
 *        decode", "FP8 and FP4 quantized experts".
 *   [F]  "Fine-grained FP8" (HF Transformers docs), the opening list (128 x 128
 *        weight blocks; per-token activation groups of 128 input channels).
 *   [S]  "AWS improves MoE model performance on Amazon SageMaker AI"
 *        (mikhbar.website), section "Swap-AB advantage in MoE workloads".
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev are DEVICE pointers of the current device; nothing
 *     else in this header takes host memory except moe_forward_hostio's
 *     x_host/out_host. Every device pointer must be 16-byte aligned.
 *   - The library never allocates, frees or synchronises: the caller owns
 *     every buffer, including the workspace `ws` (size from
 *     moe_workspace_size). Work is enqueued on `stream` (a cudaStream_t; NULL
 *     is the legacy default stream) and is stream-ordered.
 *   - bf16 tensors are raw bf16 (IEEE binary16 upper half), e4m3 tensors are
 *     OCP E4M3FN bytes, all row-major and densely packed.
 *   - Validation (pointers, alignment, dimensions, workspace size, device
 *     architecture) happens on the host before any launch. Failure returns a
 *     status without launching anything; moe_last_error() then describes it.
 *     Launch failures return MOE_ERR_CUDA. A device-side wait that runs out
 *     (a bounded spin in a kernel) records MOE_ERR_TIMEOUT in the workspace's
 *     status word, which moe_get_device_status() reads.
 *   - Results are deterministic (bitwise identical run to run).
 *   - NaN or Inf inputs: behaviour unspecified.
 *
 * Dimensions (moe_dims_t): T tokens, H hidden, I expert intermediate, E
 * experts, k experts per token. Supported: T >= 1, H and I multiples of 128,
 * 1 <= E <= 1024, 1 <= k <= min(E, 16), T*k < 2^31.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 1

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,        /* bad pointer, alignment or dimension */
  MOE_ERR_UNSUPPORTED_DEVICE = 2, /* current device is not compute capability 10.0 */
  MOE_ERR_WORKSPACE = 3,          /* workspace missing or smaller than required */
  MOE_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
  MOE_ERR_TIMEOUT = 5             /* a bounded device-side wait ran out */
} moe_status_t;

/* MOE_DTYPE_FP8_E4M3_UE8M0: e4m3 operands whose scales are powers of two
 * (MOE_SCALE_UE8M0), which the block-scaled tensor-core MMA applies itself.
 * MOE_DTYPE_FP4_E2M1: FP4 expert weights (e2m1, two per byte) with e8m0
 * scales per (row, 32 K); activations e4m3 with power-of-two scales. Its
 * workspace layout is the FP8 one. */
typedef enum {
  MOE_DTYPE_BF16 = 0,
  MOE_DTYPE_FP8_E4M3 = 1,
  MOE_DTYPE_FP8_E4M3_UE8M0 = 2,
  MOE_DTYPE_FP4_E2M1 = 3
} moe_dtype_t;

/* GEMM epilogues. The gated ones compute act(g) * u from the gate projection
 * g and the up projection u ([X] "Experts backends": experts with a gated
 * activation -- silu, gelu or relu -- i.e. SwiGLU, GeGLU, ReGLU):
 *   SWIGLU: silu(g) = g / (1 + e^-g)
 *   GEGLU:  gelu(g) = g * Phi(g) = 0.5 g (1 + erf(g / sqrt 2))   (erf form)
 *   REGLU:  relu(g) = max(g, 0) */
typedef enum {
  MOE_EPILOGUE_NONE = 0,
  MOE_EPILOGUE_SWIGLU = 1,
  MOE_EPILOGUE_GEGLU = 2,
  MOE_EPILOGUE_REGLU = 3
} moe_epilogue_t;

/* FP8 scale formats: fp32 values, or powers of two (UE8M0: the 8-bit
 * exponent format float8_e8m0fnu of [X] "UE8M0 scale format", 2^(code-127)).
 * With UE8M0 a scale is the smallest power of two >= amax / 448 (that fp32
 * quotient), clamped to 2^-127..2^127; it is still passed as an fp32 value. */
typedef enum { MOE_SCALE_F32 = 0, MOE_SCALE_UE8M0 = 1 } moe_scale_fmt_t;

typedef struct {
  int32_t T, H, I, E, k;
} moe_dims_t;

/* Thread-local text describing the last failure in this thread ("" if none). */
const char* moe_last_error(void);

/* MOE_ABI_VERSION of the loaded library. */
int32_t moe_abi_version(void);

/* Number of kernel launches this library has issued in this process (all
 * threads). Read it before and after a region to count the launches in it. */
int64_t moe_launch_count(void);

/* Bytes of workspace moe_forward (dt = BF16) or moe_forward_fp8 (dt = FP8)
 * needs for dims d, also enough for moe_route_topk, moe_permute and
 * moe_grouped_gemm on the same dims. 0 for invalid dims. */
size_t moe_workspace_size(moe_dims_t d, moe_dtype_t dt);

/* Byte offsets of the intermediates moe_forward / moe_forward_fp8 leave in
 * the workspace (for inspection and tests). -1 marks a buffer the dtype does
 * not use. Layout (all 256-byte aligned):
 *   status    int32                      device status word
 *   logits    fp32 [T, E]
 *   topk_ids  int32 [T, k]               expert of slot j, slots by descending logit
 *   topk_w    fp32 [T, k]                renormalised routing weight of slot j
 *   offsets   int32 [E + 1]              expert e owns permuted rows [offsets[e], offsets[e+1])
 *   perm_token int32 [T*k]               token of permuted row p
 *   inv_perm  int32 [T, k]               permuted row of (token t, slot j)
 *   x_perm    bf16 [T*k, H]  (BF16)      permuted token rows
 *   xq        e4m3 [T, H], xs fp32 [T, H/128]            (FP8: x quantised per token;
 *                                                       written only when T*k <= 1024, larger
 *                                                       batches quantise into xq_perm directly)
 *   xq_perm   e4m3 [T*k, H], xs_perm fp32 [T*k, H/128]   (FP8: their permuted rows)
 *   h         bf16 [T*k, I]  (BF16)      SwiGLU output per permuted row
 *   hq        e4m3 [T*k, I], hs fp32 [T*k, I/128]        (FP8)
 *   splitk    fp32 partial sums of the small-M GEMMs (BF16 with T <= 64)
 *   y_perm    bf16 [T*k, H]              expert output per permuted row          */
typedef struct {
  int64_t status, logits, topk_ids, topk_w, offsets, perm_token, inv_perm;
  int64_t x_perm, xq, xs, xq_perm, xs_perm, h, hq, hs, splitk, y_perm, scratch, total;
} moe_ws_layout_t;
moe_status_t moe_workspace_layout(moe_dims_t d, moe_dtype_t dt, moe_ws_layout_t* out);

/* Router: logits = x Wr + bias, then softmax top-k with renormalised
 * weights.  [R] section 5 steps 1-5; the pseudocode's logits / softmax / topk /
 * `values / values.sum()`.
 *   x_dev      bf16 [T, H]
 *   wr_dev     bf16 [H, E]
 *   bias_dev   fp32 [E] or NULL (added to the logits before selection)
 *   logits_dev fp32 [T, E] out, or NULL (then kept in the workspace)
 *   ids_dev    int32 [T, k] out: slot j holds the j-th largest logit; equal
 *              fp32 logits go to the lower expert index
 *   w_dev      fp32 [T, k] out: exp(l_j - l_max) / sum over selected
 *   ws/ws_bytes workspace (needed when logits_dev is NULL; may be NULL else)
 * The logits are fp32 sums of exact bf16 x bf16 products in a fixed order:
 * 8 contiguous h blocks of H/8, each summed from zero h ascending, the block
 * sums added left to right, then the bias. So they (and the ids) are
 * bit-reproducible functions of the inputs. I is ignored. */
moe_status_t moe_route_topk(const void* x_dev, const void* wr_dev, const float* bias_dev,
                            moe_dims_t d, float* logits_dev, int32_t* ids_dev, float* w_dev,
                            void* ws, size_t ws_bytes, void* stream);

/* Selection alone, from given logits fp32 [T, E] (same rules as above). */
moe_status_t moe_topk_from_logits(const float* logits_dev, moe_dims_t d, int32_t* ids_dev,
                                  float* w_dev, void* stream);

/* Permutation by expert ([X] backend table, grouped_mm row: tokens sorted by
 * chosen expert so each expert's rows are contiguous). Rows are ordered by
 * expert, then by token ascending.
 *   ids_dev        int32 [T, k] in
 *   offsets_dev    int32 [E + 1] out (exclusive prefix sum of expert counts)
 *   perm_token_dev int32 [T*k] out
 *   inv_perm_dev   int32 [T, k] out
 *   x_dev/x_perm_dev  bf16 [T, H] in / [T*k, H] out: x_perm[p] = x[perm_token[p]]
 *                  (each token's row written to its k rows); both NULL to skip it
 *   ws/ws_bytes    workspace of moe_workspace_size(d, BF16) bytes */
moe_status_t moe_permute(const int32_t* ids_dev, moe_dims_t d, int32_t* offsets_dev,
                         int32_t* perm_token_dev, int32_t* inv_perm_dev, const void* x_dev,
                         void* x_perm_dev, void* ws, size_t ws_bytes, void* stream);

/* moe_permute without a workspace. No passage on the pages corresponds to
 * this entry point: it exists for callers that cannot allocate device memory
 * when they call it -- for example an engine that plans all of its memory
 * once at start-up and must not call cudaMalloc (or a caching allocator)
 * while serving, or code that runs where allocation is not allowed. For
 * valid ids the results are identical to moe_permute's.
 *
 * The scratch lives in one fixed device array inside this library,
 * MOE_NOALLOC_SCRATCH_BYTES bytes on every device that loads it, held until
 * the process exits. Its first 256 bytes are a status word; the rest
 * (MOE_NOALLOC_SCRATCH_BYTES - 256) is the permutation's scratch. Dims whose
 * scratch exceeds that (2 * ceil(T/32) * E * 4 bytes, each of the two parts
 * rounded up to 256, plus E * 4 rounded up to 256) are rejected with
 * MOE_ERR_INVALID_ARG before anything is launched: E = 256 allows T up to
 * 16352, E = 8 up to 524032. The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress) with that device current; make that
 * first call before any stream capture. Every call uses the same array and
 * leaves its contents behind (the scratch needs no clearing: each call writes
 * every scratch word it reads), so calls that can overlap on the GPU -- two
 * streams, or two threads -- race on it: order them on one stream.
 * An expert id outside [0, E), or an expert repeated within a token, is
 * recorded as (MOE_ERR_INVALID_ARG << 8) | 6 in the array's status word
 * (the first failure is kept; read and clear it with
 * moe_permute_noalloc_status); such a pair is skipped and its outputs are
 * left unwritten. Nothing here allocates or frees memory. Arguments as for
 * moe_permute (no ws). */
#define MOE_NOALLOC_SCRATCH_BYTES (1u << 20)
moe_status_t moe_permute_noalloc(const int32_t* ids_dev, moe_dims_t d, int32_t* offsets_dev,
                                 int32_t* perm_token_dev, int32_t* inv_perm_dev,
                                 const void* x_dev, void* x_perm_dev, void* stream);

/* The status word of moe_permute_noalloc's fixed array on the current device:
 * 0, or the first recorded failure. Waits for all work on the device, then
 * reads it into *status_out; with clear != 0 it then sets it back to 0.
 * Blocking and synchronising: for checks between batches, not in hot loops
 * or stream captures. Allocates nothing. */
moe_status_t moe_permute_noalloc_status(int32_t* status_out, int32_t clear);

/* Grouped GEMM on tcgen05 tensor cores ([X] backend table, grouped_mm and
 * deepgemm rows: one grouped GEMM over expert-sorted rows).
 * For each expert e, routed rows m in [offsets[e], offsets[e+1]) of A:
 *   NONE:   C[m, n] = sum_k A[m, k] B[e, n, k]                  n < N
 *   SWIGLU: g = A B[e, 0:N]^T, u = A B[e, N:2N]^T, C = silu(g) * u,
 *           silu(z) = z / (1 + e^-z)   ([X] deepgemm_megamoe row)
 *   GEGLU, REGLU: the same with gelu or relu in place of silu
 *   A_dev  [M_total, K] (bf16, or e4m3 with a_scales fp32 [M_total, K/128]);
 *          with a_rows_dev, routed row m is row a_rows_dev[m] of A_dev
 *          [a_src_rows, K] (and of a_scales [a_src_rows, K/128]) -- the
 *          permutation's row gather done inside the GEMM (rows outside
 *          [0, a_src_rows) read as zeros). Rows-per-expert bounds <= 64 with
 *          a_rows take the large-M kernel.
 *   dt = MOE_DTYPE_FP8_E4M3_UE8M0: the scales are powers of two and the
 *          block-scaled MMA applies them (no row gather, plain needs N % 256 == 0)
 *   B_dev  [E, N or 2N, K] K-major (bf16, or e4m3 with b_scales fp32
 *          [E, rows/128, K/128], one scale per 128 x 128 block, [F])
 *   C_dev  bf16 [M_total, N]; for FP8 gated epilogues with c_scales != NULL, C is
 *          e4m3 [M_total, N] with c_scales fp32 [M_total, N/128] (each
 *          128-group scaled by amax/448, [F] activation groups)
 *   max_rows_per_expert: an upper bound on any expert's row count (0 =
 *          unknown). Bounds <= 64 select the small-M variant that puts the
 *          weight rows in the MMA M slot ([S]).
 * N, K multiples of 128. Accumulation is fp32. ws: its first 256 bytes hold
 * the status word; the small-M kernel may use the rest for fp32 split-K
 * partials (summed in a fixed order, so results stay deterministic). */
moe_status_t moe_grouped_gemm(const void* A_dev, const int32_t* a_rows_dev, int32_t a_src_rows,
                              const void* B_dev, const int32_t* offsets_dev,
                              int32_t M_total, int32_t E, int32_t N, int32_t K, moe_dtype_t dt,
                              moe_epilogue_t ep, void* C_dev, const float* a_scales_dev,
                              const float* b_scales_dev, float* c_scales_dev,
                              int32_t max_rows_per_expert, void* ws, size_t ws_bytes,
                              void* stream);

/* Row gather: dst[i, :] = src[rows[i], :] for i in [0, n), rows of
 * row_bytes bytes (a multiple of 4; 16-byte vectors when a multiple of 16).
 * The data movement of the expert-parallel regroup (rows received per source
 * rank put into local-expert order, and back). An index outside
 * [0, src_rows) skips its row and records (MOE_ERR_INVALID_ARG << 8) | 6 in
 * the status word of ws (when ws is not NULL). n == 0 is a no-op. */
moe_status_t moe_gather_rows(const void* src_dev, int64_t src_rows, const int32_t* rows_dev,
                             int64_t n, int64_t row_bytes, void* dst_dev, void* ws, void* stream);

/* Weighted combine ([R] pseudocode `y = sum_i weights_i * expert_i(x)`):
 *   out[t, :] = sum_{j = 0..k-1} w[t, j] * y_perm[inv_perm[t, j], :]
 * summed in fp32 in slot order, rounded once to bf16.
 *   y_perm_dev bf16 [T*k, H], w_dev fp32 [T, k], inv_perm_dev int32 [T, k],
 *   out_dev bf16 [T, H] */
moe_status_t moe_combine(const void* y_perm_dev, const float* w_dev, const int32_t* inv_perm_dev,
                         moe_dims_t d, void* out_dev, void* stream);

/* The whole layer, bf16: route -> permute -> GEMM1 (+SwiGLU) -> GEMM2 ->
 * combine ([X] backend table; [R] section 5).
 *   x_dev   bf16 [T, H];  wr_dev bf16 [H, E];  bias_dev fp32 [E] or NULL
 *   w13_dev bf16 [E, 2I, H]: rows [0, I) = Wg[e]^T, rows [I, 2I) = Wu[e]^T
 *   w2_dev  bf16 [E, H, I]  = Wd[e]^T
 *   out_dev bf16 [T, H]
 *   ws      >= moe_workspace_size(d, MOE_DTYPE_BF16) bytes
 * No host synchronisation; capturable in a CUDA graph. */
moe_status_t moe_forward(const void* x_dev, const void* wr_dev, const float* bias_dev,
                         const void* w13_dev, const void* w2_dev, moe_dims_t d, void* out_dev,
                         void* ws, size_t ws_bytes, void* stream);

/* moe_forward with the expert activation chosen: act is MOE_EPILOGUE_SWIGLU
 * (what moe_forward uses), MOE_EPILOGUE_GEGLU or MOE_EPILOGUE_REGLU ([X]
 * "Experts backends": gated silu / gelu / relu experts). Anything else is
 * MOE_ERR_INVALID_ARG. Other arguments as for moe_forward. */
moe_status_t moe_forward_gated(const void* x_dev, const void* wr_dev, const float* bias_dev,
                               const void* w13_dev, const void* w2_dev, moe_dims_t d,
                               moe_epilogue_t act, void* out_dev, void* ws, size_t ws_bytes,
                               void* stream);

/* The whole layer with fine-grained FP8 experts ([F]; [X] "FP8 and FP4
 * quantized experts"): x is quantised per (token, 128-channel group) to e4m3
 * with scale amax/448, the SwiGLU output likewise per (row, 128-group of I),
 * and the expert weights come as e4m3 with one fp32 scale per 128 x 128
 * block. The router stays bf16 on x.
 *   w13q_dev e4m3 [E, 2I, H], w13s_dev fp32 [E, 2I/128, H/128]
 *   w2q_dev  e4m3 [E, H, I],  w2s_dev  fp32 [E, H/128, I/128]
 *   ws >= moe_workspace_size(d, MOE_DTYPE_FP8_E4M3) bytes */
moe_status_t moe_forward_fp8(const void* x_dev, const void* wr_dev, const float* bias_dev,
                             const void* w13q_dev, const float* w13s_dev, const void* w2q_dev,
                             const float* w2s_dev, moe_dims_t d, void* out_dev, void* ws,
                             size_t ws_bytes, void* stream);

/* The FP8 layer with power-of-two (UE8M0) scales ([X] "FP8 and FP4 quantized
 * experts", "UE8M0 scale format"): weights quantised with
 * moe_quantize_weight_fp8_fmt(..., MOE_SCALE_UE8M0); x and the hidden
 * activations are quantised the same way inside; both expert GEMMs run on
 * the block-scaled MMA (kind::mxf8f6f4 with E8M0 scales), so the scales need
 * no CUDA-core promotion. act as for moe_forward_gated. Buffers as for
 * moe_forward_fp8; ws >= moe_workspace_size(d, MOE_DTYPE_FP8_E4M3_UE8M0). */
moe_status_t moe_forward_fp8_ue8m0(const void* x_dev, const void* wr_dev, const float* bias_dev,
                                   const void* w13q_dev, const float* w13s_dev,
                                   const void* w2q_dev, const float* w2s_dev, moe_dims_t d,
                                   moe_epilogue_t act, void* out_dev, void* ws, size_t ws_bytes,
                                   void* stream);

/* moe_forward_fp8 with the expert activation chosen (as moe_forward_gated;
 * the activation's output is what gets quantised per 128-group). */
moe_status_t moe_forward_fp8_gated(const void* x_dev, const void* wr_dev, const float* bias_dev,
                                   const void* w13q_dev, const float* w13s_dev,
                                   const void* w2q_dev, const float* w2s_dev, moe_dims_t d,
                                   moe_epilogue_t act, void* out_dev, void* ws, size_t ws_bytes,
                                   void* stream);

/* The layer with FP4 experts ([X] "FP8 and FP4 quantized experts": FP4
 * expert weights packed two per byte with UE8M0 weight scales). The page
 * gives no scale block; the OCP microscaling one is used: one scale per row
 * per 32 consecutive K elements, the smallest power of two >= amax / 6 (1 for
 * an all-zero block), stored as its e8m0 byte (biased exponent). Byte i of a
 * row holds element 2i in its low nibble and 2i + 1 in its high nibble.
 * The scale bytes of a [rows, K] matrix are stored in 512-byte chunks, one
 * per 128 rows x 128 K, chunks ordered (row block, K block); byte
 * 16 r + 4 g + j of a chunk is the scale of row 32 g + r of the block for
 * K elements [32 j, 32 j + 32) of the block (the layout the block-scaled MMA
 * takes its scale factors in).
 * x and the hidden activations are quantised as in moe_forward_fp8_ue8m0
 * (e4m3, power-of-two scale per 128-group); both expert GEMMs run on the
 * block-scaled MMA with e4m3 A and e2m1 B (kind::mxf8f6f4).
 *   w13q_dev u8 [E, 2I, H/2], w13s_dev u8 chunks, E * 2I * H / 32 bytes (moe_quantize_weight_fp4)
 *   w2q_dev  u8 [E, H, I/2],  w2s_dev  u8 chunks, E * H * I / 32 bytes
 *   packed weights 32-byte aligned, scales 16-byte aligned; H % 256 == 0
 *   ws >= moe_workspace_size(d, MOE_DTYPE_FP4_E2M1) bytes; act as for
 *   moe_forward_gated. */
moe_status_t moe_forward_fp4(const void* x_dev, const void* wr_dev, const float* bias_dev,
                             const void* w13q_dev, const uint8_t* w13s_dev, const void* w2q_dev,
                             const uint8_t* w2s_dev, moe_dims_t d, moe_epilogue_t act,
                             void* out_dev, void* ws, size_t ws_bytes, void* stream);

/* Grouped GEMM with FP4 weights (the two GEMMs of moe_forward_fp4):
 *   A_dev        e4m3 [M_total, K], a_scales_dev fp32 [M_total, K/128] powers of two
 *   B_dev        packed e2m1 [E, N_B, K/2] (32-byte aligned), N_B = 2N for a
 *                gated epilogue (gate rows then up rows), N otherwise
 *   b_scales_dev e8m0 bytes in the chunk layout of moe_forward_fp4, E * N_B * K / 32
 *                bytes (16-byte aligned)
 *   C_dev        bf16 [M_total, N] (plain; N % 256 == 0 in the tokens-in-M form),
 *                or with a gated epilogue e4m3 [M_total, N] + c_scales_dev fp32 [M_total, N/128]
 *                (power-of-two scales), or bf16 when c_scales_dev is NULL
 *   offsets, E, ws as for moe_grouped_gemm; max_rows_per_expert in [1, 64]
 *   (an upper bound on any expert's rows, e.g. the token count of a decode
 *   batch) selects the weights-in-M (swap-AB) form, 0 the tokens-in-M one. */
moe_status_t moe_grouped_gemm_fp4(const void* A_dev, const float* a_scales_dev, const void* B_dev,
                                  const uint8_t* b_scales_dev, const int32_t* offsets_dev,
                                  int32_t M_total, int32_t E, int32_t N, int32_t K,
                                  moe_epilogue_t ep, void* C_dev, float* c_scales_dev,
                                  int32_t max_rows_per_expert, void* ws, size_t ws_bytes,
                                  void* stream);

/* FP4 weight quantisation (one-time preparation): nb matrices bf16 [rows,
 * cols] (rows, cols multiples of 128) -> q_dev packed e2m1 [nb, rows, cols/2],
 * s_dev e8m0 bytes (nb * rows * cols / 32, the chunk layout of
 * moe_forward_fp4), by the rule of moe_forward_fp4 with IEEE fp32 division
 * and round-to-nearest-even (ties to the even code). */
moe_status_t moe_quantize_weight_fp4(const void* w_dev, int64_t nb, int64_t rows, int64_t cols,
                                     void* q_dev, uint8_t* s_dev, void* stream);

/* moe_forward with the token rows in HOST memory: copies x_host ([T, H]
 * bf16) to the workspace, runs the layer, copies the result to out_host
 * ([T, H] bf16), all on `stream`. Pinned host buffers make the copies
 * asynchronous; the call returns after enqueueing (synchronise `stream`
 * before reading out_host). ws >= moe_workspace_size(d, BF16) + 2*T*H*2. */
moe_status_t moe_forward_hostio(const void* x_host, const void* wr_dev, const float* bias_dev,
                                const void* w13_dev, const void* w2_dev, moe_dims_t d,
                                void* out_host, void* ws, size_t ws_bytes, void* stream);

/* Activation quantisation ([F]): per row, per group of 128 columns,
 * s = amax/448 (1 for an all-zero group), q = e4m3_rn(v / s) with IEEE fp32
 * division and round-to-nearest-even.
 *   x_dev bf16 [rows, cols] -> q_dev e4m3 [rows, cols], s_dev fp32 [rows, cols/128] */
moe_status_t moe_quantize_act_fp8(const void* x_dev, int64_t rows, int64_t cols, void* q_dev,
                                  float* s_dev, void* stream);

/* Weight quantisation ([F]): nb matrices bf16 [rows, cols] in 128 x 128
 * blocks, same scale and rounding rule -> q_dev e4m3 [nb, rows, cols],
 * s_dev fp32 [nb, rows/128, cols/128]. A one-time preparation step. */
moe_status_t moe_quantize_weight_fp8(const void* w_dev, int64_t nb, int64_t rows, int64_t cols,
                                     void* q_dev, float* s_dev, void* stream);

/* moe_quantize_act_fp8 / moe_quantize_weight_fp8 with the scale format
 * chosen (MOE_SCALE_F32: what those two do; MOE_SCALE_UE8M0: power-of-two
 * scales, see moe_scale_fmt_t). Same buffers and layouts. */
moe_status_t moe_quantize_act_fp8_fmt(const void* x_dev, int64_t rows, int64_t cols, void* q_dev,
                                      float* s_dev, moe_scale_fmt_t fmt, void* stream);
moe_status_t moe_quantize_weight_fp8_fmt(const void* w_dev, int64_t nb, int64_t rows,
                                         int64_t cols, void* q_dev, float* s_dev,
                                         moe_scale_fmt_t fmt, void* stream);

/* One-time weight packing ([X] backend table, grouped_mm row: each expert's
 * gate and up projections map H -> I, its down projection I -> H). Takes the
 * experts' weights in their logical layout and writes the K-major layout
 * every forward and grouped GEMM above reads:
 *   wg_dev, wu_dev bf16 [E, H, I]    gate and up projection of each expert
 *   wd_dev         bf16 [E, I, H]    down projection of each expert
 *   w13_dev        bf16 [E, 2I, H] out: rows [0, I) = Wg[e]^T, rows [I, 2I) = Wu[e]^T
 *   w2_dev         bf16 [E, H, I]  out: Wd[e]^T
 * A pure copy (bit-exact). H and I multiples of 128, 1 <= E <= 65535; the
 * outputs must not overlap the inputs or each other (MOE_ERR_INVALID_ARG).
 * Stream-ordered, no workspace; untimed preparation, not part of the layer.
 * The FP8 / FP4 weights are then quantised from w13 / w2 with
 * moe_quantize_weight_fp8(_fmt) / moe_quantize_weight_fp4. */
moe_status_t moe_pack_weights(const void* wg_dev, const void* wu_dev, const void* wd_dev,
                              int32_t E, int32_t H, int32_t I, void* w13_dev, void* w2_dev,
                              void* stream);

/* Expert-parallel exchange planned and moved on the device ([X] backend
 * table, deepgemm_megamoe row: experts spread over ranks, each token's rows
 * dispatched to the ranks owning their experts and combined back). G ranks
 * own E / G consecutive experts each (rank g: [g*El, (g+1)*El), El = E / G).
 * Every rank has routed and permuted its own tokens (moe_route_topk,
 * moe_permute: rows expert-major) and all ranks hold the same all-gathered
 * counts_all int32 [G, E] (row s: rank s's rows per expert, e.g. the
 * differences of its offsets). No count ever goes to the host.
 *
 * moe_ep_plan (one small kernel) writes rank `rank`'s plan, int32, into
 * plan_dev (moe_ep_plan_bytes(E, G) bytes, 16-byte aligned):
 *   loc_off   [El + 1]   at plan_dev: this rank's receive buffer is
 *                        expert-major (local expert j, then source rank
 *                        ascending, then the source's row order); local expert
 *                        j owns rows [loc_off[j], loc_off[j+1]) -- the offsets
 *                        to run moe_grouped_gemm on it directly
 *   send_base [E]        at plan_dev + (El + 1 rounded up to 4): row in rank
 *                        e / El's receive buffer of this rank's first row for
 *                        expert e
 *   ret_lb [El*G + 1], ret_dst [El*G]   then: the return path's blocks
 * moe_ep_plan_bytes returns 0 for E, G outside 1 <= G <= 64, E <= 1024, E % G == 0.
 *
 * moe_ep_dispatch: row p of x_perm_dev [R, row_bytes] (this rank's permuted
 * rows, offsets_dev [E + 1] from moe_permute) is stored to row
 * send_base[e] + (p - offsets[e]) of the buffer at dst_bufs_dev[e / El]
 * (a DEVICE array of G addresses: the ranks' receive buffers, mapped into
 * this process, e.g. symmetric memory; each dst_rows rows long).
 * moe_ep_return: row q < loc_off[El] of y_loc_dev [cap_rows, row_bytes]
 * (this rank's expert outputs in receive order) is stored back to its
 * source rank s, at the row of src_bufs_dev[s] (the ranks' y_perm buffers,
 * src_rows rows each) it was dispatched from. cap_rows is any upper bound on
 * the received rows (the kernel reads the exact count from the plan).
 * Plain 16-byte stores, each warp's ended by a system-scope fence; the caller
 * orders them before the other ranks' reads with a cross-rank
 * synchronisation on the stream (e.g. an NCCL collective). A destination row
 * outside its buffer is skipped and (MOE_ERR_INVALID_ARG << 8) | 6 recorded
 * in ws's status word (ws may be NULL). row_bytes a multiple of 16. */
size_t moe_ep_plan_bytes(int32_t E, int32_t G);
moe_status_t moe_ep_plan(const int32_t* counts_all_dev, int32_t G, int32_t rank, int32_t E,
                         int32_t* plan_dev, void* stream);
moe_status_t moe_ep_dispatch(const void* x_perm_dev, const int32_t* offsets_dev,
                             const int32_t* plan_dev, int32_t E, int32_t G, int32_t R,
                             int64_t row_bytes, const uint64_t* dst_bufs_dev, int64_t dst_rows,
                             void* ws, void* stream);
moe_status_t moe_ep_return(const void* y_loc_dev, const int32_t* plan_dev, int32_t E, int32_t G,
                           int64_t cap_rows, int64_t row_bytes, const uint64_t* src_bufs_dev,
                           int64_t src_rows, void* ws, void* stream);

/* Reads the workspace's device status word into *status_out: 0 (MOE_OK), or
 * (code << 8) | site for the first failure a kernel recorded. code is
 * MOE_ERR_TIMEOUT for a bounded wait that ran out, the site naming it: 1 a
 * GEMM producer waiting for a free stage, 2 an MMA thread waiting for its
 * operands, 3 an MMA thread waiting for a free accumulator, 4 an epilogue
 * waiting for a full accumulator, 5 the final drain, 7 the self-test below,
 * 8 a row load of the row scatter; code MOE_ERR_INVALID_ARG with site 6 means
 * an expert id or row index out of range was met and skipped. Synchronises
 * the device (a blocking copy); not for hot loops. */
moe_status_t moe_get_device_status(const void* ws, int32_t* status_out);

/* Clears the workspace's device status word (stream-ordered). */
moe_status_t moe_clear_device_status(void* ws, void* stream);

/* Self-test of the bounded device waits the pipelined kernels use (failure
 * detection without a GPU fault): one CTA waits on an mbarrier that nothing
 * arrives at, for budget_cycles SM clocks (1000 .. 2e9), then gives up and
 * records (MOE_ERR_TIMEOUT << 8) | 7 in the status word of ws, unless the
 * word already holds a failure, in which case it gives up at once and leaves
 * the word unchanged. Stream-ordered; read the result with
 * moe_get_device_status. The context stays usable. */
moe_status_t moe_check_wait_timeout(void* ws, int64_t budget_cycles, void* stream);

/* Stage timing for moe_forward / moe_forward_fp8 on the calling thread: when
 * set, the next forwards record events[0..5] (cudaEvent_t) on their stream at
 * entry, after routing, after the permutation, after GEMM1, after GEMM2 and
 * after the combine. Pass NULL to stop. */
moe_status_t moe_set_stage_events(void* const* events, int32_t n);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
