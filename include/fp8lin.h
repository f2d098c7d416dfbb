/*
 * fp8lin.h -- C ABI of the B200 (sm_100a) FP8 W8A8 linear-layer library.
 *
 * The library implements the linear layer that the DeepSeek-V3 deployment page
 * ("FP8 推理提速 83.6%: DeepSeek-V3 在 AMD MI250 上的完整落地指南", section 运行时)
 * runs when dtype is fp8:
 *     x, scale = act_quant(x, block_size, scale_fmt)   # per token, per 128 channels
 *     y        = fp8_gemm(x, scale, weight, weight.scale)
 * with weights stored as E4M3 codes plus one fp32 scale_inv per 128x128 block
 * (same page, FP8 权重转换命令与关键配置参数), and the MoE variant over 256 routed
 * experts with 8 active per token (same page, 官方配置中最关键的四个参数).
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    allocates and frees no device memory and keeps no per-call state.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call only enqueues work on that stream and returns; results are ready
 *    when the stream reaches that point.
 *  - Arguments are validated on the host before anything is launched; a rejected
 *    call returns a non-zero fp8_status and enqueues nothing.  A failed launch
 *    returns FP8_ERR_CUDA.  Nothing aborts or throws across the ABI.
 *  - Row-major layouts throughout.  "codes" are one byte per element (E4M3 or
 *    E5M2 bit patterns).  Scales are fp32 dequantisation multipliers:
 *    x ~= decode(code) * s  ("量化：FP8 与混合精度推理", FP8 也需要 scale).
 *  - Rounding: q = saturate(round_to_nearest_even(fl32(x / s))) to +-Fmax, so no
 *    code is ever Inf (E4M3 Fmax = 448, E5M2 Fmax = 57344; "LLM 推理的 FP8 混合精度
 *    工程 2026", section 2).  s = max(fl32(amax / Fmax), 2^-126); with
 *    FP8_SCALE_UE8M0 s is that value rounded up to a power of two (stored as fp32).
 *  - Pipelined waits inside the GEMM kernels are bounded (about 2 s); a wait that
 *    runs out sets a device-side error word that fp8_device_error() reports.
 */
#ifndef FP8LIN_H
#define FP8LIN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8_OK = 0,
    FP8_ERR_INVALID_ARG = 1,   /* null pointer, bad enum value, negative size */
    FP8_ERR_SHAPE = 2,         /* shape outside what the operation supports      */
    FP8_ERR_ALIGNMENT = 3,     /* pointer or leading dimension misaligned        */
    FP8_ERR_UNSUPPORTED = 4,   /* valid request this build does not implement    */
    FP8_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed           */
    FP8_ERR_TIMEOUT = 6,       /* a bounded device-side wait ran out             */
    FP8_ERR_INVALID_SCALE = 7  /* fp8_mx_pack_pow2 got a scale that is not a
                                  positive normal power of two (reported by
                                  fp8_device_error)                              */
} fp8_status;

typedef enum { FP8_E4M3 = 0, FP8_E5M2 = 1 } fp8_format;
typedef enum { FP8_SCALE_FP32 = 0, FP8_SCALE_UE8M0 = 1 } fp8_scale_fmt;
typedef enum { FP8_OUT_BF16 = 0, FP8_OUT_FP32 = 1 } fp8_out_dtype;

/*
 * fp8_act_quant -- dynamic per-token, per-group activation quantisation
 * (DeepSeek-V3 page, 运行时: act_quant per token per 128 channels; "FP8 推理",
 * Dynamic Scaling: scale = max|x| / 448 from the current batch).
 *
 *   x      bf16 [M][ldx] (only the first K columns are read); 16-byte aligned.
 *   M, K   rows and columns, M >= 0, K > 0, K % 16 == 0.  The last group of a row
 *          may be shorter than `group` (its amax covers the valid columns only).
 *   ldx    row stride of x in elements, ldx >= K, ldx % 8 == 0.
 *   group  channels per scale; 128 is the supported value.
 *   fmt    FP8_E4M3 or FP8_E5M2 codes.
 *   scale_fmt  FP8_SCALE_FP32 or FP8_SCALE_UE8M0.
 *   q      codes [M][K] (dense, row stride K); 16-byte aligned.
 *   s      fp32 scales [M][ceil(K/group)] (dense).
 * Returns FP8_OK, or INVALID_ARG / SHAPE / ALIGNMENT / UNSUPPORTED / CUDA.
 * M == 0 is a no-op.
 */
int fp8_act_quant(const void* x, int64_t M, int64_t K, int64_t ldx, int group,
                  int fmt, int scale_fmt, void* q, float* s, void* stream);

/*
 * fp8_weight_quant -- weight quantisation with one scale_inv per block x block
 * tile (DeepSeek-V3 page, FP8 权重转换命令与关键配置参数: e4m3 weights, 128x128
 * block scales), or with one scale for the whole tensor when block == 0 (the
 * per-tensor OCP scaling the ROCm page contrasts with block scaling, section 1.2;
 * E5M2 allowed here, Fmax 57344).
 *
 *   w      bf16 [N][K] (dense); 16-byte aligned.
 *   N, K   N >= 0, K > 0, K % 16 == 0.  Edge blocks may be partial.
 *   block  128, or 0 for per-tensor.
 *   q      codes [N][K]; 16-byte aligned.
 *   s_inv  fp32 [ceil(N/128)][ceil(K/128)] for block == 128, fp32 [1] for block == 0.
 *          In per-tensor mode s_inv[0] also serves, in stream order, as the amax
 *          accumulator of the first pass, so it must not alias w or q.
 * Returns FP8_OK or an error status; N == 0 is a no-op.
 */
int fp8_weight_quant(const void* w, int64_t N, int64_t K, int block, int fmt,
                     int scale_fmt, void* q, float* s_inv, void* stream);

/*
 * fp8_block_gemm -- block-scaled FP8 GEMM with fp32 accumulation
 * (DeepSeek-V3 page, 运行时: fp8_gemm(x, scale, weight, weight.scale);
 * "LLM 推理的 FP8 混合精度工程 2026", section 3: FP32 accumulation):
 *
 *   y[m][n] = sum_{kb < K/128} sa[m][kb] * sw[n/128][kb] *
 *             sum_{k in block kb} dec(qa[m][k]) * dec(qw[n][k])
 *
 *   qa     E4M3 codes [M][K]; 16-byte aligned.
 *   sa     fp32 [M][K/128] (act_quant's layout).
 *   qw     E4M3 codes [N][K]; 16-byte aligned.
 *   sw     fp32 [ceil(N/128)][K/128] (weight_quant's layout).
 *   M >= 0, N > 0 with N % 16 == 0, K > 0 with K % 128 == 0.
 *   out_dtype  FP8_OUT_BF16 (round to nearest even) or FP8_OUT_FP32.
 *   y      [M][N] of out_dtype; 16-byte aligned.
 * Each 128-deep K-block is one tensor-core partial product that is scaled and
 * added into an fp32 accumulator (per-K-block promotion).
 */
int fp8_block_gemm(const void* qa, const float* sa, const void* qw, const float* sw,
                   int64_t M, int64_t N, int64_t K, int out_dtype, void* y, void* stream);

/*
 * fp8_block_gemm_quant -- fp8_block_gemm with bf16 output whose epilogue also applies
 * the next layer's act_quant to that output (the DeepSeek-V3 page's linear layer runs
 * act_quant on every linear input, 运行时; here the quantisation of y happens while y is
 * still in registers instead of in a separate pass over HBM):
 *   y = fp8_block_gemm(...) rounded to bf16;
 *   qy, sy = fp8_act_quant(y, group 128, fmt, scale_fmt)   -- bit-exact with it.
 *
 *   Arguments as fp8_block_gemm, plus N % 128 == 0 (whole 128-channel groups).
 *   y      bf16 [M][N], 16-byte aligned, or NULL when only the quantised output is wanted.
 *   fmt, scale_fmt  as fp8_act_quant.
 *   qy     codes [M][N], 16-byte aligned; sy fp32 [M][N/128].
 * Returns FP8_OK or an error status; M == 0 is a no-op.
 */
int fp8_block_gemm_quant(const void* qa, const float* sa, const void* qw, const float* sw, int64_t M, int64_t N,
                         int64_t K, void* y, int fmt, int scale_fmt, void* qy, float* sy, void* stream);

/*
 * fp8_weight_dequant -- FP8 weights back to bf16, the BF16 path of the DeepSeek-V3 page
 * (运行时: weight = weight_dequant(weight, weight.scale), then a plain GEMM; FP8 权重转换:
 * fp8_cast_bf16.py): w[n][k] = bf16_rne(fl32(dec(q[n][k]) * s_inv[n/128][k/128])), or
 * with the single scale s_inv[0] when block == 0.
 *
 *   q      codes [N][K] (fmt), 16-byte aligned; N >= 0, K > 0, K % 16 == 0.
 *   s_inv  fp32 [ceil(N/128)][ceil(K/128)] (block 128) or [1] (block 0).
 *   w      bf16 [N][K], 16-byte aligned.
 * Returns FP8_OK or an error status; N == 0 is a no-op.
 */
int fp8_weight_dequant(const void* q, const float* s_inv, int64_t N, int64_t K, int block, int fmt, void* w,
                       void* stream);

/*
 * fp8_grouped_gemm -- the same GEMM per MoE expert over expert-sorted rows
 * (ROCm page, section 2.3: block-scale fused MoE; DeepSeek-V3 page: 256 routed
 * experts, 8 active per token).  Row m of qa belongs to expert e when
 * group_offsets[e] <= m < group_offsets[e+1]; it is multiplied by qw[e].
 *
 *   qa     E4M3 codes [total_M][K]; sa fp32 [total_M][K/128].
 *   qw     E4M3 codes [E][N][K]; sw fp32 [E][ceil(N/128)][K/128].
 *   group_offsets  DEVICE int32 [E+1], non-decreasing, [0] == 0,
 *          [E] <= total_M.  Not read on the host (no synchronisation).
 *   E > 0, total_M >= 0, N % 16 == 0, K % 128 == 0.
 *   y      [total_M][N] of out_dtype.  Rows outside every group are not written.
 */
int fp8_grouped_gemm(const void* qa, const float* sa, const void* qw, const float* sw,
                     const int32_t* group_offsets, int64_t E, int64_t total_M,
                     int64_t N, int64_t K, int out_dtype, void* y, void* stream);

/*
 * MXFP8 scale layout ("tiled").  The exponent bytes of an operand with R rows and K
 * columns are stored in the order the tensor core's block-scaled MMA reads them:
 * ceil(R/128) x ceil(K/128) atoms of 512 bytes, atom (rb, kb) at byte offset
 * (rb * ceil(K/128) + kb) * 512; inside an atom, row r (0..127 of row block rb) and
 * 32-element block j (0..3 of K-block kb) are at byte (r % 32) * 16 + (r / 32) * 4 + j.
 * Size in bytes: FP8_MX_SF_BYTES(R, K).  Bytes of rows >= R or of blocks beyond K are
 * not written by fp8_mx_quant and not read for any output.
 */
#define FP8_MX_SF_BYTES(R, K) ((((int64_t)(R) + 127) / 128) * (((int64_t)(K) + 127) / 128) * 512)

/*
 * fp8_mx_quant -- MXFP8 quantisation ("ROCm 7 原生 FP8/MXFP8 ... AITER", section 1.2:
 * the tensor is split into blocks of 32 elements, each with its own scale factor;
 * section 1.1: MXFP8 = 8-bit elements plus a shared exponent).  Every row of x is cut
 * into blocks of 32 consecutive elements; a block's scale is the power of two
 * s = 2^e = 2^ceil(log2(amax / Fmax)), e >= -126 (the pages do not fix the exponent
 * rule; this is the ue8m0 rule above, applied per block, so no element saturates),
 * stored as the E8M0 byte e + 127; codes are q = saturate(RNE(x / s)).  Used for
 * activations and, row by row, for weights alike.
 *
 *   x      bf16 [M][ldx] (first K columns); 16-byte aligned; ldx >= K, ldx % 8 == 0.
 *   M, K   M >= 0, K > 0, K % 16 == 0 (a row's last block may hold 16 elements).
 *   fmt    FP8_E4M3 or FP8_E5M2.
 *   q      codes [M][K]; 16-byte aligned.
 *   e8     exponent bytes in the tiled layout above, FP8_MX_SF_BYTES(M, K) bytes.
 * Returns FP8_OK or an error status; M == 0 is a no-op.
 */
int fp8_mx_quant(const void* x, int64_t M, int64_t K, int64_t ldx, int fmt, void* q, void* e8,
                 void* stream);

/*
 * fp8_mx_gemm -- FP8 GEMM with power-of-two scales per 32-element block of K, applied
 * by the tensor core (the block-scaled MMA of sm_100a) to every product, accumulating
 * all of K in fp32 with no per-K-block promotion:
 *
 *   y[m][n] = sum_k dec(qa[m][k]) 2^(ea(m, k/32) - 127) * dec(qw[n][k]) 2^(ew(n, k/32) - 127)
 *
 *   qa     E4M3 codes [M][K]; sfa its exponent bytes, tiled (FP8_MX_SF_BYTES(M, K)).
 *   qw     E4M3 codes [N][K]; sfw its exponent bytes, tiled (FP8_MX_SF_BYTES(N, K)).
 *   M >= 0, N > 0 with N % 16 == 0, K > 0 with K % 128 == 0; qa, qw, sfa, sfw, y
 *   16-byte aligned.
 *   out_dtype, y  as fp8_block_gemm.
 * The ue8m0 block GEMM (act_quant / weight_quant with FP8_SCALE_UE8M0, fp8_block_gemm's
 * scale layout) runs on this path after fp8_mx_pack_pow2 and gives fp8_block_gemm's
 * result.  Accumulation: fp32 in tensor memory over all K (one rounding per 32-element
 * block product); the tolerance this implies is stated with the parity tests.
 */
int fp8_mx_gemm(const void* qa, const void* sfa, const void* qw, const void* sfw, int64_t M, int64_t N,
                int64_t K, int out_dtype, void* y, void* stream);

/*
 * fp8_mx_pack_pow2 -- converts fp32 power-of-two scales in fp8_block_gemm's layout
 * (the ue8m0 scales of "FP8 推理提速 83.6%: DeepSeek-V3 在 AMD MI250 上的完整落地指南",
 * 关键配置参数: scale_fmt ue8m0) into the tiled exponent layout of fp8_mx_gemm, each
 * 128-element scale replicated onto its four 32-element blocks.
 *
 *   s          fp32 [rows][K/128] (row_block 1: act_quant's layout) or
 *              fp32 [ceil(rows/128)][K/128] (row_block 128: weight_quant's 128x128 blocks).
 *   rows, K    rows >= 0, K > 0 with K % 128 == 0.
 *   sf         FP8_MX_SF_BYTES(rows, K) bytes; 16-byte aligned.
 * A scale that is not a positive normal power of two is flagged: the next
 * fp8_device_error() returns FP8_ERR_INVALID_SCALE.  rows == 0 is a no-op.
 */
int fp8_mx_pack_pow2(const float* s, int64_t rows, int64_t K, int row_block, void* sf, void* stream);

/* History rule of fp8_delayed_quant. */
typedef enum { FP8_AMAX_MOST_RECENT = 0, FP8_AMAX_MAX = 1 } fp8_amax_algo;

/*
 * fp8_delayed_quant -- one step of delayed per-tensor scaling, a single pass over x
 * ("ROCm 7 原生 FP8/MXFP8 ... AITER", section 4.3 延迟缩放: the tensor is divided by the
 * scale of the PREVIOUS step, clamped to +-Fmax and cast; the scale of the next step is
 * derived from this step's amax with a margin, amax / 400 for E4M3, starting from 1.0;
 * section 6: an amax history, "max" over it; its checklist tracks the share of clipped
 * elements):
 *   q[i]        = saturate(RNE(x[i] / s_prev)),  s_prev = *scale on entry
 *   *n_clipped  = number of i with |fl32(x[i] / s_prev)| > Fmax
 *   *s_used     = s_prev (dequantise with x ~= dec(q) * s_used)
 *   history[*pos] = max |x|;  then  *scale = max(A / target, 2^-126) with A = the max
 *   over history[0..hist_len) (FP8_AMAX_MAX) or this step's amax (FP8_AMAX_MOST_RECENT);
 *   history[(*pos + 1) % hist_len] = 0;  *pos = (*pos + 1) % hist_len.
 *
 *   x        bf16 [n], 16-byte aligned; n >= 0, n % 8 == 0.
 *   fmt      FP8_E4M3 or FP8_E5M2; target > 0, finite (the page: 400 for E4M3).
 *   scale, pos, history   DEVICE state owned by the caller and carried from step to
 *            step: fp32 [1], int32 [1], fp32 [hist_len] (1 <= hist_len <= 65536).
 *            Before the first step: *scale = 1.0, *pos = 0, history all 0.  Steps on
 *            one state must be ordered on one stream.
 *   q        codes [n], 16-byte aligned.
 *   n_clipped  DEVICE uint64 [1] (8-byte aligned); s_used DEVICE fp32 [1].
 * Returns FP8_OK or an error status.  Enqueues a memset of *n_clipped and two kernels.
 */
int fp8_delayed_quant(const void* x, int64_t n, int fmt, float target, int64_t hist_len, int algo, float* scale,
                      int32_t* pos, float* history, void* q, uint64_t* n_clipped, float* s_used, void* stream);

/*
 * MoE routing and the expert GEMMs around it ("FP8 推理提速 83.6%: DeepSeek-V3 在 AMD MI250
 * 上的完整落地指南", 官方配置中最关键的四个参数: 256 routed experts, 8 active per token;
 * "ROCm 7 ... AITER", section 2.3: block-scale fused MoE).  A layer runs
 *   fp8_moe_route -> fp8_act_quant_permute -> fp8_moe_gemm.
 *
 * fp8_moe_route -- per token, the k experts of largest score (ties to the lower expert
 * index; a NaN score never wins), gate weights w = selected scores / their fp32 sum in
 * selection order (1/k each if that sum is 0); then the T*k (token, j) pairs sorted
 * stably by (expert, token).  All pointers DEVICE.
 *   scores     fp32 [T][E] (non-negative affinities), 1 <= E <= 1024, 1 <= k <= min(E, 32).
 *   ids, w     int32 / fp32 [T][k], in selection order.
 *   offsets    int32 [E+1]: rows of expert e are [offsets[e], offsets[e+1]).
 *   row_token, row_weight   int32 / fp32 [T*k]: token and gate weight of each sorted row.
 *   token_row  int32 [T*k]: sorted row of pair (t, j) at t*k + j.
 *   workspace  DEVICE scratch owned by the caller, at least FP8_MOE_ROUTE_WS_BYTES(T, k, E)
 *              bytes, 4-byte aligned, no initial contents required; it carries the
 *              per-chunk expert counts of the sort (chunks of 512 pairs, one CTA each),
 *              so calls that share a workspace must be ordered on one stream.
 * Returns FP8_OK or an error status (FP8_ERR_SHAPE for a workspace that is too small).
 */
#define FP8_MOE_ROUTE_WS_BYTES(T, k, E) \
  (((((int64_t)(T) * (int64_t)(k)) + 511) / 512 + 1) * (int64_t)(E) * 4)

int fp8_moe_route(const float* scores, int64_t T, int64_t E, int64_t k, int32_t* ids, float* w, int32_t* offsets,
                  int32_t* row_token, float* row_weight, int32_t* token_row, void* workspace, int64_t workspace_bytes,
                  void* stream);

/*
 * fp8_moe_route_noalloc -- fp8_moe_route with the sort's scratch inside the library
 * instead of a caller workspace; the pages have no counterpart (it is an interface
 * variant, not a step of the method).  Same arguments and results as fp8_moe_route,
 * without workspace / workspace_bytes.  The scratch is a fixed device array of 256 KiB
 * per device: problems with FP8_MOE_ROUTE_WS_BYTES(T, k, E) > 262144 are rejected with
 * FP8_ERR_SHAPE (e.g. 4096 tokens, top-8 of 256 experts fit; 16384 tokens do not).  The
 * array's address is looked up once per device (with that device current); the call
 * allocates and frees no memory, and nothing in the array has to start at zero.  All
 * calls on one device share the array, so calls that overlap in time (different
 * streams, or host threads without ordering) race and give undefined results.
 */
int fp8_moe_route_noalloc(const float* scores, int64_t T, int64_t E, int64_t k, int32_t* ids, float* w,
                          int32_t* offsets, int32_t* row_token, float* row_weight, int32_t* token_row, void* stream);

/*
 * fp8_act_quant_permute -- fp8_act_quant (group 128) of the T token rows of x, each
 * row's codes and scales written to its k expert-sorted rows token_row[t*k + j]
 * (fp8_moe_route's map).  Per-token quantisation commutes with duplicating a row, so
 * this equals quantising the permuted activations, without materialising them in
 * bf16 or running a separate gather.
 *   x, T, K, ldx, fmt, scale_fmt   as fp8_act_quant (M = T).
 *   token_row  DEVICE int32 [T*k], 1 <= k <= 32.
 *   q          codes [T*k][K]; s fp32 [T*k][ceil(K/128)].
 */
int fp8_act_quant_permute(const void* x, int64_t T, int64_t K, int64_t ldx, int fmt, int scale_fmt,
                          const int32_t* token_row, int64_t k, void* q, float* s, void* stream);

/*
 * fp8_moe_gemm -- the grouped expert GEMM over the expert-sorted rows with the gate-
 * weighted combine fused into its epilogue:
 *   out[t][n] = sum over the rows r with row_token[r] == t of
 *               row_weight[r] * (sum_kb sa[r][kb] sw[e][n/128][kb] P_kb[r][n]),
 * e = the expert whose range holds r; each row's product is added into out with an
 * fp32 reduction (order unspecified), so the per-expert outputs are never stored.
 *   qa, sa     sorted codes [T*k][K] / scales [T*k][K/128] (fp8_act_quant_permute).
 *   qw, sw     [E][N][K] / [E][ceil(N/128)][K/128]; offsets DEVICE int32 [E+1].
 *   row_token, row_weight   DEVICE [T*k] (fp8_moe_route).
 *   N % 16 == 0, K % 128 == 0.
 *   out        DEVICE fp32 [T][N]; zeroed by this call, then accumulated.
 */
int fp8_moe_gemm(const void* qa, const float* sa, const void* qw, const float* sw, const int32_t* offsets,
                 const int32_t* row_token, const float* row_weight, int64_t T, int64_t E, int64_t k, int64_t N,
                 int64_t K, float* out, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* fp8_status_string(int status);

/*
 * fp8_device_error -- synchronises `stream`, then reads and clears the
 * library's device-side error word on the current device.  Returns FP8_OK, or
 * FP8_ERR_TIMEOUT if a bounded wait in an earlier kernel ran out (that kernel
 * skipped its remaining work and returned), FP8_ERR_INVALID_SCALE if an earlier
 * fp8_mx_pack_pow2 was given a scale that is not a power of two, or FP8_ERR_CUDA.
 */
int fp8_device_error(void* stream);

/*
 * fp8_selftest_bounded_wait -- diagnostic with no counterpart in the pages.  Launches
 * one warp on `stream` whose mbarrier is never satisfied; the same bounded wait that
 * guards every pipelined wait of the GEMM kernels gives up after `limit_ns`
 * nanoseconds (0 < limit_ns <= 1e10, else FP8_ERR_INVALID_ARG), sets the device-side
 * error word and the kernel returns normally, so the CUDA context stays usable.  A
 * following fp8_device_error() returns FP8_ERR_TIMEOUT.  Returns the launch status.
 */
int fp8_selftest_bounded_wait(int64_t limit_ns, void* stream);

/*
 * fp8_set_wait_limit_ns -- diagnostic with no counterpart in the pages.  Sets the
 * limit of the bounded pipeline waits of the GEMM kernels on the current device to
 * `limit_ns` nanoseconds (0 restores the default of 2 s; 0 <= limit_ns <= 1e10, else
 * FP8_ERR_INVALID_ARG).  A limit under 1000 ns makes a GEMM give up at its first
 * wait whose first poll fails: the CTA raises its abort flag, every role leaves its loop,
 * the producer waits for the loads it has issued and each MMA issuer for its MMAs,
 * then tensor memory is freed and the kernel returns; fp8_device_error() then reports
 * FP8_ERR_TIMEOUT and the outputs of that call are unspecified.  Synchronous with
 * respect to the host; affects launches made after it returns.
 */
int fp8_set_wait_limit_ns(int64_t limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* FP8LIN_H */
