/*
 * quads.h -- C ABI of libquads.so: the NVFP4 Mixture-of-Experts expert layer
 * of RL rollout/trainer alignment, as hand-written CUDA for sm_100a (B200).
 *
 * Sources cited below by short tag:
 *   [QUADS-fr] "QUADS: Stabilizing NVFP4 Reinforcement Learning for MoE via
 *              QUantization-error Alignment across Dual Sides", gist.science
 *              French summary, "Résumé Technique" sections 1-5.
 *   [QUADS-es] the same paper, gist.science Spanish summary, sections 1-5.
 *   [TRACE]    "TRACE : un entraînement conscient de la quantification guidé
 *              par le rollout pour le RL en FP4 des modèles MoE", sns.style.
 *   [format]   the public NVFP4 format: E2M1 elements, one E4M3 scale per 16
 *              consecutive elements along K, one FP32 per-tensor scale.
 *
 * Conventions (all entry points):
 *   - Pointers named in comments as "device" point to GPU memory owned by the
 *     caller; the library keeps no reference after the call is enqueued.
 *     The library allocates no memory: calls that need scratch take a
 *     caller-provided workspace whose size a *_workspace_bytes() query gives.
 *   - Every call is asynchronous on the given stream (NULL = legacy default
 *     stream) and does not synchronize, except quads_device_status().
 *   - BF16 tensors are passed as uint16_t bit patterns; E2M1 codes are packed
 *     two per byte (element 2j in the low nibble of byte j); E4M3 block scales
 *     are one byte each.
 *   - Scale layouts: QUADS_SCALES_LINEAR = [rows][K/16] row-major;
 *     QUADS_SCALES_TILED = the tensor-core layout: tiles of 128 rows x 4
 *     scales (512 bytes) in row-major tile order, rows padded to a multiple
 *     of 128 and K/16 to a multiple of 4 with zero scales; inside a tile row r
 *     and scale column c sit at byte (r % 32) * 16 + (r / 32) * 4 + c.
 *     quads_scales_bytes() gives the size of either layout.
 *   - Arguments are validated on the host before anything is launched. A
 *     negative return value is an error; quads_last_error() (thread-local)
 *     describes the last one.  Launch failures return QUADS_ERR_CUDA.
 *   - The per-tensor scale g is a decode scale: value = e2m1 * e4m3 * g, with
 *     g = fp32(amax / 2688) (2688 = 6 * 448).  Element codes are
 *     E2M1_RNE(fp32(x * fp32(1 / fp32(e4m3 * g)))) and the block scale is
 *     E4M3_RN_satfinite(fp32(amax_block / fp32(6 * g))).  A block whose scale
 *     is 0 gets signed-zero codes.  Inputs must be finite; a tensor amax must
 *     be 0 or at least 2^-100.
 */
#ifndef QUADS_H
#define QUADS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* quads_stream_t;   /* a cudaStream_t */

enum {
  QUADS_OK = 0,
  QUADS_ERR_INVALID_ARG = -1,       /* null pointer, negative or inconsistent size, misalignment */
  QUADS_ERR_UNSUPPORTED_SHAPE = -2, /* a size outside what the kernels support */
  QUADS_ERR_CUDA = -3,              /* a CUDA runtime/launch error */
  QUADS_ERR_TIMEOUT = -4,           /* a bounded device-side wait gave up */
  QUADS_ERR_BAD_RECORD = -5         /* a TRACE record failed validation */
};

enum { QUADS_SCALES_LINEAR = 0, QUADS_SCALES_TILED = 1 };
enum { QUADS_OUT_BF16 = 0, QUADS_OUT_F32 = 1 };

/* Message of the last error on this thread ("" if none). */
const char* quads_last_error(void);
/* ABI version of this header (1). */
int quads_abi_version(void);
/* Number of kernels this library has launched in this process. */
uint64_t quads_launch_count(void);
/* Synchronizes the stream, then returns QUADS_ERR_TIMEOUT if a kernel of this
 * library recorded a timed-out wait on the current device since the last call
 * (and clears the record), QUADS_OK otherwise. */
int quads_device_status(quads_stream_t stream);
/* Self-test of the bounded waits: launches one block that waits on a barrier
 * nothing will complete, with the given limit in nanoseconds (<= 10 s); the
 * wait gives up, records a timeout and the kernel returns.  A following
 * quads_device_status() returns QUADS_ERR_TIMEOUT. */
int quads_selftest_bounded_wait(uint64_t timeout_ns, quads_stream_t stream);
/* Output tile of the grouped FP4 GEMMs with the BF16 correction (or none)
 * and N % 256 == 0 (a tuning and testing switch, not a reading of the pages):
 *   0  128 x 128 on one CTA, the correction in its own FP32 accumulator;
 *   1  128 x 256 on one CTA (the default);
 *   2  256 x 256 on a pair of CTAs (tcgen05 cta_group::2, each CTA loads
 *      its own half of the rows and of the weight rows).
 * Shapes 1 and 2 accumulate the correction into the FP4 accumulator as
 * (R / G) . Wc, with R / G = bf16(fp32(R * fp32(1 / G))) and G = g_a g_w[e].
 * Other FP4 GEMMs (the FP4 correction, N % 256 != 0) always take shape 0.
 * The W4A16 GEMMs take their tensor-memory kernel under shapes 1 and 2
 * (N % 256 == 0) and the 128 x N kernel under shape 0.
 * Returns the previous shape, or QUADS_ERR_INVALID_ARG for another value.
 * Process-wide; not synchronized with launches in flight. */
int quads_gemm_set_tile_shape(int shape);
/* Decode tiles for the same GEMMs when they carry no fused quantization:
 * the weights become the MMA's M operand (128 weight rows on the TMEM
 * lanes) and the expert's rows its N operand (128 per tile); each tile
 * computes 256 weight rows (for SwiGLU: 128 gate rows and the matching
 * 128 up rows, so SwiGLU needs no exchange between TMEM lanes).
 * Taken when N % 256 == 0 and the average rows per expert,
 * max(0, rows_cap / 128 - E) * 128 / E, is at most `rows` (default 64);
 * 0 never takes it.  The correction is folded as in shapes 1 and 2.  A
 * tuning and testing switch, not a reading of the pages.  Returns the
 * previous value, or QUADS_ERR_INVALID_ARG for a negative one.
 * Process-wide; not synchronized with launches in flight. */
int quads_gemm_set_decode_rows(int rows);

/* SM budget for kernels launched afterwards (from any host thread), so that
 * an HBM-bound stream and the tensor-core GEMMs can run side by side on
 * disjoint SMs.  With 0 < n < the device's SM count:
 *   - the persistent grouped GEMMs (every tile shape, the decode tiles and
 *     the W4A16 GEMM) launch at most n CTAs (n / 2 CTA pairs);
 *   - quads_fakequant_weight_ste_backward, whose CTAs each request more
 *     than half of an SM's shared memory (one CTA per SM), launches n of
 *     them instead of one per SM of the device.
 * A persistent GEMM CTA needs all of an SM's shared memory, so the two
 * never share an SM: launched on concurrent streams with budgets n_gemm
 * and n_ste, n_gemm + n_ste <= the SM count, they split the GPU.  Results do
 * not depend on the budget.  n = 0 (or n >= the SM count) restores the
 * default: grids sized to the whole device.  Returns the previous budget,
 * or QUADS_ERR_INVALID_ARG for n < 0.  Process-wide; read at launch (and so
 * at CUDA graph capture) time. */
int quads_set_sm_budget(int n);

/* Bytes of a scale array of `rows` x K/16 scales in the given layout. */
size_t quads_scales_bytes(int64_t rows, int64_t K, int scale_layout);

/* ---------------------------------------------------------------- a1: amax
 * Per-group max |x| of a BF16 matrix (the tensor statistic behind the FP32
 * per-tensor scale, [format]).  Rows are split into groups either by
 * group_off (device int32 [n_groups + 1], ascending, group_off[0] = 0; rows
 * at or past group_off[n_groups] belong to no group and are not read) or,
 * when group_off is NULL, into n_groups groups of rows / n_groups rows each.
 * amax_out: device float[n_groups], overwritten.  K % 16 == 0, ld_x >= K,
 * ld_x % 8 == 0, x 16-byte aligned. */
int quads_amax_bf16(const uint16_t* x, int64_t rows, int64_t K, int64_t ld_x,
                    const int32_t* group_off, int n_groups, float* amax_out,
                    quads_stream_t stream);

/* ------------------------------------------------- a2 + a3: NVFP4 quantize
 * NVFP4-quantizes a BF16 matrix x [rows][K] (row stride ld_x elements) with
 * one per-tensor scale per row group (see quads_amax_bf16 for groups).
 * [TRACE] "Fonctionnement": block scaling, one 4-bit value per element, the
 * rounding direction a discrete choice; [format] block = 16 elements along
 * K, E4M3 scale, FP32 tensor scale; [QUADS-fr §2.2.B] the residual of the
 * high-residual channels feeds the rollout's compensation.
 *   amax_in   device float[n_groups] calibrated amax, or NULL: the amax is
 *             computed from x first (needs the workspace).
 *   codes     device uint8 [rows][K/2], packed E2M1.
 *   scales    device uint8, quads_scales_bytes(rows, K, scale_layout) bytes.
 *   g_out     device float[n_groups]: the per-tensor decode scales.
 *   chan      device int32[n_chan] or NULL: the compensation channels, valid
 *             entries (0 <= c < K) strictly ascending and first, then -1
 *             padding.  n_chan <= 256.
 *   resid_out device uint16 (BF16) [rows][n_chan] or NULL:
 *             r = bf16(fp32(x - fp32(deq(q(x))))) on each channel, 0 on padding.
 *   ws        device workspace of quads_quantize_workspace_bytes(n_groups)
 *             bytes (may be NULL when amax_in is given).
 * Constraints: K % 16 == 0, K <= 65536, n_groups >= 1 (<= 1024 with
 * group_off), rows >= 0.  With rows == 0 only g_out is written (zeros) and
 * codes and scales may be NULL. */
size_t quads_quantize_workspace_bytes(int n_groups);
int quads_quantize_nvfp4(const uint16_t* x, int64_t rows, int64_t K, int64_t ld_x,
                         const int32_t* group_off, int n_groups, const float* amax_in,
                         uint8_t* codes, uint8_t* scales, int scale_layout, float* g_out,
                         const int32_t* chan, int n_chan, uint16_t* resid_out,
                         void* ws, size_t ws_bytes, quads_stream_t stream);

/* The same quantization as quads_quantize_nvfp4, for callers that cannot
 * give this library any device memory beyond their inputs and outputs: code
 * whose GPU memory is all owned by another allocator (a framework's pool, an
 * arena sized once at start-up), plugin interfaces with no way to pass a
 * workspace, latency-critical loops that cannot afford an allocation.  The
 * pages have no counterpart: this is a deployment convenience, not a step of
 * the method.
 *   - It allocates nothing and takes no workspace.  The one scratch it needs
 *     (one FP32 amax per row group, used when amax_in is NULL) lives in a
 *     4 KiB file-scope device array that every GPU which loads the library
 *     holds until the process exits.
 *   - n_groups <= 1024; larger requests return QUADS_ERR_UNSUPPORTED_SHAPE
 *     before anything is launched.  All other arguments and limits are those
 *     of quads_quantize_nvfp4.
 *   - The first call with a given device and CUDA context current looks up
 *     the array's device address there (cudaGetSymbolAddress) and caches it
 *     for that device and context; make that first call before any stream
 *     capture.  A device reset (cudaDeviceReset) unloads the array and the
 *     context it comes back with can carry the same handle, so the cached
 *     address is not valid after a reset: a process that resets a device
 *     must not call this entry point on it again.
 *   - Every call reuses the same array and clears it before use.  Calls that
 *     can run at the same time on one GPU (other streams, other host threads)
 *     race on it: serialize them. */
int quads_quantize_nvfp4_noalloc(const uint16_t* x, int64_t rows, int64_t K, int64_t ld_x,
                                 const int32_t* group_off, int n_groups, const float* amax_in,
                                 uint8_t* codes, uint8_t* scales, int scale_layout, float* g_out,
                                 const int32_t* chan, int n_chan, uint16_t* resid_out,
                                 quads_stream_t stream);

/* --------------------------------------------------------------- dequant
 * deq = e2m1 * e4m3 * g of a quantized matrix (the rollout's weight or
 * activation as the trainer sees it, [QUADS-fr §2.1]).  g: device
 * float[n_groups] (groups as in quads_amax_bf16).  out: device BF16 or FP32
 * [rows][K] per out_dtype (QUADS_OUT_BF16 rounds the FP32 value to BF16). */
int quads_dequant(const uint8_t* codes, const uint8_t* scales, int scale_layout,
                  const float* g, const int32_t* group_off, int n_groups,
                  int64_t rows, int64_t K, void* out, int out_dtype,
                  quads_stream_t stream);

/* ---------------------------------------------- calibration of the channels
 * [QUADS-fr §2.2.B]: a binary mask picks the channels with the largest
 * residual magnitude.  scores: device float[K], score_c = sum over rows of
 * |fp32(x - fp32(deq(q(x))))| for the tensor's own quantization (amax_in as
 * in quads_quantize_nvfp4), summed in a fixed order.  Needs
 * quads_channel_scores_workspace_bytes(rows, K) bytes of workspace. */
size_t quads_channel_scores_workspace_bytes(int64_t rows, int64_t K);
int quads_channel_scores(const uint16_t* x, int64_t rows, int64_t K, const float* amax_in,
                         float* scores, void* ws, size_t ws_bytes, quads_stream_t stream);
/* The n_sel channels with the largest score (ties: lower index), written to
 * chan_out (device int32[n_sel]) in ascending channel order.  K <= 16384. */
int quads_select_channels(const float* scores, int64_t K, int n_sel, int32_t* chan_out,
                          quads_stream_t stream);

/* ------------------------------------------------------------ a4: router
 * Top-k experts per token from FP32 logits [T][E] (E <= 256, k <= 8,
 * k <= E): experts ordered by (logit desc, index asc).  topk_w = softmax
 * over the k selected logits (renorm = 1) or the full softmax at the
 * selected experts (renorm = 0).  The router's choice is discrete
 * ([TRACE] "Fonctionnement").  topk_idx: device int32 [T][k]; topk_w:
 * device float [T][k]. */
int quads_moe_router_topk(const float* logits, int64_t T, int E, int k, int renorm,
                          int32_t* topk_idx, float* topk_w, quads_stream_t stream);

/* ------------------------------------------------------- a5: permutation
 * Stable counting sort of the (token, slot) pairs by expert, in increasing
 * token * k + slot order, each expert's segment padded to a multiple of 128
 * rows.  Outputs (device): expert_off int32[E + 1]; row_of int32[T * k] (the
 * expert-ordered row of each pair); src_of int32[rows_cap] (the token of each
 * expert-ordered row, -1 on pad rows; rows >= expert_off[E] are untouched).
 * rows_cap = quads_moe_rows_capacity(T, k, E) bounds expert_off[E].
 * Workspace: quads_moe_permute_workspace_bytes(T, k, E). */
int64_t quads_moe_rows_capacity(int64_t T, int k, int E);
size_t quads_moe_permute_workspace_bytes(int64_t T, int k, int E);
int quads_moe_permute(const int32_t* topk_idx, int64_t T, int k, int E,
                      int32_t* expert_off, int32_t* row_of, int32_t* src_of,
                      void* ws, size_t ws_bytes, quads_stream_t stream);
/* Gathers the quantized activation rows into expert order: pa_codes
 * [rows_cap][K/2], pa_scales (tiled layout over rows_cap rows) and pa_resid
 * [rows_cap][n_chan] from a_codes [T][K/2], a_scales (linear layout) and
 * a_resid [T][n_chan] (both resid pointers NULL when n_chan == 0).  Pad rows
 * get zero codes, scales and residuals.  K % 64 == 0. */
int quads_moe_gather(const int32_t* src_of, const int32_t* expert_off, int E, int64_t rows_cap,
                     const uint8_t* a_codes, const uint8_t* a_scales, int64_t K,
                     const uint16_t* a_resid, int n_chan,
                     uint8_t* pa_codes, uint8_t* pa_scales, uint16_t* pa_resid,
                     quads_stream_t stream);
/* Gathers BF16 rows into expert order: out[p] = x[src_of[p]] for
 * p < expert_off[E], zeros on pad rows (src_of[p] == -1); rows >= expert_off[E]
 * are untouched.  x [T][H], out [rows_cap][H], both 16-byte aligned,
 * H % 8 == 0.  The trainer's BF16 activations for the W4A16 GEMMs
 * ([QUADS-fr §2.2.A]: the trainer keeps BF16 activations). */
int quads_moe_gather_bf16(const int32_t* src_of, const int32_t* expert_off, int E, int64_t rows_cap,
                          const uint16_t* x, int64_t H, uint16_t* out, quads_stream_t stream);
/* Router + permutation + gather in one call (same arguments as above). */
int quads_moe_route_permute(const float* logits, int64_t T, int E, int k, int renorm,
                            int32_t* topk_idx, float* topk_w, int32_t* expert_off,
                            int32_t* row_of, int32_t* src_of, int64_t rows_cap,
                            const uint8_t* a_codes, const uint8_t* a_scales, int64_t K,
                            const uint16_t* a_resid, int n_chan,
                            uint8_t* pa_codes, uint8_t* pa_scales, uint16_t* pa_resid,
                            void* ws, size_t ws_bytes, quads_stream_t stream);

/* -------------------------------- a6: NVFP4 grouped GEMM + compensation
 * For every expert e and its rows [off[e], off[e+1]) of the expert-ordered
 * activations ([QUADS-fr §1] native W4A4 GEMM; [QUADS-fr §2.2.B] the
 * residual correction added to the quantized output):
 *   Y[r][n] = g_a(e) * g_w[e] * sum_k e2m1(A)e4m3(A) * e2m1(W_e)e4m3(W_e)
 *           + sum_j a_resid[r][j] * w_resid[e][n][j]
 * accumulated in FP32 on the tensor cores (tcgen05 block-scaled FP4 MMA for
 * the first term, BF16 MMA for the second), stored as BF16.
 *   a_codes  [rows_cap][K/2], a_scales tiled over rows_cap rows;
 *   g_a      device float[E] if g_a_per_expert else float[1];
 *   w_codes  [E][N][K/2] (row n = output feature n), w_scales tiled over
 *            E*N rows; g_w device float[E];
 *   expert_off device int32[E + 1], 128-row aligned, expert_off[E] <= rows_cap;
 *   a_resid  [rows_cap][n_chan] BF16, w_resid [E][N][n_chan] BF16 (both NULL
 *            when n_chan == 0);
 *   y        [rows_cap][N] BF16; rows >= expert_off[E] are untouched.
 * Constraints: 1 <= E <= 256, N % 128 == 0, K % 64 == 0, rows_cap % 128 == 0,
 * n_chan % 16 == 0, n_chan <= 128; all matrix pointers 16-byte aligned.
 * A device wait that exceeds ~4 s records a timeout (quads_device_status). */
int quads_moe_grouped_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales,
                                 const float* g_a, int g_a_per_expert,
                                 const uint8_t* w_codes, const uint8_t* w_scales, const float* g_w,
                                 const int32_t* expert_off, int E, int64_t rows_cap,
                                 int64_t N, int64_t K,
                                 const uint16_t* a_resid, const uint16_t* w_resid, int n_chan,
                                 uint16_t* y, quads_stream_t stream);

/* a6 + a7 in one pass ([QUADS-fr §1]: the rollout's MoE expert GEMMs in
 * NVFP4; the SwiGLU expert FFN is a reading, the pages name no activation):
 * the gate/up grouped GEMM with the SwiGLU applied in the epilogue.  The operands are those of quads_moe_grouped_gemm_nvfp4 with
 * N = 2F, except that the W rows (w_codes, w_scales, w_resid) are in the
 * 64-row interleaved gate/up order that quads_fakequant_weight_ste_gate_up
 * writes.  Each 128-row tile then holds gate rows 64b..64b+63 followed by the
 * matching up rows.  Writes
 *   h[r][f] = bf16(silu(y_gate[r][f]) * y_up[r][f]),
 * where y_gate and y_up are the BF16 GEMM outputs exactly as
 * quads_moe_grouped_gemm_nvfp4 would store them.  SwiGLU is computed in FP32
 * as in quads_swiglu.  h is [rows_cap][F] BF16.  amax_out (device float[E],
 * nullable, overwritten) receives the per-expert max |h|.  F % 64 == 0. */
int quads_moe_grouped_gemm_nvfp4_swiglu(const uint8_t* a_codes, const uint8_t* a_scales,
                                        const float* g_a, int g_a_per_expert,
                                        const uint8_t* w_codes, const uint8_t* w_scales,
                                        const float* g_w, const int32_t* expert_off, int E,
                                        int64_t rows_cap, int64_t F, int64_t K,
                                        const uint16_t* a_resid, const uint16_t* w_resid,
                                        int n_chan, uint16_t* h, float* amax_out,
                                        quads_stream_t stream);

/* The literal second quantization pass ([QUADS-fr §2.2.B]: the correction
 * on the high-residual channels is a second quantization pass added to the
 * quantized output): the residual channels R and the weights' channel
 * columns Wc are NVFP4 operands, multiplied on the FP4 tensor cores in the
 * same accumulator as the main product:
 *   y = bf16(G_e * (sum_k a w + sum_c q(r) q(wc)))   (NVFP4 values)
 * r_codes [rows_cap][Kc/2] and r_scales (tiled over rows_cap x Kc) are R
 * quantized per expert segment with amax_r from quads_moe_fp4_comp_amax;
 * wc_codes [E*N][Kc/2] and wc_scales (tiled over E*N x Kc) are Wc quantized
 * per expert with its own amax.  Kc % 64 == 0, Kc <= 1024 (pad channel
 * columns with zeros); everything else as quads_moe_grouped_gemm_nvfp4 with
 * n_chan = 0.  The SwiGLU variant is quads_moe_grouped_gemm_nvfp4_swiglu with
 * this correction. */
int quads_moe_grouped_gemm_nvfp4_fp4comp(const uint8_t* a_codes, const uint8_t* a_scales,
                                         const float* g_a, int g_a_per_expert,
                                         const uint8_t* w_codes, const uint8_t* w_scales,
                                         const float* g_w, const int32_t* expert_off, int E,
                                         int64_t rows_cap, int64_t N, int64_t K,
                                         const uint8_t* r_codes, const uint8_t* r_scales,
                                         const uint8_t* wc_codes, const uint8_t* wc_scales,
                                         int64_t Kc, uint16_t* y, quads_stream_t stream);
int quads_moe_grouped_gemm_nvfp4_swiglu_fp4comp(const uint8_t* a_codes, const uint8_t* a_scales,
                                                const float* g_a, int g_a_per_expert,
                                                const uint8_t* w_codes, const uint8_t* w_scales,
                                                const float* g_w, const int32_t* expert_off, int E,
                                                int64_t rows_cap, int64_t F, int64_t K,
                                                const uint8_t* r_codes, const uint8_t* r_scales,
                                                const uint8_t* wc_codes, const uint8_t* wc_scales,
                                                int64_t Kc, uint16_t* h, float* amax_out,
                                                quads_stream_t stream);
/* Trainer-side W4A16 grouped GEMM ([QUADS-fr §2.2.A]: the trainer keeps BF16
 * activations and multiplies them by its fake-quantized weights):
 *   y[r][n] = bf16(sum_k x[r][k] * W_fq[e][n][k]),  FP32 accumulation,
 *   W_fq = bf16(fp32(val(q) * val(s)) * g_w[e])  (the folded fake-quant),
 * for every row r of expert e's segment, with the weights read as their
 * NVFP4 codes w_codes [E*N][K/2] and tiled scales (what
 * quads_fakequant_weight_ste writes with want_codes) and dequantized on
 * chip, so W_fq is never stored.  x [rows_cap][K] BF16, 16-byte aligned;
 * other arguments as quads_moe_grouped_gemm_nvfp4.  The SwiGLU variant
 * writes h [rows_cap][F] from weights in the 64-row interleaved gate/up order
 * (N = 2F) and the per-expert max |h| (amax_out, nullable).  Where N % 256
 * == 0 (and the tile shape is not 0) W_fq is converted into tensor memory
 * and read there by the MMA (units of 128 weight rows by up to 256 rows);
 * otherwise, or with tile shape 0, it is converted into shared memory. */
int quads_moe_grouped_gemm_w4a16(const uint16_t* x, const uint8_t* w_codes, const uint8_t* w_scales,
                                 const float* g_w, const int32_t* expert_off, int E,
                                 int64_t rows_cap, int64_t N, int64_t K, uint16_t* y,
                                 quads_stream_t stream);
int quads_moe_grouped_gemm_w4a16_swiglu(const uint16_t* x, const uint8_t* w_codes,
                                        const uint8_t* w_scales, const float* g_w,
                                        const int32_t* expert_off, int E, int64_t rows_cap,
                                        int64_t F, int64_t K, uint16_t* h, float* amax_out,
                                        quads_stream_t stream);

/* Per-expert amax of the residual operand above, chosen so that its decode
 * scale times g_wc[e] is G_e = fp32(g_a g_w[e]) up to one rounding:
 * amax_r[e] = fp32(fp32(G_e / g_wc[e]) * 2688), 0 where g_wc[e] == 0.
 * g_a is device float[E] when g_a_per_expert, else float[1]; all device. */
int quads_moe_fp4_comp_amax(const float* g_a, int g_a_per_expert, const float* g_w,
                            const float* g_wc, int E, float* amax_r, quads_stream_t stream);

/* a6 + a7 + the re-quantization of h in one pass ([QUADS-fr §1]: the down
 * GEMM's input is NVFP4 too): the SwiGLU GEMM above whose epilogue also
 * NVFP4-quantizes h for the down projection.  Each
 * expert uses the decode scale g_e = fp32(amax_h_in[e] / 2688), computed from
 * an amax given in advance (calibrated, or the previous step's: delayed
 * scaling).  Written:
 *   h_codes  [rows_cap][F/2], h_scales tiled over rows_cap x F,
 *   h_resid  [rows_cap][n_chan_h] BF16 residuals on chan_h (ascending valid
 *            channels first, then -1; 0 on padding slots), NULL if n_chan_h = 0,
 *   g_h_out  device float[E] = g_e.
 * Rows below expert_off[E] are quantized, including the zero pad rows of
 * each expert's segment.  The values written are those quads_quantize_nvfp4
 * writes for this h with group_off = expert_off, amax_in = amax_h_in, the
 * tiled layout and chan_h.  amax_h_out (nullable, overwritten) receives
 * this h's per-expert max |h| (the next step's amax_h_in), and h (nullable)
 * receives h itself in BF16.  F % 64 == 0, n_chan_h <= 256. */
int quads_moe_grouped_gemm_nvfp4_swiglu_quant(const uint8_t* a_codes, const uint8_t* a_scales,
                                              const float* g_a, int g_a_per_expert,
                                              const uint8_t* w_codes, const uint8_t* w_scales,
                                              const float* g_w, const int32_t* expert_off, int E,
                                              int64_t rows_cap, int64_t F, int64_t K,
                                              const uint16_t* a_resid, const uint16_t* w_resid,
                                              int n_chan, const float* amax_h_in,
                                              const int32_t* chan_h, int n_chan_h, uint8_t* h_codes,
                                              uint8_t* h_scales, uint16_t* h_resid, float* g_h_out,
                                              float* amax_h_out, uint16_t* h, quads_stream_t stream);

/* --------------------------------------------------------- a7: SwiGLU
 * (reading: the pages name no activation; SwiGLU is the plainest MoE FFN)
 * h[r][j] = bf16(silu(Y[r][j]) * Y[r][F + j]) for rows r < expert_off[E],
 * silu(v) = v / (1 + exp(-v)), computed in FP32 from the BF16 gate/up GEMM
 * output y [rows_cap][2F].  amax_out (device float[E], nullable, overwritten)
 * receives the per-expert max |h| for the re-quantization of h.  F % 8 == 0. */
int quads_swiglu(const uint16_t* y, int64_t rows_cap, int64_t F,
                 const int32_t* expert_off, int E, uint16_t* h, float* amax_out,
                 quads_stream_t stream);

/* --------------------------------------------------------- a8: combine
 * ([TRACE] "Fonctionnement": the router's discrete choice of experts; the
 * weighted sum of the k expert outputs is the plainest reading)
 * out[t] = bf16(sum over s = 0..k-1 of topk_w[t][s] * Y[row_of[t*k + s]]),
 * FP32 accumulation in slot order.  y [rows_cap][H], out [T][H], H % 8 == 0. */
int quads_moe_unpermute_combine(const uint16_t* y, const int32_t* row_of, const float* topk_w,
                                int64_t T, int k, int64_t H, uint16_t* out,
                                quads_stream_t stream);

/* ------------------------------------------ a9: weight fake-quant + STE
 * [QUADS-fr §2.2.A] asymmetric W4A16 QAT: the trainer's forward sees its
 * BF16 master weights fake-quantized onto the rollout's NVFP4 grid
 * ([QUADS-fr §2.1]: the same quantize-dequantize path as the rollout).  One
 * pass over n_mat matrices [rows][K] (one per-tensor scale each) writes:
 *   w_fq     BF16 [n_mat][rows][K]: bf16(e2m1 * e4m3 * g) if fold_global,
 *            else the exact e2m1 * e4m3 (g then applies to the matmul output);
 *   codes    (nullable) packed E2M1 [n_mat][rows][K/2] -- the rollout's
 *            weights, identical to quads_quantize_nvfp4 of the same matrix;
 *   scales   (nullable) tiled layout over n_mat * rows rows (rows % 128 == 0)
 *            or linear when rows % 128 != 0;
 *   g_out    device float[n_mat];
 *   w_chan   (nullable) BF16 [n_mat][rows][n_chan]: the compensation weight
 *            operand, column chan[j] of bf16(deq(W)) (chan_raw = 0) or of the
 *            input W itself (chan_raw = 1); 0 on padding channels.
 *   amax_in  device float[n_mat] per-matrix amax (e.g. from quads_amax_bf16),
 *            or NULL: computed first, which needs the workspace of
 *            quads_quantize_workspace_bytes(n_mat) bytes. */
int quads_fakequant_weight_ste(const uint16_t* w, int64_t n_mat, int64_t rows, int64_t K,
                               const float* amax_in, int fold_global, uint16_t* w_fq,
                               uint8_t* codes, uint8_t* scales, float* g_out,
                               const int32_t* chan, int n_chan, int chan_raw, uint16_t* w_chan,
                               void* ws, size_t ws_bytes, quads_stream_t stream);
/* The same pass for gate/up weight matrices [n_mat][rows][K] whose first
 * rows / 2 rows are the gate projection and the rest the up projection
 * (rows % 128 == 0).  w_fq keeps the input row order.  codes, scales
 * (tiled) and w_chan are written with each matrix's rows interleaved in blocks
 * of 64: gate rows 64b..64b+63 go to rows 128b..128b+63, and up rows
 * 64b..64b+63 go to rows 128b+64..128b+127.  That way every 128-row tile of
 * the rollout's weights holds matching gate and up rows.  This is the operand
 * layout of quads_moe_grouped_gemm_nvfp4_swiglu. */
int quads_fakequant_weight_ste_gate_up(const uint16_t* w, int64_t n_mat, int64_t rows, int64_t K,
                                       const float* amax_in, int fold_global, uint16_t* w_fq,
                                       uint8_t* codes, uint8_t* scales, float* g_out,
                                       const int32_t* chan, int n_chan, int chan_raw, uint16_t* w_chan,
                                       void* ws, size_t ws_bytes, quads_stream_t stream);
/* Straight-through backward ([QUADS-fr §2.2.A]: the QAT trainer's gradient
 * passes through the weight fake-quant): grad_w = grad_wfq (accumulate = 0) or
 * grad_w = bf16(fp32(grad_w + grad_wfq)) (accumulate = 1); n BF16 elements,
 * both arrays 16-byte aligned.  One CTA per SM streams 16 KB chunks of both
 * through a shared-memory ring (see quads_set_sm_budget). */
int quads_fakequant_weight_ste_backward(const uint16_t* grad_wfq, uint16_t* grad_w, int64_t n,
                                        int accumulate, quads_stream_t stream);

/* ------------------------------------------- a10 + a11: TRACE record
 * [TRACE] "L'idée centrale": the rollout records its quantization results of
 * the deep layers (mantissa and scale factors) and the trainer reproduces
 * that rounding; "Impact": the engine exports, the trainer consumes.
 *
 * One record per layer: a header followed by 256-byte aligned sections.  A
 * record holds up to two quantized tensors (slot 0: the gate/up GEMM input
 * X in token order; slot 1: the down GEMM input h in expert order) and the
 * router's top-k indices.  All offsets are bytes from the record start. */
#define TRACE_QRECORD_MAGIC 0x31434552u   /* "REC1" little-endian */
#define TRACE_QRECORD_VERSION 1u
#define TRACE_MAX_TENSORS 2

typedef struct trace_qtensor_desc {
  int64_t rows, K;
  int32_t n_groups;        /* per-tensor scales (1, or one per expert) */
  int32_t n_chan;          /* compensation channels (0: none) */
  int32_t scale_layout;    /* QUADS_SCALES_LINEAR / QUADS_SCALES_TILED */
  int32_t present;         /* 1 if this slot holds a tensor */
  uint64_t codes_off, scales_off, g_off, group_off_off, chan_off, resid_off;
  uint64_t codes_bytes, scales_bytes;
} trace_qtensor_desc;

typedef struct trace_qrecord_header {
  uint32_t magic, version;
  int32_t layer_id;
  int32_t k;               /* experts per token (0: no routing section) */
  int64_t T;               /* tokens */
  uint64_t total_bytes;
  uint64_t topk_idx_off;   /* int32 [T][k] */
  trace_qtensor_desc t[TRACE_MAX_TENSORS];
} trace_qrecord_header;

/* What one slot of a record holds, as device pointers (all owned by the
 * caller): codes, scales, g[n_groups], group_off[n_groups + 1] (NULL when
 * n_groups == 1), chan[n_chan] and resid[rows][n_chan] (NULL when
 * n_chan == 0). */
typedef struct trace_qtensor_src {
  int64_t rows, K;
  int32_t n_groups, n_chan, scale_layout, present;
  const uint8_t* codes;
  const uint8_t* scales;
  const float* g;
  const int32_t* group_off;
  const int32_t* chan;
  const uint16_t* resid;
} trace_qtensor_src;

/* Fills *hdr (host memory) with the layout of a record for these tensors and
 * returns its total size in bytes (0 on invalid arguments).  Only the sizes
 * in `tensors` are read (the pointers may be NULL), so a producer can place
 * its outputs at the returned offsets of the record before exporting. */
size_t trace_qrecord_layout(int layer_id, int64_t T, int k,
                            const trace_qtensor_src* tensors, int n_tensors,
                            trace_qrecord_header* hdr);
/* Writes the record (header + copies of every section) into `record`
 * (device, record_bytes >= trace_qrecord_layout(...), 256-byte aligned).
 * topk_idx: device int32 [T][k] or NULL when k == 0.  A section whose source
 * pointer already equals its place in the record (a producer that wrote its
 * output into the record) is not copied. */
int trace_export_qrecord(int layer_id, int64_t T, int k, const int32_t* topk_idx,
                         const trace_qtensor_src* tensors, int n_tensors,
                         void* record, size_t record_bytes, quads_stream_t stream);
/* Trainer replay of slot `which` of a record (device memory) ([TRACE]
 * "Fonctionnement": the trainer reads the record during its forward pass and
 * reproduces the rollout's rounding):
 *   x_hat [rows][K] BF16 = bf16(fp32(deq) + r) on the compensation channels,
 *         bf16(deq) elsewhere -- the operand the rollout's compensated GEMM
 *         effectively used;
 *   x_train (nullable) BF16 [rows][K]: the trainer's own activation; its
 *         quantization with the recorded per-tensor scale is compared with
 *         the record, and the numbers of differing element codes and block
 *         scales are added to counts[0] and counts[1] (device uint64[2]).
 * The record is validated on the device (magic, version, layer id, slot,
 * shape, bounds within record_bytes); a bad record writes nothing and sets
 * *status (device int32) to QUADS_ERR_BAD_RECORD, else *status = 0. */
int trace_replay_qrecord(const void* record, size_t record_bytes, int layer_id, int which,
                         int64_t rows, int64_t K, const uint16_t* x_train,
                         uint16_t* x_hat, unsigned long long* counts, int32_t* status,
                         quads_stream_t stream);

/* ------------------------------- compact record: rounding directions
 * [TRACE] "Fonctionnement, côté ingénierie": on a block-scaled FP4 grid each
 * value's rounding (up to the grid point above or down to the one below) is
 * a discrete choice, and the trainer uses the rollout's record to make the
 * same choice; [TRACE] "L'idée centrale": the cache is kept small.
 *
 * One bit per element replaces the 4-bit code; the block scales and the
 * per-tensor scale(s) are kept as they are.  With S = fp32(val(s) g) and
 * y = fp32(x * fp32(1/S)), level(y) is the index (0..7) of the largest E2M1
 * level (0, .5, 1, 1.5, 2, 3, 4, 6) at or below |y|.
 *
 * trace_direction_bits: bit = 1 where the rollout's code magnitude index is
 * above level(y) of its own input x (it rounded up), else 0; 0 in blocks
 * with S == 0.  x [rows][K] BF16 and codes [rows][K/2] are the rollout's
 * quantizer input and output, scales are in scale_layout, g is device
 * float[n_groups] over row groups (group_off as in quads_quantize_nvfp4;
 * rows past group_off[n_groups] are skipped).  bits: device [rows][K/8],
 * element 8j + i in bit i of byte j.
 *
 * trace_replay_direction: the trainer's guided rounding of x_train:
 * code = sign(y_t) | min(level(y_t) + bit, 7) (signed zeros where S == 0),
 * x_hat = bf16(fp32(val(code) val(s) g)), and on the compensation channels
 * chan (ascending valid channels first, then -1) x_hat = bf16(fp32(deq) + r)
 * with r = resid [rows][n_chan] BF16.  codes_out (nullable) receives the
 * guided codes [rows][K/2]; *corrections (device u64, nullable, accumulated)
 * counts the elements where the guided code differs from the trainer's own
 * nearest-even rounding with the recorded scale.  Where x_train lies between
 * the same two levels as the rollout's x, the guided code is the rollout's.
 * K % 16 == 0, n_groups <= 1024, n_chan <= 256; x, x_train, x_hat 16-byte
 * aligned, codes 8-byte, bits 2-byte. */
int trace_direction_bits(const uint16_t* x, int64_t rows, int64_t K, const uint8_t* codes,
                         const uint8_t* scales, int scale_layout, const float* g,
                         const int32_t* group_off, int n_groups, uint8_t* bits,
                         quads_stream_t stream);
int trace_replay_direction(const uint8_t* bits, const uint8_t* scales, int scale_layout,
                           const float* g, const int32_t* group_off, int n_groups, int64_t rows,
                           int64_t K, const uint16_t* x_train, const int32_t* chan, int n_chan,
                           const uint16_t* resid, uint16_t* x_hat, uint8_t* codes_out,
                           unsigned long long* corrections, quads_stream_t stream);

/* ------------------------------------------------------ layer stacking
 * The pages describe the MoE layer, not the model around it; a stack of
 * layers is joined here in the plainest way: x_{l+1} = x_l + MoE_l(x_l), and
 * the router logits of layer l are x_l . W_r[l].
 *
 * Router logits: logits[t][e] = sum over h of x[t][h] * w_r[h][e], one FP32
 * FMA chain per output in increasing h.  x: device BF16 [T][H]; w_r: device
 * FP32 [H][E] (row-major); logits: device FP32 [T][E].  1 <= E <= 4096. */
int quads_router_logits(const uint16_t* x, int64_t T, int64_t H, const float* w_r, int E,
                        float* logits, quads_stream_t stream);
/* Residual connection: out[i] = bf16(fp32(x[i]) + fp32(y[i])) for n BF16
 * elements (n % 8 == 0, all three 16-byte aligned; out may alias x or y). */
int quads_residual_add(const uint16_t* x, const uint16_t* y, int64_t n, uint16_t* out,
                       quads_stream_t stream);
/* n floats copied device to device by a kernel (not a copy engine): the
 * delayed-scaling amax handed from one step to the next inside a captured
 * step, where a copy-engine copy would queue behind host transfers. */
int quads_copy_f32(const float* src, float* dst, int64_t n, quads_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* QUADS_H */
