/*
 * nvfp4_moe.h — C ABI of the B200 (sm_100a) NVFP4 Mixture-of-Experts expert-FFN library.
 *
 * The operation is the MoE expert FFN of the nvfp4-megamoe-kernel pages:
 *   route -> quantize activations (NVFP4, global scale from amax on the GPU) ->
 *   L1 2D x 3D block-scaled grouped GEMM with SwiGLU and FP4 re-quantization in its epilogue ->
 *   L2 grouped GEMM with the routing weight and scatter-add in its epilogue.
 * ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", sections "Our Adaptation" and "Phase 3: Full MoE
 *  pipeline"; "May 24, 2026 — Session Start Plan", section 5 "NVFP4-1.1: Fuse FP4 into SwiGLU
 *  Epilogue".)
 *
 * Data formats
 *   NVFP4 tensor (rows x cols): E2M1 codes packed two per byte, row-major, element 2j in the low
 *   nibble of byte j (uint8 [rows][cols/2]); one E4M3 block scale per 16 consecutive elements of a
 *   row; one FP32 global scale gs.  Value = E2M1(code) * E4M3(scale) / gs.
 *   Block scales are stored TILED: the (rows x cols/16) scale matrix is cut into atoms of
 *   128 rows x 4 scale columns (512 bytes), atoms row-major over (rows/128, cols/64); inside an
 *   atom scale (r, c) is at byte (r%32)*16 + ((r/32)%4)*4 + c%4.  A scale buffer for R rows holds
 *   ceil(R/128)*128 * cols/16 bytes.
 *   Grouped ("2D x 3D") operands: activations A (R rows x K) whose rows are bucketed by expert,
 *   expert e owning rows [offs[e], offs[e+1]) (every offs a multiple of 128); weights B
 *   (E x N x K) as one NVFP4 tensor of E*N rows with a global scale per expert gs_b[e].
 *
 * Conventions (every call)
 *   - All pointers not marked "host" are device pointers, 16-byte aligned; the caller owns and
 *     allocates every buffer.  The library never allocates, never synchronizes the host (except
 *     nvfp4_read_status, which exists to do so) and never throws.
 *   - Work is enqueued on `stream`; arguments are checked on the host first and nothing is
 *     launched when a check fails.
 *   - dev_status (nullable): device int32 that kernels OR error bits into (NVFP4_DEVERR_*).
 *     Every wait inside a kernel is bounded; a wait that runs out sets NVFP4_DEVERR_TIMEOUT and
 *     the kernel returns instead of hanging.  Out-of-range routing ids set NVFP4_DEVERR_BAD_INDEX
 *     and are skipped.
 *   - Launch failures return NVFP4_ERR_CUDA; nvfp4_last_error() gives the CUDA error string.
 */
#ifndef NVFP4_MOE_H
#define NVFP4_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* same handle as cudaStream_t */

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2,
  NVFP4_ERR_MISALIGNED = 3,
  NVFP4_ERR_WORKSPACE_TOO_SMALL = 4,
  NVFP4_ERR_CUDA = 5,
  NVFP4_ERR_TIMEOUT = 6,
  NVFP4_ERR_BAD_INDEX = 7
} nvfp4_status_t;

/* Bits a kernel ORs into *dev_status. */
#define NVFP4_DEVERR_TIMEOUT 1
#define NVFP4_DEVERR_BAD_INDEX 2
#define NVFP4_DEVERR_BAD_OFFSETS 4

/* ---------------------------------------------------------------------------------------------
 * nvfp4_quantize — BF16 -> NVFP4 with the FP8-round-tripped block scale.
 *
 * Follows the commit log of dsv4/kernels/cuda (nvfp4-megamoe-kernel): the global scale "gsa" is
 * computed from amax on the GPU into a GPU buffer with no host sync ("Two-kernel approach":
 * amax kernel, then a quantize kernel that reads gsa from the buffer), and the element codes are
 * computed against the decoded FP8 block scale ("quantize must use the FP8-round-tripped block
 * scale").  NVFP4 itself: "May 24, 2026 — Session Start Plan", section 1 "NVFP4-0".
 *
 *   gs = 2688 / max|x| (1.0 if that is not finite and positive)            [compute_gs = 1]
 *   per 16-element block: s = (amax_b / 6) * gs ; scale = E4M3_rn_satfinite(s) ; d = decode(scale)
 *   code_i = E2M1_rn_satfinite(x_i * (gs / d))   (all-zero codes when d == 0)
 *
 *   x        bf16 [rows][ld] (ld >= cols, ld % 8 == 0)
 *   dst_row  NULL: row i goes to output row i (out_rows >= rows).  Otherwise int32 [rows*k]: row i
 *            is written to output rows dst_row[i*k + j], j < k; entries < 0 are skipped; entries
 *            >= out_rows set NVFP4_DEVERR_BAD_INDEX and are skipped.  (The permuted write of the
 *            MoE path: each token's codes go straight to its k expert rows.)
 *   codes    uint8 [out_rows][cols/2];  sf: tiled scales for out_rows rows (see top).
 *   gs       device float[1]: written when compute_gs = 1, read when compute_gs = 0.
 *   ws       device scratch of nvfp4_quantize_workspace_size() bytes (the amax word).
 *   Constraints: cols % 64 == 0, 0 <= rows <= 2^31 - 1, cols <= 268,431,360 (65535 chunks of 256
 *   blocks), k in [1, 64] when dst_row != NULL.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_quantize_workspace_size(void);
NVFP4_API nvfp4_status_t nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                              const int32_t* dst_row, int k, int64_t out_rows,
                              uint8_t* codes, uint8_t* sf, float* gs, int compute_gs,
                              void* ws, size_t ws_bytes, int32_t* dev_status,
                              nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * mxfp4_quantize — BF16 -> MXFP4: E2M1 elements with one UE8M0 (power-of-two) scale per 32
 * elements and no global scale: the format the pages contrast with NVFP4 ("May 24, 2026 —
 * Session Start Plan", section 1 "NVFP4-0": 32-element blocks, UE8M0 scales).  The pages give no
 * rounding rule; the OCP Microscaling v1.0 one is used:
 *
 *   e = floor(log2(max|x_i|)) - 2, clamped to [-127, 127] (-127 for an all-zero block)
 *   scale byte = e + 127;   code_i = E2M1_rn_satfinite(x_i * 2^-e)   (exact multiply)
 *   value = E2M1(code) * 2^(byte - 127)
 *
 *   x      bf16 [rows][ld] (ld >= cols, ld % 8 == 0)
 *   codes  uint8 [rows][cols/2] (element 2j in the low nibble of byte j)
 *   sf     scale bytes in the tiled layout of the NVFP4 scales (atoms of 128 rows x 4 scale
 *          columns), with cols/32 scale columns per row: ceil(rows/128)*128 * cols/32 bytes
 *   Constraints: cols % 128 == 0.  dev_status is unused (kept for a uniform signature).
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t mxfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                        uint8_t* codes, uint8_t* sf, int32_t* dev_status,
                                        nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * nvfp4_rmsnorm_quantize — RMSNorm fused in front of the BF16 -> NVFP4 quantizer.
 *
 * The commit log of dsv4/kernels/cuda (nvfp4-megamoe-kernel) fuses the RMSNorm with the amax and
 * the quantize (its kernel keeps the row's inverse RMS, s_inv_rms, beside the amax).  Reading:
 *
 *   ss = sum of x_i^2 over the row in float64;  ms = fl32(ss / cols);  rstd = 1 / sqrt_rn(ms + eps)
 *   y_i = fl32(fl32(x_i * rstd) * gamma_i)      (float32, one rounding per operation)
 *
 * then y is quantized exactly as nvfp4_quantize quantizes x (gs = 2688 / max|y| when
 * compute_gs = 1).  Two kernels: per-row rstd + the amax of y, then the quantize, which
 * normalizes each block as it loads it; the normalized tensor is never written.
 *
 *   gamma    bf16 [cols] (16-byte aligned);  eps >= 0
 *   ws       device scratch of nvfp4_rmsnorm_quantize_workspace_size(rows) bytes (the amax word
 *            and one float per row)
 *   everything else, the size limits included, as nvfp4_quantize.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_rmsnorm_quantize_workspace_size(int64_t rows);
NVFP4_API nvfp4_status_t nvfp4_rmsnorm_quantize(const void* x, int64_t rows, int64_t cols,
                              int64_t ld, const void* gamma, float eps,
                              const int32_t* dst_row, int k, int64_t out_rows,
                              uint8_t* codes, uint8_t* sf, float* gs, int compute_gs,
                              void* ws, size_t ws_bytes, int32_t* dev_status,
                              nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * moe_permute — top-k softmax routing and the expert-bucketed row map.
 *
 * The pages list "the MoE routing logic (top-k selection, slot mapping)" as work outside the
 * grouped GEMM ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section "Our Adaptation").  Reading:
 * the k largest logits of a token (ties to the lower expert id; a -inf logit is a dropped slot),
 * weights softmax(logits)[e], renormalized over the k when renormalize != 0.  Rows: experts in
 * ascending id, each segment padded to a multiple of 128 rows, slots inside a segment in
 * ascending (token, j).
 *
 *   logits    float [T][E], or NULL: topk_ids/topk_w are then INPUTS (ids < 0 = dropped slot)
 *   topk_ids  int32 [T][k] (output when logits != NULL); topk_w float [T][k] likewise
 *   offs      int32 [E+1]: start row of each expert's segment, offs[E] = rows used
 *   dst_row   int32 [T*k]: row of slot (t, j), -1 when dropped
 *   row_slot  int32 [R_max]: slot t*k + j of each row (its token is row_slot / k), -1 for padding
 *             and unused rows
 *   row_w     float [R_max]: routing weight of each row, 0 for padding and unused rows
 *   R_max     = moe_rows_max(T, E, k)
 *   ws        device scratch of moe_permute_workspace_size(T, E, k) bytes (4-byte aligned): from
 *             4096 slots the map is built by many CTAs, which exchange per-chunk expert counts
 *             there.  NULL or smaller: one CTA builds the same map (slower for large T*k).
 *   Constraints: 1 <= k <= E <= 256, k <= 32, T >= 0.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API int64_t moe_rows_max(int T, int E, int k);
NVFP4_API size_t moe_permute_workspace_size(int T, int E, int k);
NVFP4_API nvfp4_status_t moe_permute(const float* logits, int T, int E, int k, int renormalize,
                           int32_t* topk_ids, float* topk_w, int32_t* offs, int32_t* dst_row,
                           int32_t* row_slot, float* row_w, void* ws, size_t ws_bytes,
                           int32_t* dev_status, nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * nvfp4_grouped_gemm — plain 2D x 3D block-scaled grouped GEMM, C = A_e * B_e^T per expert.
 *
 * The grouped GEMM of "NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section "The Reference Kernel:
 * ScaledGroupedGemmKernel" (NVFP4: E2M1 + E4M3 per 16, 2D x 3D A(tokens,K) x B(experts,K,N)).
 * FP32 accumulation in tensor memory; C[r][n] = acc * 1/(gs_a * gs_b[e]).
 *
 *   a, sfa    NVFP4 [R_max][K] (tiled scales), gs_a device float[1]
 *   b, sfb    NVFP4 [E*N][K], gs_b device float[E]
 *   offs      device int32 [E+1], multiples of 128, offs[E] <= R_max
 *   out       [R_max][N], out_dtype 0 = float32, 1 = bf16; every row of every segment is written
 *             (rows of a segment beyond its real tokens hold whatever A's padding rows give)
 *   Constraints: K % 64 == 0, N % 256 == 0, R_max % 128 == 0, 1 <= E <= 256.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t nvfp4_grouped_gemm(const uint8_t* a, const uint8_t* sfa, const float* gs_a,
                                  const uint8_t* b, const uint8_t* sfb, const float* gs_b,
                                  const int32_t* offs, int E, int N, int K, int64_t R_max,
                                  void* out, int out_dtype, int32_t* dev_status,
                                  nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * mxfp4_grouped_gemm — the 2D x 3D grouped GEMM on MXFP4 operands (E2M1, one UE8M0 scale per 32
 * elements, no global scale; mxfp4_quantize's format), C = A_e * B_e^T per expert, FP32
 * accumulation: the variant of nvfp4_grouped_gemm for the format the pages contrast with NVFP4
 * ("May 24, 2026 — Session Start Plan", section 1 "NVFP4-0").  Same tiles, scheduler and
 * roles; the tensor cores read 2 scales per row per 64 of K (tcgen05.mma kind::mxf4,
 * scale_vec::2X).  C[r][n] = acc (no global scale to divide by).
 *
 *   a, sfa    MXFP4 [R_max][K] (codes [R_max][K/2], tiled scales with K/32 columns)
 *   b, sfb    MXFP4 [E*N][K]
 *   offs, out, out_dtype, R_max: as nvfp4_grouped_gemm
 *   Constraints: K % 128 == 0, N % 256 == 0, R_max % 128 == 0, 1 <= E <= 256.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t mxfp4_grouped_gemm(const uint8_t* a, const uint8_t* sfa,
                                            const uint8_t* b, const uint8_t* sfb,
                                            const int32_t* offs, int E, int N, int K,
                                            int64_t R_max, void* out, int out_dtype,
                                            int32_t* dev_status, nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * nvfp4_gemm_dense — dense block-scaled GEMM on NVFP4 activations: out = A W^T, bf16 out.
 *
 * The GEMM of the pages' dense layer (Nvfp4Linear; the shared expert), commit log of
 * dsv4/kernels/cuda (nvfp4-megamoe-kernel), on the grouped GEMM's core ("NVFP4 MegaMoE Kernel
 * Rewrite — CuTeDSL", section "The Reference Kernel: ScaledGroupedGemmKernel") with one dense
 * segment in place of expert offsets.
 *
 *   a, sfa    NVFP4 activations for round_up(M, 128) rows (codes [.][K/2], tiled scales);
 *             rows at or past M are padding: read, never stored, their content is irrelevant
 *   gs_a      device float[1]
 *   w, sfw    NVFP4 [N][K], gs_w device float[1]
 *   out       bf16 [M][N]:  out[m][n] = bf16( sum_k a[m][k] * w[n][k] / (gs_a * gs_w) )
 *   ws        device scratch of nvfp4_gemm_dense_workspace_size(M, N, K) bytes (0 = none
 *             needed): when M gives fewer output tiles than half the SMs, several CTAs share
 *             an output tile, each over one range of K, and their FP32 partial products are
 *             added afterwards in a fixed order (split-K; the result is reproducible)
 *   Constraints: K % 64 == 0, N % 256 == 0, M >= 0.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_gemm_dense_workspace_size(int64_t M, int N, int K);
NVFP4_API nvfp4_status_t nvfp4_gemm_dense(const uint8_t* a, const uint8_t* sfa,
                                          const float* gs_a, int64_t M, const uint8_t* w,
                                          const uint8_t* sfw, const float* gs_w, int N, int K,
                                          void* out, void* ws, size_t ws_bytes,
                                          int32_t* dev_status, nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * nvfp4_linear — dense NVFP4 linear: out = x W^T, bf16 in and out.
 *
 * The dense layer of the pages (Nvfp4Linear; the MoE shared expert's projections), commit log
 * of dsv4/kernels/cuda (nvfp4-megamoe-kernel), "Updated layers" of the fused amax + quantize
 * commit: the activation is quantized with a GPU-computed global scale (no host sync) and
 * multiplied by pre-packed NVFP4 weights.
 *
 *   x         bf16 [M][ld] (ld >= K, ld % 8 == 0)
 *   gamma     NULL, or bf16 [K]: x is first RMSNorm'd with gamma and eps (as in
 *             nvfp4_rmsnorm_quantize), fused into the quantizer
 *   w, sfw    NVFP4 [N][K] (codes [N][K/2], tiled scales), gs_w device float[1]
 *   out       bf16 [M][N]:  out[m][n] = bf16( sum_k xq[m][k] * wq[n][k] / (gs_x * gs_w) )
 *   ws        device scratch of nvfp4_linear_workspace_size(M, N, K) bytes: the quantized
 *             activation (rows padded to 128), its global scale and nvfp4_gemm_dense's
 *             partial products.  The steps are nvfp4_quantize (or nvfp4_rmsnorm_quantize) and
 *             nvfp4_gemm_dense.
 *   Constraints: K % 64 == 0, N % 256 == 0, M >= 0.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_linear_workspace_size(int64_t M, int N, int K);
NVFP4_API nvfp4_status_t nvfp4_linear(const void* x, int64_t M, int K, int64_t ld,
                                      const void* gamma, float eps, const uint8_t* w,
                                      const uint8_t* sfw, const float* gs_w, int N, void* out,
                                      void* ws, size_t ws_bytes, int32_t* dev_status,
                                      nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * nvfp4_shared_expert — the MoE shared expert: the expert FFN on every token, weight 1.
 *
 * The shared expert of the pages' model quantizes with a GPU-side gsa for both its projections
 * (commit log of dsv4/kernels/cuda, nvfp4-megamoe-kernel, "Updated layers": shared_expert.py).
 * Steps: [RMSNorm +] amax -> quantize -> L1 GEMM with SwiGLU and FP4 re-quantization in the
 * epilogue (moe_grouped_gemm_l1_swiglu_q's kernel, one dense segment) -> down projection
 * (nvfp4_gemm_dense) -> bf16.
 *
 *   x          bf16 [M][ld] (ld >= H, ld % 8 == 0); gamma NULL or bf16 [H] (RMSNorm, eps)
 *   w1, sfw1   NVFP4 [2I][H] in the gate/up interleave of moe_w1_row_map; gs_w1 device float[1]
 *   w2, sfw2   NVFP4 [H][I]; gs_w2 device float[1]
 *   gs_h       device float[1]: static global scale of the intermediate
 *   out        bf16 [M][H]
 *   ws         device scratch of nvfp4_shared_expert_workspace_size(M, H, I) bytes
 *   Constraints: H % 256 == 0, I % 128 == 0, M >= 0.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_shared_expert_workspace_size(int64_t M, int H, int I);
NVFP4_API nvfp4_status_t nvfp4_shared_expert(const void* x, int64_t M, int H, int64_t ld,
                                             const void* gamma, float eps, const uint8_t* w1,
                                             const uint8_t* sfw1, const float* gs_w1,
                                             const uint8_t* w2, const uint8_t* sfw2,
                                             const float* gs_w2, int I, const float* gs_h,
                                             void* out, void* ws, size_t ws_bytes,
                                             int32_t* dev_status, nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * moe_grouped_gemm_l1_swiglu_q — L1 grouped GEMM with SwiGLU and NVFP4 re-quantization fused in
 * the epilogue ("May 24, 2026 — Session Start Plan", section 5 "NVFP4-1.1": L1 GEMM -> SwiGLU ->
 * FP4 pack in registers -> FP4 GMEM).
 *
 *   W1 of expert e is [2I][H] with gate and up rows interleaved in blocks of 16: stored row
 *   32*j + i (i < 16) is gate row 16*j + i, stored row 32*j + 16 + i is up row 16*j + i
 *   (moe_w1_row_map gives the map; nvfp4_quantize applies it through dst_row at pre-pack).
 *   g = acc_gate / (gs_a*gs_w1[e]), u = acc_up / (gs_a*gs_w1[e]), h = g*u / (1 + exp(-g)) in
 *   FP32 (hardware exp2 and reciprocal: a few ulp), then quantized with the static global scale
 *   *gs_h by the same rule as nvfp4_quantize.
 *
 *   a, sfa, gs_a    activations NVFP4 [R_max][H]
 *   w1, sfw1, gs_w1 NVFP4 [E*2I][H], gs_w1 float[E]
 *   offs            int32 [E+1] (from moe_permute)
 *   row_slot        optional int32 [R_max] (from moe_permute).  NULL: every row of every segment
 *                   is written.  Given: groups of 32 rows that are all padding (row_slot < 0)
 *                   are skipped and their h rows left unwritten.
 *   gs_h            device float[1]
 *   h, sfh          output NVFP4 [R_max][I] (tiled scales)
 *   Constraints: H % 64 == 0, I % 128 == 0, R_max % 128 == 0, 1 <= E <= 256.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t moe_grouped_gemm_l1_swiglu_q(const uint8_t* a, const uint8_t* sfa, const float* gs_a,
                                            const uint8_t* w1, const uint8_t* sfw1,
                                            const float* gs_w1, const int32_t* offs,
                                            const int32_t* row_slot, int E, int H, int I,
                                            int64_t R_max, const float* gs_h, uint8_t* h,
                                            uint8_t* sfh, int32_t* dev_status,
                                            nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * moe_grouped_gemm_l1_swiglu_q_stats — moe_grouped_gemm_l1_swiglu_q, plus what its epilogue sees
 * of the intermediate h before quantizing it.
 *
 * The pages take every activation's global scale from its amax on the GPU (commit log of
 * dsv4/kernels/cuda, nvfp4-megamoe-kernel: the "Two-kernel approach" fix), but fuse h's
 * re-quantization into the L1 epilogue ("May 24, 2026 — Session Start Plan", section 5
 * "NVFP4-1.1"), where the amax of all of h is unknown when a tile is written.  This call records
 * that amax as the tiles are written, so that a later call can quantize with it (delayed
 * scaling, nvfp4_scale_from_amax), and counts the block scales the static scale could not hold.
 *
 *   h32      device float [R_max][I] or NULL: the FP32 h values (g*u/(1+exp(-g))) before
 *            quantization, for the real rows (row_slot >= 0, or every row when row_slot is NULL);
 *            other rows are not written.  A diagnostic output: it adds R_max*I*4 bytes of writes.
 *   h_stats  device uint32 [3] or NULL, ACCUMULATED into (zero it first): [0] = float bits of
 *            max|h| over the real rows (atomicMax on the bits, valid because |h| >= 0);
 *            [1] = block scales that saturated (s = (amax_b/6)*gs_h > 448); [2] = block scales
 *            that underflowed (amax_b > 0 but s rounded to the E4M3 zero: the block is all zeros).
 *   Everything else as moe_grouped_gemm_l1_swiglu_q.  h32 must be 16-byte aligned, h_stats 4.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t moe_grouped_gemm_l1_swiglu_q_stats(
    const uint8_t* a, const uint8_t* sfa, const float* gs_a, const uint8_t* w1,
    const uint8_t* sfw1, const float* gs_w1, const int32_t* offs, const int32_t* row_slot, int E,
    int H, int I, int64_t R_max, const float* gs_h, uint8_t* h, uint8_t* sfh, float* h32,
    uint32_t* h_stats, int32_t* dev_status, nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * nvfp4_scale_from_amax — *gs = 2688 / amax (1.0 when that is not finite and positive), amax
 * given as the float bits in *amax_bits: the global-scale rule of nvfp4_quantize applied to an
 * amax recorded earlier (h_stats[0] above), on the device, with no host sync.  One thread.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t nvfp4_scale_from_amax(const uint32_t* amax_bits, float* gs,
                                                nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * moe_w1_row_map — host helper: the stored row of each logical W1 row (gate rows [0, I), up rows
 * [I, 2I)) in the 16-row interleaved layout above.  map: host int32 [2I].  I % 16 == 0.
 * The pages deinterleave gate and up after the GEMM ("May 24, 2026 — Session Start Plan",
 * section 5 "NVFP4-1.1"); interleaving the weight rows instead puts each gate row next to its
 * up partner inside one accumulator tile, so the SwiGLU runs in the L1 epilogue.
 * Pure host computation, no CUDA call.  Pass the map (copied to the device) as dst_row with k = 1
 * to nvfp4_quantize when pre-packing an expert's W1.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t moe_w1_row_map(int I, int32_t* map);

/* ---------------------------------------------------------------------------------------------
 * moe_grouped_gemm_l2_scatter — L2 grouped GEMM with the routing weight and the scatter to token
 * order in its epilogue ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section "Our Adaptation":
 * "Scatter with routing weights"; section "Phase 3").
 *
 *   ys[s] = row_w[r] * (h_r . W2_e^T) / (gs_h*gs_w2[e]) for the row r of slot s (FP32), then
 *   out[t] = sum over j < k of ys[t*k + j], skipping dropped slots (dst_row < 0), added in j order
 *   in FP32 (bitwise reproducible); written as FP32 (out_f32) and/or bf16 (out_bf16, RN).
 *   Tokens whose slots are all dropped get exact zeros.
 *
 *   h, sfh, gs_h     NVFP4 [R_max][I]
 *   w2, sfw2, gs_w2  NVFP4 [E*H][I], gs_w2 float[E]
 *   offs, row_slot, row_w, dst_row  from moe_permute
 *   ys_ws            float [T*k][H] scratch (the weighted expert output of every slot)
 *   out_f32          float [T][H] or NULL;  out_bf16  bf16 [T][H] or NULL (not both NULL)
 *   Constraints: H % 256 == 0, I % 64 == 0, R_max % 128 == 0, 1 <= E <= 256, T >= 0, k >= 1.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t moe_grouped_gemm_l2_scatter(const uint8_t* h, const uint8_t* sfh, const float* gs_h,
                                           const uint8_t* w2, const uint8_t* sfw2,
                                           const float* gs_w2, const int32_t* offs,
                                           const int32_t* row_slot, const float* row_w,
                                           const int32_t* dst_row, int E, int H, int I, int T,
                                           int k, int64_t R_max, float* ys_ws, float* out_f32,
                                           void* out_bf16, int32_t* dev_status,
                                           nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * moe_grouped_gemm_l2_scatter_add — the L2 grouped GEMM with the routing weight and a true
 * scatter-ADD in its epilogue ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section "Our
 * Adaptation": "Scatter with routing weights"; section "Phase 3"): each routed row's weighted
 * output row_w[r] * (h_r . W2_e^T) / (gs_h*gs_w2[e]) is added into its token's row of an FP32
 * [T][H] accumulator as the tile is produced (vector reductions performed at L2), the tiles
 * running N-slice by N-slice so that the accumulator slice being added into stays in L2; then
 * the accumulator is rounded to bf16.
 *
 *   acc        float [T][H]: zeroed by this call (in stream order), holds the FP32 result after
 *   out_bf16   bf16 [T][H] or NULL
 *   The k additions into a token's row happen in whatever order the tiles finish, so the last
 *   bits of the FP32 sum (rarely a bf16 bit) may change from run to run; moe_grouped_gemm_l2_scatter
 *   is the bitwise-reproducible form.  Tokens whose slots are all dropped get exact zeros.
 *   Other arguments and constraints as moe_grouped_gemm_l2_scatter.
 *
 * moe_ffn_l2_form — which L2 form moe_ffn_forward(_ex) uses for a batch: 0 = per-slot rows summed
 * in slot order (moe_grouped_gemm_l2_scatter), 1 = token-row reductions (this call).  Host only.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t moe_grouped_gemm_l2_scatter_add(
    const uint8_t* h, const uint8_t* sfh, const float* gs_h, const uint8_t* w2,
    const uint8_t* sfw2, const float* gs_w2, const int32_t* offs, const int32_t* row_slot,
    const float* row_w, const int32_t* dst_row, int E, int H, int I, int T, int k, int64_t R_max,
    float* acc, void* out_bf16, int32_t* dev_status, nvfp4_stream_t stream);
NVFP4_API int moe_ffn_l2_form(int T, int k, int E, int flags);

/* ---------------------------------------------------------------------------------------------
 * moe_grouped_gemm_l2_scatter_noalloc — moe_grouped_gemm_l2_scatter without a caller-provided
 * FP32 accumulation buffer.  The pages have no counterpart to this call; it exists for callers
 * that cannot allocate device memory for scratch: runtimes that reserve all device memory up front
 * (weights, KV cache, a fixed activation pool) and forbid later cudaMalloc, or foreign-language
 * callers that are handed input and output buffers but have no device allocator of their own.
 *
 *   Same arguments and result as moe_grouped_gemm_l2_scatter, minus ys_ws and out_f32; out_bf16
 *   is required.  The FP32 per-slot buffer lives in a static device array inside this library of
 *   NVFP4_L2_NOALLOC_MAX_ELEMS floats (4 MiB), which every GPU that loads the library holds until
 *   the process exits.  T*k*H beyond that returns NVFP4_ERR_WORKSPACE_TOO_SMALL (nothing launched;
 *   nvfp4_last_error() says why).
 *   The array's device address is looked up once per device (cudaGetSymbolAddress) by the first
 *   call made with that device current; make that first call before any stream capture.  The
 *   library keeps that address for the life of the process: after cudaDeviceReset (or anything
 *   else that destroys the device's primary context) it is stale, so do not call this entry point
 *   on that device again in the same process.
 *   No cudaMalloc / cudaFree or allocating library routine is called.  All calls share the one
 *   array and every call rewrites the rows it reads back; calls that overlap on the GPU (other
 *   streams, other threads) race on it.
 * ------------------------------------------------------------------------------------------- */
#define NVFP4_L2_NOALLOC_MAX_ELEMS (1 << 20)
NVFP4_API nvfp4_status_t moe_grouped_gemm_l2_scatter_noalloc(
    const uint8_t* h, const uint8_t* sfh, const float* gs_h, const uint8_t* w2,
    const uint8_t* sfw2, const float* gs_w2, const int32_t* offs, const int32_t* row_slot,
    const float* row_w, const int32_t* dst_row, int E, int H, int I, int T, int k, int64_t R_max,
    void* out_bf16, int32_t* dev_status, nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * moe_ffn_forward — the whole expert FFN in one stream-ordered call, the pipeline of "NVFP4
 * MegaMoE Kernel Rewrite — CuTeDSL", section "Phase 3: Full MoE pipeline":
 *   moe_permute -> nvfp4_quantize (amax -> gs on the GPU, permuted write) ->
 *   moe_grouped_gemm_l1_swiglu_q -> L2 grouped GEMM + routing weight + scatter-add -> bf16 out.
 *   The scatter-add: below 32 routed rows per expert on average, per-slot rows summed in slot
 *   order (moe_grouped_gemm_l2_scatter); from there, FP32 vector reductions into each token's
 *   row as the L2 tiles are produced, whose order is not fixed (moe_ffn_forward_ex with
 *   NVFP4_FFN_DETERMINISTIC keeps the slot-ordered sum at every size).
 *
 *   x_bf16   bf16 [T][H];  logits float [T][E] (softmax top-k routing, renormalized)
 *   w1.. / w2..  expert weights as above; gs_h device float[1] (static intermediate scale)
 *   out_bf16 bf16 [T][H]; tokens whose slots are all dropped get exact zeros.
 *   ws       device scratch of moe_ffn_workspace_size(T, H, I, E, k) bytes (256-byte aligned)
 *   Constraints: those of the four calls above.
 * ------------------------------------------------------------------------------------------- */
NVFP4_API size_t moe_ffn_workspace_size(int T, int H, int I, int E, int k);
NVFP4_API nvfp4_status_t moe_ffn_forward(const void* x_bf16, const float* logits, int T, int H, int I, int E,
                               int k, const uint8_t* w1, const uint8_t* sfw1, const float* gs_w1,
                               const uint8_t* w2, const uint8_t* sfw2, const float* gs_w2,
                               const float* gs_h, void* out_bf16, void* ws, size_t ws_bytes,
                               int32_t* dev_status, nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * moe_ffn_forward_ex — moe_ffn_forward with options: the intermediate's statistics, an opt-in
 * delayed global scale for h (see moe_grouped_gemm_l1_swiglu_q_stats for why h's scale is not
 * dynamic), and the choice of a bitwise-reproducible output sum.
 *
 *   gs_h     device float[1], the scale this call quantizes h with
 *   flags    0, or an OR of:
 *            NVFP4_FFN_DELAYED_GS_H  after this call's L2 has used it, *gs_h is replaced, in
 *                stream order, by 2688 / max|h| of this call (1.0 when not finite and positive):
 *                call i+1 then quantizes h with call i's amax.  The first call uses the scale the
 *                caller wrote.  Without it *gs_h is only read (a static scale).
 *            NVFP4_FFN_DETERMINISTIC  every slot's weighted row is stored and a token's k rows
 *                are added in slot order, so the output is bitwise reproducible.  Without it,
 *                from 32 routed rows per expert on average, the rows are added into the token's
 *                FP32 row as the L2 tiles produce them (vector reductions at L2; no per-slot round
 *                trip through memory): the order of those k additions, and so the last bits of
 *                the FP32 sum (rarely a bf16 output bit), may change from run to run.
 *   h_stats  device uint32[3] or NULL: zeroed by the call, then filled as in
 *            moe_grouped_gemm_l1_swiglu_q_stats (amax bits, saturated, underflowed).
 *   Everything else as moe_ffn_forward (same workspace size).  moe_ffn_forward is this call
 *   with flags = 0 and no statistics.
 * ------------------------------------------------------------------------------------------- */
#define NVFP4_FFN_DELAYED_GS_H 1
#define NVFP4_FFN_DETERMINISTIC 2
NVFP4_API nvfp4_status_t moe_ffn_forward_ex(const void* x_bf16, const float* logits, int T, int H,
                                  int I, int E, int k, const uint8_t* w1, const uint8_t* sfw1,
                                  const float* gs_w1, const uint8_t* w2, const uint8_t* sfw2,
                                  const float* gs_w2, float* gs_h, int flags, uint32_t* h_stats,
                                  void* out_bf16, void* ws, size_t ws_bytes, int32_t* dev_status,
                                  nvfp4_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Status helpers.
 *   nvfp4_read_status: copies *dev_status to *host_code (host pointer) on `stream` and waits for
 *   the stream; returns NVFP4_ERR_TIMEOUT / NVFP4_ERR_BAD_INDEX when the matching bit is set.
 *   nvfp4_last_error: the last CUDA error string seen by this library on this thread.
 * ------------------------------------------------------------------------------------------- */
/* ---------------------------------------------------------------------------------------------
 * nvfp4_wait_selftest — diagnostic (no counterpart in the pages): runs one CTA whose first warp
 * waits, with the library's bounded wait and a limit of limit_ns, on an mbarrier that nothing
 * arrives on.  When the wait runs out it raises the CTA's abort flag; a second warp waiting on
 * another such barrier (default 2 s limit) must then give up early, as the grouped GEMM's roles
 * do; NVFP4_DEVERR_TIMEOUT is ORed into *dev_status.  No fault, no trap, no unbounded wait: it
 * checks the timeout path on a GPU and leaves the context usable.
 *   limit_ns    1 .. 2e9
 *   elapsed_ns  optional device uint64: time from the start of the waits to the report
 * ------------------------------------------------------------------------------------------- */
NVFP4_API nvfp4_status_t nvfp4_wait_selftest(int64_t limit_ns, int32_t* dev_status,
                                             uint64_t* elapsed_ns, nvfp4_stream_t stream);

NVFP4_API nvfp4_status_t nvfp4_read_status(const int32_t* dev_status, int32_t* host_code,
                                 nvfp4_stream_t stream);
NVFP4_API const char* nvfp4_last_error(void);
NVFP4_API int nvfp4_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_MOE_H */
