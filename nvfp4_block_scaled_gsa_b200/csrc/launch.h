// launch.h — host-side launch helpers shared by the library's .cu files (internal; not part of
// the C ABI).  Each validates nothing: the extern "C" entry points check their arguments first.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4_moe.h"

namespace nvfp4 {

nvfp4_status_t quantize_launch(const void* x, int64_t rows, int64_t cols, int64_t ld,
                               const int32_t* dst_row, int k, int64_t out_rows, uint8_t* codes,
                               uint8_t* sf, float* gs, int compute_gs, void* ws,
                               int32_t* dev_status, cudaStream_t s);
nvfp4_status_t rmsnorm_quantize_launch(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                       const void* gamma, float eps, const int32_t* dst_row,
                                       int k, int64_t out_rows, uint8_t* codes, uint8_t* sf,
                                       float* gs, int compute_gs, void* ws, int32_t* dev_status,
                                       cudaStream_t s);
nvfp4_status_t permute_launch(const float* logits, int T, int E, int k, int renorm,
                              int32_t* topk_ids, float* topk_w, int32_t* offs, int32_t* dst_row,
                              int32_t* row_slot, float* row_w, int64_t R_max, int32_t* hist_ws,
                              int32_t* dev_status, cudaStream_t s);
size_t permute_workspace_bytes(int T, int E, int k);

nvfp4_status_t gemm_dense(const uint8_t* a, const uint8_t* sfa, const float* gs_a,
                          const uint8_t* b, const uint8_t* sfb, const float* gs_b, int64_t M, int N,
                          int K, void* out_bf16, float* part, int64_t part_floats, int32_t* status,
                          cudaStream_t s);
int dense_k_splits(int64_t M, int N, int K, int sms, int64_t part_floats);
int device_sms();
nvfp4_status_t gemm_dense_parts(const uint8_t* a, const uint8_t* sfa, const float* gs_a,
                                const uint8_t* b, const uint8_t* sfb, const float* gs_b,
                                int64_t M, int N, int K, int ks, float* part, int32_t* status,
                                cudaStream_t s);

// L1 grouped GEMM + SwiGLU + NVFP4 re-quantization.  h32 (optional): the FP32 h values before
// quantization, [R_max][I].  h_stats (optional, device uint32[3], accumulated): amax bits of |h|
// over real rows (atomicMax), block scales saturated above 448, block scales underflowed to 0.
nvfp4_status_t gemm_l1(const uint8_t* a, const uint8_t* sfa, const float* gs_a, const uint8_t* w1,
                       const uint8_t* sfw1, const float* gs_w1, const int32_t* offs,
                       const int32_t* row_slot, int E, int H, int I, int64_t R_max,
                       const float* gs_h, uint8_t* h, uint8_t* sfh, float* h32,
                       uint32_t* h_stats, int32_t* status, cudaStream_t s);
// L2 grouped GEMM + routing weight + scatter to token order.  atomic = false: each slot's
// weighted row goes to ys [T*k][H] and a combine kernel sums a token's rows in slot order
// (bitwise reproducible).  atomic = true: the rows are added into an FP32 [T][H] accumulator
// (out_f32 if given, else ys) as they are produced, then rounded to bf16; the order of the
// additions, and so the last bits of the sum, may change from run to run.
nvfp4_status_t gemm_l2(const uint8_t* h, const uint8_t* sfh, const float* gs_h, const uint8_t* w2,
                       const uint8_t* sfw2, const float* gs_w2, const int32_t* offs,
                       const int32_t* row_slot, const float* row_w, const int32_t* dst_row, int E,
                       int H, int I, int T, int k, int64_t R_max, float* ys, float* out_f32,
                       void* out_bf16, bool atomic, int32_t* status, cudaStream_t s);
bool l2_use_atomic(int T, int k, int E, bool deterministic);

}  // namespace nvfp4
