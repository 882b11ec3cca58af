// ffn.cu — moe_ffn_forward (the whole expert FFN, stream-ordered), its workspace layout, and
// the status / error helpers of the C ABI.
//
// Pipeline ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section "Phase 3: Full MoE pipeline";
// "May 24, 2026 — Session Start Plan", section 5 "NVFP4-1.1"):
//   topk + permute  ->  amax -> quantize (permuted write)  ->  L1 GEMM + SwiGLU + FP4 pack
//   ->  L2 GEMM + routing weight, per-slot rows  ->  combine (k-sum per token) + bf16
// No host synchronization anywhere; every intermediate lives in the caller's workspace.
#include <cstdio>

#include "common.cuh"
#include "launch.h"

namespace nvfp4 {

namespace {
thread_local char g_last_error[256] = "";
}

void set_last_error(const char* msg) { std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

nvfp4_status_t check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return NVFP4_OK;
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
  return NVFP4_ERR_CUDA;
}

// Byte offsets of the moe_ffn_forward workspace regions (each 256-byte aligned).
struct FfnLayout {
  int64_t amax, gs_x, ids, w, offs, dst_row, row_slot, row_w, hist, xq, xsf, hq, hsf, ys, hstats;
  int64_t total;
  int64_t R_max;
};

FfnLayout ffn_layout(int T, int H, int I, int E, int k) {
  FfnLayout L{};
  const int64_t S = (int64_t)T * k;
  L.R_max = moe_rows_max(T, E, k);
  int64_t o = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = o;
    o = round_up(o + bytes, 256);
    return at;
  };
  L.amax = take(4);
  L.gs_x = take(4);
  L.ids = take(S * 4);
  L.w = take(S * 4);
  L.offs = take((int64_t)(E + 1) * 4);
  L.dst_row = take(S * 4);
  L.row_slot = take(L.R_max * 4);
  L.row_w = take(L.R_max * 4);
  L.hist = take((int64_t)permute_workspace_bytes(T, E, k));
  L.xq = take(L.R_max * H / 2);
  L.xsf = take(L.R_max * H / 16);
  L.hq = take(L.R_max * I / 2);
  L.hsf = take(L.R_max * I / 16);
  L.ys = take(S * H * 4);
  L.hstats = take(3 * 4);
  L.total = o;
  return L;
}

// The next call's global scale of h from this call's amax (delayed scaling): 2688 / amax,
// 1.0 when that is not finite and positive.
__global__ void scale_from_amax_kernel(const uint32_t* amax_bits, float* gs) {
  if (threadIdx.x == 0) *gs = gs_from_amax(__uint_as_float(*amax_bits));
}

nvfp4_status_t ffn_forward(const void* x_bf16, const float* logits, int T, int H, int I, int E,
                           int k, const uint8_t* w1, const uint8_t* sfw1, const float* gs_w1,
                           const uint8_t* w2, const uint8_t* sfw2, const float* gs_w2,
                           float* gs_h, int flags, uint32_t* h_stats, void* out_bf16, void* ws,
                           size_t ws_bytes, int32_t* dev_status, nvfp4_stream_t stream) {
  if (T < 0 || E < 1 || E > 256 || k < 1 || k > 32 || k > E || H <= 0 || I <= 0)
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (H % 256 || I % 128) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)T * k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (flags & ~(NVFP4_FFN_DELAYED_GS_H | NVFP4_FFN_DETERMINISTIC)) return NVFP4_ERR_INVALID_ARG;
  const bool delayed = (flags & NVFP4_FFN_DELAYED_GS_H) != 0;
  if (T == 0) return NVFP4_OK;
  if (!x_bf16 || !logits || !w1 || !sfw1 || !gs_w1 || !w2 || !sfw2 || !gs_w2 || !gs_h ||
      !out_bf16 || !ws)
    return NVFP4_ERR_INVALID_ARG;
  const FfnLayout L = ffn_layout(T, H, I, E, k);
  if (ws_bytes < static_cast<size_t>(L.total)) return NVFP4_ERR_WORKSPACE_TOO_SMALL;
  const void* ptrs16[] = {x_bf16, w1, sfw1, w2, sfw2, out_bf16};
  for (const void* p : ptrs16)
    if (!aligned16(p)) return NVFP4_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) || (reinterpret_cast<uintptr_t>(logits) & 3u) ||
      (reinterpret_cast<uintptr_t>(h_stats) & 3u))
    return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  auto i32 = [&](int64_t off) { return reinterpret_cast<int32_t*>(base + off); };
  auto f32 = [&](int64_t off) { return reinterpret_cast<float*>(base + off); };
  // statistics of h: the caller's words, or the workspace's when only the delayed scale needs them
  uint32_t* stats = h_stats != nullptr ? h_stats
                    : delayed ? reinterpret_cast<uint32_t*>(base + L.hstats) : nullptr;

  nvfp4_status_t st = permute_launch(logits, T, E, k, 1, i32(L.ids), f32(L.w), i32(L.offs),
                                     i32(L.dst_row), i32(L.row_slot), f32(L.row_w), L.R_max,
                                     permute_workspace_bytes(T, E, k) ? i32(L.hist) : nullptr,
                                     dev_status, s);
  if (st != NVFP4_OK) return st;
  st = quantize_launch(x_bf16, T, H, H, i32(L.dst_row), k, L.R_max, base + L.xq, base + L.xsf,
                       f32(L.gs_x), 1, base + L.amax, dev_status, s);
  if (st != NVFP4_OK) return st;
  if (stats != nullptr && cudaMemsetAsync(stats, 0, 3 * sizeof(uint32_t), s) != cudaSuccess)
    return check_launch("cudaMemsetAsync(h_stats)");
  st = gemm_l1(base + L.xq, base + L.xsf, f32(L.gs_x), w1, sfw1, gs_w1, i32(L.offs),
               i32(L.row_slot), E, H, I, L.R_max, gs_h, base + L.hq, base + L.hsf, nullptr, stats,
               dev_status, s);
  if (st != NVFP4_OK) return st;
  st = gemm_l2(base + L.hq, base + L.hsf, gs_h, w2, sfw2, gs_w2, i32(L.offs), i32(L.row_slot),
               f32(L.row_w), i32(L.dst_row), E, H, I, T, k, L.R_max, f32(L.ys), nullptr,
               out_bf16, l2_use_atomic(T, k, E, (flags & NVFP4_FFN_DETERMINISTIC) != 0),
               dev_status, s);
  if (st != NVFP4_OK || !delayed) return st;
  // stream order: the L2 above has read this call's gs_h before it is replaced
  scale_from_amax_kernel<<<1, 32, 0, s>>>(stats, gs_h);
  return check_launch("scale_from_amax_kernel");
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" size_t moe_ffn_workspace_size(int T, int H, int I, int E, int k) {
  if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0) return 0;
  return static_cast<size_t>(ffn_layout(T, H, I, E, k).total);
}

extern "C" nvfp4_status_t moe_ffn_forward(const void* x_bf16, const float* logits, int T, int H,
                                          int I, int E, int k, const uint8_t* w1,
                                          const uint8_t* sfw1, const float* gs_w1,
                                          const uint8_t* w2, const uint8_t* sfw2,
                                          const float* gs_w2, const float* gs_h, void* out_bf16,
                                          void* ws, size_t ws_bytes, int32_t* dev_status,
                                          nvfp4_stream_t stream) {
  // static scale (gs_h is only read), the fastest L2 form for the batch
  return ffn_forward(x_bf16, logits, T, H, I, E, k, w1, sfw1, gs_w1, w2, sfw2, gs_w2,
                     const_cast<float*>(gs_h), 0, nullptr, out_bf16, ws, ws_bytes, dev_status,
                     stream);
}

extern "C" nvfp4_status_t moe_ffn_forward_ex(const void* x_bf16, const float* logits, int T,
                                             int H, int I, int E, int k, const uint8_t* w1,
                                             const uint8_t* sfw1, const float* gs_w1,
                                             const uint8_t* w2, const uint8_t* sfw2,
                                             const float* gs_w2, float* gs_h, int flags,
                                             uint32_t* h_stats, void* out_bf16, void* ws,
                                             size_t ws_bytes, int32_t* dev_status,
                                             nvfp4_stream_t stream) {
  return ffn_forward(x_bf16, logits, T, H, I, E, k, w1, sfw1, gs_w1, w2, sfw2, gs_w2, gs_h, flags,
                     h_stats, out_bf16, ws, ws_bytes, dev_status, stream);
}

extern "C" nvfp4_status_t nvfp4_scale_from_amax(const uint32_t* amax_bits, float* gs,
                                                nvfp4_stream_t stream) {
  if (!amax_bits || !gs) return NVFP4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(amax_bits) & 3u) || (reinterpret_cast<uintptr_t>(gs) & 3u))
    return NVFP4_ERR_MISALIGNED;
  scale_from_amax_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(amax_bits, gs);
  return check_launch("scale_from_amax_kernel");
}

extern "C" nvfp4_status_t nvfp4_read_status(const int32_t* dev_status, int32_t* host_code,
                                            nvfp4_stream_t stream) {
  if (!dev_status || !host_code) return NVFP4_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host_code, dev_status, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return check_launch("nvfp4_read_status");
  if (*host_code & NVFP4_DEVERR_TIMEOUT) return NVFP4_ERR_TIMEOUT;
  if (*host_code & (NVFP4_DEVERR_BAD_INDEX | NVFP4_DEVERR_BAD_OFFSETS)) return NVFP4_ERR_BAD_INDEX;
  return NVFP4_OK;
}

extern "C" const char* nvfp4_last_error(void) { return g_last_error; }

extern "C" int nvfp4_abi_version(void) { return 1; }

extern "C" nvfp4_status_t moe_w1_row_map(int I, int32_t* map) {
  if (I <= 0 || I % 16 != 0 || map == nullptr) return NVFP4_ERR_INVALID_ARG;
  for (int p = 0; p < 2 * I; ++p) {
    const int up = p >= I, r = up ? p - I : p;  // logical gate or up row r
    map[p] = 32 * (r / 16) + 16 * up + (r % 16);
  }
  return NVFP4_OK;
}
