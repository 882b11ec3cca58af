// linear.cu — dense NVFP4 linear, y = x W^T, with the activation quantized on the fly and an
// optional RMSNorm fused into that quantizer.
//
// The pages' dense layer (Nvfp4Linear, and the shared expert's two projections) quantizes its
// bf16 activation with a GPU-computed global scale and runs an NVFP4 GEMM against pre-packed
// weights (commit log of dsv4/kernels/cuda, nvfp4-megamoe-kernel: the "Updated layers" of the
// fused amax + quantize commit).  Here: [RMSNorm +] amax -> quantize -> the grouped GEMM core
// with one dense segment (split along K when the output has too few tiles to fill the SMs).
#include "common.cuh"

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
nvfp4_status_t gemm_dense(const uint8_t* a, const uint8_t* sfa, const float* gs_a,
                          const uint8_t* b, const uint8_t* sfb, const float* gs_b, int64_t M, int N,
                          int K, void* out_bf16, float* part, int64_t part_floats, int32_t* status,
                          cudaStream_t s);
int dense_k_splits(int64_t M, int N, int K, int sms, int64_t part_floats);

namespace {

// The SM count the workspace is sized for; on a device with more SMs the split is clamped to
// what the workspace holds.
constexpr int kSizingSms = 148;

// FP32 partial products the dense GEMM may use (split-K), sized for kSizingSms.
int64_t dense_part_floats(int64_t M, int N, int K) {
  const int ks = dense_k_splits(M, N, K, kSizingSms, INT64_MAX / 4);
  return ks > 1 ? ks * M * (int64_t)N : 0;
}

// Byte offsets of the nvfp4_linear workspace regions (each 256-byte aligned).
struct LinearLayout {
  int64_t quant_ws, gs, codes, sf, part, total;
  int64_t part_floats;
};

LinearLayout linear_layout(int64_t M, int N, int K) {
  LinearLayout L{};
  const int64_t Mp = round_up(M, 128);
  int64_t o = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = o;
    o += round_up(bytes, 256);
    return at;
  };
  L.quant_ws = take(static_cast<int64_t>(nvfp4_rmsnorm_quantize_workspace_size(M)));
  L.gs = take(4);
  L.codes = take(Mp * (K / 2));
  L.sf = take(Mp * (K / 16));
  L.part_floats = dense_part_floats(M, N, K);
  L.part = take(L.part_floats * 4);
  L.total = o;
  return L;
}

}  // namespace
}  // namespace nvfp4

extern "C" size_t nvfp4_gemm_dense_workspace_size(int64_t M, int N, int K) {
  if (M < 0 || N <= 0 || K <= 0) return 0;
  return static_cast<size_t>(nvfp4::dense_part_floats(M, N, K) * 4);
}

extern "C" nvfp4_status_t nvfp4_gemm_dense(const uint8_t* a, const uint8_t* sfa,
                                           const float* gs_a, int64_t M, const uint8_t* w,
                                           const uint8_t* sfw, const float* gs_w, int N, int K,
                                           void* out, void* ws, size_t ws_bytes,
                                           int32_t* dev_status, nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (M < 0 || N <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
  if (K % 64 || N % 256) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t)INT32_MAX - 127) return NVFP4_ERR_UNSUPPORTED_SHAPE;  // rows index as int
  if (!gs_a || !w || !sfw || !gs_w) return NVFP4_ERR_INVALID_ARG;
  if (M > 0 && (!a || !sfa || !out)) return NVFP4_ERR_INVALID_ARG;
  const int64_t need = dense_part_floats(M, N, K) * 4;
  if (need > 0 && (ws == nullptr || (int64_t)ws_bytes < need)) return NVFP4_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(a) || !aligned16(sfa) || !aligned16(w) || !aligned16(sfw) || !aligned16(out) ||
      !aligned16(ws) || (reinterpret_cast<uintptr_t>(gs_a) & 3u) ||
      (reinterpret_cast<uintptr_t>(gs_w) & 3u))
    return NVFP4_ERR_MISALIGNED;
  if (M == 0) return NVFP4_OK;
  return gemm_dense(a, sfa, gs_a, w, sfw, gs_w, M, N, K, out, static_cast<float*>(ws),
                    need / 4, dev_status, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t nvfp4_linear_workspace_size(int64_t M, int N, int K) {
  if (M < 0 || N <= 0 || K <= 0) return 0;
  return static_cast<size_t>(nvfp4::linear_layout(M, N, K).total);
}

extern "C" nvfp4_status_t nvfp4_linear(const void* x, int64_t M, int K, int64_t ld,
                                       const void* gamma, float eps, const uint8_t* w,
                                       const uint8_t* sfw, const float* gs_w, int N, void* out,
                                       void* ws, size_t ws_bytes, int32_t* dev_status,
                                       nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (M < 0 || N <= 0 || K <= 0 || ld < K || !(eps >= 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (K % 64 || N % 256 || ld % 8) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t)INT32_MAX - 127) return NVFP4_ERR_UNSUPPORTED_SHAPE;  // rows index as int
  if (!w || !sfw || !gs_w || !ws) return NVFP4_ERR_INVALID_ARG;
  if (M > 0 && (!x || !out)) return NVFP4_ERR_INVALID_ARG;
  const LinearLayout L = linear_layout(M, N, K);
  if ((int64_t)ws_bytes < L.total) return NVFP4_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(x) || !aligned16(w) || !aligned16(sfw) || !aligned16(out) || !aligned16(ws) ||
      !aligned16(gamma) || (reinterpret_cast<uintptr_t>(gs_w) & 3u))
    return NVFP4_ERR_MISALIGNED;
  if (M == 0) return NVFP4_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* codes = base + L.codes;
  uint8_t* sf = base + L.sf;
  float* gs = reinterpret_cast<float*>(base + L.gs);
  const int64_t Mp = round_up(M, 128);
  nvfp4_status_t st =
      gamma != nullptr
          ? rmsnorm_quantize_launch(x, M, K, ld, gamma, eps, nullptr, 1, Mp, codes, sf, gs, 1,
                                    base + L.quant_ws, dev_status, s)
          : quantize_launch(x, M, K, ld, nullptr, 1, Mp, codes, sf, gs, 1, base + L.quant_ws,
                            dev_status, s);
  if (st != NVFP4_OK) return st;
  float* part = L.part_floats > 0 ? reinterpret_cast<float*>(base + L.part) : nullptr;
  return gemm_dense(codes, sf, gs, w, sfw, gs_w, M, N, K, out, part, L.part_floats, dev_status, s);
}
