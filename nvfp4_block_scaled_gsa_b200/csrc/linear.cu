// linear.cu — dense NVFP4 linear, y = x W^T, with the activation quantized on the fly and an
// optional RMSNorm fused into that quantizer; and the shared expert built from the same pieces.
//
// The pages' dense layer (Nvfp4Linear, and the shared expert's two projections) quantizes its
// bf16 activation with a GPU-computed global scale and runs an NVFP4 GEMM against pre-packed
// weights (commit log of dsv4/kernels/cuda, nvfp4-megamoe-kernel: the "Updated layers" of the
// fused amax + quantize commit).  Here: [RMSNorm +] amax -> quantize -> the grouped GEMM core
// with one dense segment (split along K when the output has too few tiles to fill the SMs).
#include "common.cuh"
#include "launch.h"

namespace nvfp4 {

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

// The shared expert's L1 from split-K partial products (few rows: the fused-epilogue L1 would
// run one CTA per N tile).  Per 16-feature block: the ks planes of its 16 gate columns and 16 up
// columns (the W1 interleave: column 32j + i is gate feature 16j + i, column 32j + 16 + i its up
// partner) are added in plane order, then h = g * u / (1 + e^-g) and the block is quantized
// with the static gs_h, the fused L1 epilogue's arithmetic.  One thread per 4 features on a
// (row x chunk) grid, loads issued 4 planes at a time; the 4 lanes of a block share its amax by
// shuffles, and lanes 16g, +4, +8, +12 (blocks 4g..4g+3) assemble one scale word.
__global__ void __launch_bounds__(256) swiglu_quant_kernel(const float* __restrict__ part, int ks,
                                                           int64_t M, int I,
                                                           const float* __restrict__ gs_h_p,
                                                           uint8_t* __restrict__ h,
                                                           uint8_t* __restrict__ sfh) {
  const int64_t r = blockIdx.x;
  const int64_t t = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;  // features 4t .. 4t+3
  const bool valid = r < M && t < I / 4;
  const int64_t blk = t >> 2, q = t & 3;
  float hv[4] = {0.f, 0.f, 0.f, 0.f};
  float amax = 0.0f;
  if (valid) {
    const int64_t n2 = 2 * (int64_t)I;
    const float* gate = part + r * n2 + 32 * blk + 4 * q;
    float g[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
    for (int p0 = 0; p0 < ks; p0 += 4) {
      float4 a[4], b[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (p0 + j < ks) {
          const float* pg = gate + (p0 + j) * M * n2;
          a[j] = __ldg(reinterpret_cast<const float4*>(pg));
          b[j] = __ldg(reinterpret_cast<const float4*>(pg + 16));
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (p0 + j < ks) {
          g[0] += a[j].x; g[1] += a[j].y; g[2] += a[j].z; g[3] += a[j].w;
          u[0] += b[j].x; u[1] += b[j].y; u[2] += b[j].z; u[3] += b[j].w;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hv[i] = __fdividef(g[i] * u[i], 1.0f + __expf(-g[i]));
      amax = fmaxf(amax, fabsf(hv[i]));
    }
  }
  // the block's amax over its 4 consecutive lanes (invalid lanes hold 0 and sit in whole
  // invalid blocks: I / 4 is a multiple of 32)
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  const float gs_h = __ldg(gs_h_p);
  float rcp;
  const uint32_t sb = nvfp4_block_scale(amax, gs_h, rcp);
  uint32_t sword = sb;
  sword |= __shfl_down_sync(0xffffffffu, sb, 4) << 8;
  sword |= __shfl_down_sync(0xffffffffu, sb, 8) << 16;
  sword |= __shfl_down_sync(0xffffffffu, sb, 12) << 24;
  if (!valid) return;
  const uint32_t codes =
      rcp == 0.0f ? 0u
                  : (cvt_e2m1x2(scaled(hv[0], rcp), scaled(hv[1], rcp)) |
                     (cvt_e2m1x2(scaled(hv[2], rcp), scaled(hv[3], rcp)) << 8));
  *reinterpret_cast<uint16_t*>(h + r * (I / 2) + 2 * t) = static_cast<uint16_t>(codes);
  if ((t & 15) == 0) *reinterpret_cast<uint32_t*>(sfh + sf_offset(r, blk, I / 16)) = sword;
}

// L1 partial products of the shared expert, sized for kSizingSms (0 when the fused L1 is used).
int64_t shared_l1_part_floats(int64_t M, int H, int I) {
  const int ks = dense_k_splits(M, 2 * I, H, kSizingSms, INT64_MAX / 4);
  return ks > 1 ? ks * M * 2 * (int64_t)I : 0;
}

// Byte offsets of the nvfp4_shared_expert workspace regions (each 256-byte aligned).
struct SharedLayout {
  int64_t quant_ws, gs, xq, xsf, hq, hsf, part, part1, total;
  int64_t part_floats, part1_floats;
};

SharedLayout shared_layout(int64_t M, int H, int I) {
  SharedLayout L{};
  const int64_t Mp = round_up(M, 128);
  int64_t o = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = o;
    o += round_up(bytes, 256);
    return at;
  };
  L.quant_ws = take(static_cast<int64_t>(nvfp4_rmsnorm_quantize_workspace_size(M)));
  L.gs = take(4);
  L.xq = take(Mp * (H / 2));
  L.xsf = take(Mp * (H / 16));
  L.hq = take(Mp * (I / 2));
  L.hsf = take(Mp * (I / 16));
  L.part_floats = dense_part_floats(M, H, I);
  L.part = take(L.part_floats * 4);
  L.part1_floats = shared_l1_part_floats(M, H, I);
  L.part1 = take(L.part1_floats * 4);
  L.total = o;
  return L;
}

// [RMSNorm +] quantize x into the workspace's code rows (rows past M are padding).
nvfp4_status_t quantize_rows(const void* x, int64_t M, int K, int64_t ld, const void* gamma,
                             float eps, uint8_t* codes, uint8_t* sf, float* gs, void* qws,
                             int32_t* dev_status, cudaStream_t s) {
  const int64_t Mp = round_up(M, 128);
  return gamma != nullptr
             ? rmsnorm_quantize_launch(x, M, K, ld, gamma, eps, nullptr, 1, Mp, codes, sf, gs, 1,
                                       qws, dev_status, s)
             : quantize_launch(x, M, K, ld, nullptr, 1, Mp, codes, sf, gs, 1, qws, dev_status, s);
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
  nvfp4_status_t st =
      quantize_rows(x, M, K, ld, gamma, eps, codes, sf, gs, base + L.quant_ws, dev_status, s);
  if (st != NVFP4_OK) return st;
  float* part = L.part_floats > 0 ? reinterpret_cast<float*>(base + L.part) : nullptr;
  return gemm_dense(codes, sf, gs, w, sfw, gs_w, M, N, K, out, part, L.part_floats, dev_status, s);
}

extern "C" size_t nvfp4_shared_expert_workspace_size(int64_t M, int H, int I) {
  if (M < 0 || H <= 0 || I <= 0) return 0;
  return static_cast<size_t>(nvfp4::shared_layout(M, H, I).total);
}

extern "C" nvfp4_status_t nvfp4_shared_expert(const void* x, int64_t M, int H, int64_t ld,
                                              const void* gamma, float eps, const uint8_t* w1,
                                              const uint8_t* sfw1, const float* gs_w1,
                                              const uint8_t* w2, const uint8_t* sfw2,
                                              const float* gs_w2, int I, const float* gs_h,
                                              void* out, void* ws, size_t ws_bytes,
                                              int32_t* dev_status, nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (M < 0 || H <= 0 || I <= 0 || ld < H || !(eps >= 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (H % 256 || I % 128 || ld % 8) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t)INT32_MAX - 127) return NVFP4_ERR_UNSUPPORTED_SHAPE;  // rows index as int
  if (!w1 || !sfw1 || !gs_w1 || !w2 || !sfw2 || !gs_w2 || !gs_h || !ws)
    return NVFP4_ERR_INVALID_ARG;
  if (M > 0 && (!x || !out)) return NVFP4_ERR_INVALID_ARG;
  const SharedLayout L = shared_layout(M, H, I);
  if ((int64_t)ws_bytes < L.total) return NVFP4_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(w1) || !aligned16(sfw1) ||
      !aligned16(w2) || !aligned16(sfw2) || !aligned16(out) || !aligned16(ws) ||
      (reinterpret_cast<uintptr_t>(gs_w1) & 3u) || (reinterpret_cast<uintptr_t>(gs_w2) & 3u) ||
      (reinterpret_cast<uintptr_t>(gs_h) & 3u))
    return NVFP4_ERR_MISALIGNED;
  if (M == 0) return NVFP4_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* gs_x = reinterpret_cast<float*>(base + L.gs);
  nvfp4_status_t st = quantize_rows(x, M, H, ld, gamma, eps, base + L.xq, base + L.xsf, gs_x,
                                    base + L.quant_ws, dev_status, s);
  if (st != NVFP4_OK) return st;
  // L1 + SwiGLU + FP4 re-quantization: split along K when the output has too few tiles for the
  // SMs (partials, then swiglu_quant_kernel); otherwise the fused-epilogue kernel over one dense
  // segment (no offsets, every row written)
  const int ks1 = dense_k_splits(M, 2 * I, H, device_sms(), L.part1_floats);
  if (ks1 > 1) {
    float* part1 = reinterpret_cast<float*>(base + L.part1);
    st = gemm_dense_parts(base + L.xq, base + L.xsf, gs_x, w1, sfw1, gs_w1, M, 2 * I, H, ks1,
                          part1, dev_status, s);
    if (st != NVFP4_OK) return st;
    const int64_t quads = I / 4;  // threads per row, a multiple of 32 (I % 128 == 0)
    const int64_t chunks = (quads + 255) / 256;
    const int64_t per = (quads + chunks - 1) / chunks;
    swiglu_quant_kernel<<<dim3(static_cast<unsigned>(M), static_cast<unsigned>(chunks)),
                          dim3(static_cast<unsigned>((per + 31) / 32 * 32)), 0, s>>>(
        part1, ks1, M, I, gs_h, base + L.hq, base + L.hsf);
    st = check_launch("swiglu_quant_kernel");
  } else {
    st = gemm_l1(base + L.xq, base + L.xsf, gs_x, w1, sfw1, gs_w1, nullptr, nullptr, 1, H, I,
                 round_up(M, 128), gs_h, base + L.hq, base + L.hsf, nullptr, nullptr, dev_status,
                 s);
  }
  if (st != NVFP4_OK) return st;
  float* part = L.part_floats > 0 ? reinterpret_cast<float*>(base + L.part) : nullptr;
  return gemm_dense(base + L.hq, base + L.hsf, gs_h, w2, sfw2, gs_w2, M, H, I, out, part,
                    L.part_floats, dev_status, s);
}
