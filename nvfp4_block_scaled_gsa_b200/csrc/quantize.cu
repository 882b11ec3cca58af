// quantize.cu — BF16 -> NVFP4 quantization (amax -> global scale on the GPU, then codes).
//
// Two stream-ordered kernels, as the commit log of dsv4/kernels/cuda (nvfp4-megamoe-kernel)
// settles on after a single-launch version raced across CTAs: an amax kernel reduces max|x| into
// one device word, and the quantize kernel derives gs = 2688 / amax from that word itself (no
// host sync, no .item()).  Codes are computed against the decoded FP8 block scale (the commit
// log's "quantize must use the FP8-round-tripped block scale").
//
// The same pair of kernels with an RMSNorm in front (the fused RMSNorm + quantize of the same
// commit log, whose kernel keeps the row's inverse RMS beside the amax): a row-statistics
// kernel writes each row's 1/rms and reduces the amax of the normalized tensor, and the
// quantize kernel normalizes each block as it loads it.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;
// quantize_kernel's grid: one row per blockIdx.x, at most 65535 column chunks of kThreads blocks
constexpr int64_t kMaxQuantRows = 0x7FFFFFFF;
constexpr int64_t kMaxQuantCols = 65535LL * kThreads * 16;

// max|x| over the (rows x cols) bf16 matrix with row stride ld -> atomicMax on the float bits
// (non-negative floats order like their bit patterns).
__global__ void __launch_bounds__(kThreads) amax_kernel(const __nv_bfloat16* __restrict__ x,
                                                        int64_t rows, int64_t cols, int64_t ld,
                                                        uint32_t* __restrict__ amax_bits) {
  const int64_t vec_per_row = cols / 8;
  const int64_t nvec = rows * vec_per_row;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  uint32_t m = 0;  // max of |bf16| bit patterns (sign cleared)
  auto fold = [&](const uint4& q) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      m = max(m, w[i] & 0x7FFFu);
      m = max(m, (w[i] >> 16) & 0x7FFFu);
    }
  };
  // contiguous rows (ld == cols, the usual case): the flat index is the address, with no 64-bit
  // division per load
  const bool flat = ld == cols;
  auto load = [&](int64_t v) {
    if (flat) return __ldg(reinterpret_cast<const uint4*>(x) + v);
    const int64_t r = v / vec_per_row, c = (v - r * vec_per_row) * 8;
    return __ldg(reinterpret_cast<const uint4*>(x + r * ld + c));
  };
  int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  for (; v + 3 * stride < nvec; v += 4 * stride) {  // four independent loads in flight
    const uint4 q0 = load(v), q1 = load(v + stride), q2 = load(v + 2 * stride),
                q3 = load(v + 3 * stride);
    fold(q0);
    fold(q1);
    fold(q2);
    fold(q3);
  }
  for (; v < nvec; v += stride) fold(load(v));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t red[kThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0;
    for (int i = 0; i < kThreads / 32; ++i) b = max(b, red[i]);
    atomicMax(amax_bits, b << 16);  // bf16 bits -> float bits
  }
}

// RMSNorm of one element, FP32 with one rounding per step: y = (x * rstd) * gamma.
__device__ __forceinline__ float rms_apply(float x, float rstd, float g) {
  return __fmul_rn(__fmul_rn(x, rstd), g);
}

// rstd = 1 / sqrt(mean(x^2) + eps) of each row, then the amax of the normalized rows.  One
// 256-thread block per row (grid-stride over rows): the row's first 8192 columns are loaded
// into registers at once (every load in flight), summed, and reused for the amax; the block's
// next row is loaded meanwhile.  The sum of
// squares is taken in float64 (each square of a bf16 value is exact) with the warps' partial
// sums added in warp order; its mean is rounded once to float32, and the rest is float32 with
// one rounding per operation:
//   ms = fl32(ss / cols); v = ms + eps; s = sqrt_rn(v); rstd = 1 / s (rn); y = (x*rstd)*gamma.
// The amax is an unsigned max over the float bits with the sign cleared, so a NaN wins (and
// then gives gs = 1), as in the plain amax kernel; one atomic per block.
constexpr int kRmsChunks = 4;  // uint4 chunks (8 columns each) per thread held in registers

__global__ void __launch_bounds__(kThreads, 4) rms_stats_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    const __nv_bfloat16* __restrict__ gamma, float eps, float* __restrict__ rstd_out,
    uint32_t* __restrict__ amax_bits) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n8 = cols / 8;
  __shared__ double part[kThreads / 32];
  __shared__ float s_rstd;
  __shared__ uint32_t red[kThreads / 32];
  uint32_t m = 0;
  auto sq = [](const uint4& q) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    double t = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const double lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xFFFF0000u);
      t += lo * lo;
      t += hi * hi;
    }
    return t;
  };
  auto fold_amax = [&](const uint4& q, const uint4& g, float rstd) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float y0 = rms_apply(__uint_as_float(w[i] << 16), rstd, __uint_as_float(gw[i] << 16));
      const float y1 = rms_apply(__uint_as_float(w[i] & 0xFFFF0000u), rstd,
                                 __uint_as_float(gw[i] & 0xFFFF0000u));
      m = max(m, __float_as_uint(y0) & 0x7FFFFFFFu);
      m = max(m, __float_as_uint(y1) & 0x7FFFFFFFu);
    }
  };
  auto load_row = [&](int64_t r, uint4 (&q)[kRmsChunks]) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * ld);
#pragma unroll
    for (int j = 0; j < kRmsChunks; ++j) {
      const int64_t c = tid + (int64_t)j * kThreads;
      q[j] = (r < rows && c < n8) ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 q[kRmsChunks];
  load_row(blockIdx.x, q);
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + row * ld);
    // the block's next row is loaded while this one is reduced
    uint4 qn[kRmsChunks];
    load_row(row + gridDim.x, qn);
    double ss = 0.0;
#pragma unroll
    for (int j = 0; j < kRmsChunks; ++j) ss += sq(q[j]);
    for (int64_t c = tid + (int64_t)kRmsChunks * kThreads; c < n8; c += kThreads)
      ss += sq(__ldg(xr + c));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) part[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < kThreads / 32; ++w) t += part[w];
      const float ms = __double2float_rn(t / static_cast<double>(cols));
      const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
      s_rstd = rstd;
      rstd_out[row] = rstd;
    }
    __syncthreads();
    const float rstd = s_rstd;
    if (amax_bits != nullptr) {
      const uint4* gr = reinterpret_cast<const uint4*>(gamma);
#pragma unroll
      for (int j = 0; j < kRmsChunks; ++j) {
        const int64_t c = tid + (int64_t)j * kThreads;
        if (c < n8) fold_amax(q[j], __ldg(gr + c), rstd);
      }
      for (int64_t c = tid + (int64_t)kRmsChunks * kThreads; c < n8; c += kThreads)
        fold_amax(__ldg(xr + c), __ldg(gr + c), rstd);
    }
    __syncthreads();  // part[] and s_rstd are rewritten for the next row
#pragma unroll
    for (int j = 0; j < kRmsChunks; ++j) q[j] = qn[j];
  }
  if (amax_bits == nullptr) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (tid == 0) {
    uint32_t b = 0;
    for (int i = 0; i < kThreads / 32; ++i) b = max(b, red[i]);
    atomicMax(amax_bits, b);
  }
}

// One thread per 16-element block, on a 2-D grid: blockIdx.x is the row, blockIdx.y a chunk of
// blockDim.x blocks of it (no index division).  gs comes from the amax word (compute mode, and
// the first thread publishes it to *gs) or is read from *gs.  Codes and the scale byte go to
// output row i (dst_row == nullptr) or to the k rows dst_row[i*k + j].  NORM: each element is
// first normalized with its row's rstd and gamma (rms_apply), exactly as rms_stats_kernel did.
template <bool NORM>
__global__ void __launch_bounds__(kThreads) quantize_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    const int32_t* __restrict__ dst_row, int k, int64_t out_rows, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ sf, float* __restrict__ gs_io, const uint32_t* __restrict__ amax_bits,
    const float* __restrict__ rstd, const __nv_bfloat16* __restrict__ gamma,
    int32_t* __restrict__ dev_status) {
  const int64_t nblk_row = cols / 16;
  float gs;
  if (amax_bits != nullptr) {
    gs = gs_from_amax(__uint_as_float(__ldg(amax_bits)));
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *gs_io = gs;
  } else {
    gs = __ldg(gs_io);
  }
  // no early return: the 4 lanes of a 4-block group exchange their scale bytes with shuffles
  // (blocks 4g..4g+3 of a row are 4 consecutive lanes: blockDim.x is a multiple of 32)
  const int64_t r = blockIdx.x;
  const int64_t c = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
  const bool valid = r < rows && c < nblk_row;
  uint32_t sbyte = 0;
  uint2 packed = make_uint2(0u, 0u);
  if (valid) {
    const uint4* src = reinterpret_cast<const uint4*>(x + r * ld + c * 16);
    const uint4 q0 = __ldg(src), q1 = __ldg(src + 1);
    const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    float v[16];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    if constexpr (NORM) {
      const float rs = __ldg(rstd + r);
      const uint4* gsrc = reinterpret_cast<const uint4*>(gamma + c * 16);
      const uint4 g0 = __ldg(gsrc), g1 = __ldg(gsrc + 1);
      const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        v[2 * i] = rms_apply(v[2 * i], rs, __uint_as_float(gw[i] << 16));
        v[2 * i + 1] = rms_apply(v[2 * i + 1], rs, __uint_as_float(gw[i] & 0xFFFF0000u));
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
    float rcp;
    sbyte = nvfp4_block_scale(amax, gs, rcp);
    packed.x = nvfp4_pack8(v, rcp);
    packed.y = nvfp4_pack8(v + 8, rcp);
  }
  // the group's 4 scale bytes, assembled in its first lane (scale columns 4g..4g+3 are one
  // aligned 4-byte group of the tiled layout)
  uint32_t sword = sbyte;
  sword |= __shfl_down_sync(0xffffffffu, sbyte, 1) << 8;
  sword |= __shfl_down_sync(0xffffffffu, sbyte, 2) << 16;
  sword |= __shfl_down_sync(0xffffffffu, sbyte, 3) << 24;
  if (!valid) return;
  const bool leader = (c & 3) == 0;
  const int64_t row_bytes = cols / 2;
  auto put = [&](int64_t d) {
    *reinterpret_cast<uint2*>(codes + d * row_bytes + c * 8) = packed;
    if (leader) *reinterpret_cast<uint32_t*>(sf + sf_offset(d, c, nblk_row)) = sword;
  };
  if (dst_row == nullptr) {
    put(r);
    return;
  }
  for (int j = 0; j < k; ++j) {
    const int64_t d = __ldg(dst_row + r * k + j);
    if (d < 0) continue;
    if (d >= out_rows) {
      report(dev_status, NVFP4_DEVERR_BAD_INDEX);
      continue;
    }
    put(d);
  }
}

// Launch shape of quantize_kernel: one row per block column, each row's cols/16 blocks cut into
// the fewest chunks of at most kThreads threads, each chunk a whole number of warps (448 blocks
// of a 7168-column row: 2 chunks of 224).  A grid of one row when there are none, so that the
// global scale is still published.
struct QuantGrid {
  dim3 grid, block;
};

QuantGrid quant_grid(int64_t rows, int64_t cols) {
  const int64_t nblk_row = cols / 16;
  const int64_t chunks = (nblk_row + kThreads - 1) / kThreads;
  const int64_t per = (nblk_row + chunks - 1) / chunks;
  QuantGrid q;
  q.block = dim3(static_cast<unsigned>((per + 31) / 32 * 32));
  q.grid = dim3(static_cast<unsigned>(rows > 0 ? rows : 1), static_cast<unsigned>(chunks));
  return q;
}

}  // namespace

nvfp4_status_t quantize_launch(const void* x, int64_t rows, int64_t cols, int64_t ld,
                               const int32_t* dst_row, int k, int64_t out_rows, uint8_t* codes,
                               uint8_t* sf, float* gs, int compute_gs, void* ws,
                               int32_t* dev_status, cudaStream_t s) {
  if (rows > kMaxQuantRows || cols > kMaxQuantCols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  uint32_t* amax = nullptr;
  if (compute_gs) {
    amax = static_cast<uint32_t*>(ws);
    if (cudaMemsetAsync(amax, 0, sizeof(uint32_t), s) != cudaSuccess)
      return check_launch("memset amax");
    const int64_t nvec = rows * (cols / 8);
    if (nvec > 0) {
      const int64_t want = (nvec + kThreads - 1) / kThreads;
      const int grid = static_cast<int>(want < 148 * 8 ? want : 148 * 8);
      amax_kernel<<<grid, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), rows, cols, ld,
                                            amax);
      nvfp4_status_t st = check_launch("amax_kernel");
      if (st != NVFP4_OK) return st;
    }
  }
  const QuantGrid qg = quant_grid(rows, cols);
  quantize_kernel<false><<<qg.grid, qg.block, 0, s>>>(
      static_cast<const __nv_bfloat16*>(x), rows, cols, ld, dst_row, k, out_rows, codes, sf, gs,
      amax, nullptr, nullptr, dev_status);
  return check_launch("quantize_kernel");
}

// Workspace of the fused RMSNorm + quantize: the amax word, then rstd float[rows].
constexpr int64_t kRmsRstdOffset = 256;

nvfp4_status_t rmsnorm_quantize_launch(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                       const void* gamma, float eps, const int32_t* dst_row,
                                       int k, int64_t out_rows, uint8_t* codes, uint8_t* sf,
                                       float* gs, int compute_gs, void* ws, int32_t* dev_status,
                                       cudaStream_t s) {
  if (rows > kMaxQuantRows || cols > kMaxQuantCols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  uint32_t* amax = compute_gs ? static_cast<uint32_t*>(ws) : nullptr;
  float* rstd = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kRmsRstdOffset);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* gb = static_cast<const __nv_bfloat16*>(gamma);
  if (amax != nullptr && cudaMemsetAsync(amax, 0, sizeof(uint32_t), s) != cudaSuccess)
    return check_launch("memset amax");
  if (rows > 0) {
    const int64_t blocks = rows < 148 * 4 ? rows : 148 * 4;  // 4 resident blocks per SM (64 regs)
    rms_stats_kernel<<<static_cast<unsigned>(blocks), kThreads, 0, s>>>(xb, rows, cols, ld, gb,
                                                                        eps, rstd, amax);
    nvfp4_status_t st = check_launch("rms_stats_kernel");
    if (st != NVFP4_OK) return st;
  }
  const QuantGrid qg = quant_grid(rows, cols);
  quantize_kernel<true><<<qg.grid, qg.block, 0, s>>>(
      xb, rows, cols, ld, dst_row, k, out_rows, codes, sf, gs, amax, rstd, gb, dev_status);
  return check_launch("quantize_kernel");
}

}  // namespace nvfp4

extern "C" size_t nvfp4_quantize_workspace_size(void) { return 256; }

extern "C" size_t nvfp4_rmsnorm_quantize_workspace_size(int64_t rows) {
  return static_cast<size_t>(nvfp4::kRmsRstdOffset +
                             nvfp4::round_up((rows > 0 ? rows : 0) * 4, 256));
}

extern "C" nvfp4_status_t nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                         const int32_t* dst_row, int k, int64_t out_rows,
                                         uint8_t* codes, uint8_t* sf, float* gs, int compute_gs,
                                         void* ws, size_t ws_bytes, int32_t* dev_status,
                                         nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (rows < 0 || out_rows < 0 || cols <= 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 64 != 0 || ld % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows > kMaxQuantRows || cols > kMaxQuantCols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (gs == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (rows > 0 && (x == nullptr || codes == nullptr || sf == nullptr)) return NVFP4_ERR_INVALID_ARG;
  if (dst_row == nullptr) {
    if (out_rows < rows) return NVFP4_ERR_INVALID_ARG;
  } else if (k < 1 || k > 64) {
    return NVFP4_ERR_INVALID_ARG;
  }
  if (compute_gs) {
    if (ws == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (ws_bytes < nvfp4_quantize_workspace_size()) return NVFP4_ERR_WORKSPACE_TOO_SMALL;
  }
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf) || !aligned16(ws) ||
      (reinterpret_cast<uintptr_t>(gs) & 3u) || (reinterpret_cast<uintptr_t>(dst_row) & 3u))
    return NVFP4_ERR_MISALIGNED;
  return quantize_launch(x, rows, cols, ld, dst_row, k, out_rows, codes, sf, gs, compute_gs, ws,
                         dev_status, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" nvfp4_status_t nvfp4_rmsnorm_quantize(const void* x, int64_t rows, int64_t cols,
                                                 int64_t ld, const void* gamma, float eps,
                                                 const int32_t* dst_row, int k, int64_t out_rows,
                                                 uint8_t* codes, uint8_t* sf, float* gs,
                                                 int compute_gs, void* ws, size_t ws_bytes,
                                                 int32_t* dev_status, nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (rows < 0 || out_rows < 0 || cols <= 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 64 != 0 || ld % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows > kMaxQuantRows || cols > kMaxQuantCols) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (gs == nullptr || ws == nullptr || !(eps >= 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (rows > 0 && (x == nullptr || gamma == nullptr || codes == nullptr || sf == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (dst_row == nullptr) {
    if (out_rows < rows) return NVFP4_ERR_INVALID_ARG;
  } else if (k < 1 || k > 64) {
    return NVFP4_ERR_INVALID_ARG;
  }
  if (ws_bytes < nvfp4_rmsnorm_quantize_workspace_size(rows)) return NVFP4_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(codes) || !aligned16(sf) ||
      !aligned16(ws) || (reinterpret_cast<uintptr_t>(gs) & 3u) ||
      (reinterpret_cast<uintptr_t>(dst_row) & 3u))
    return NVFP4_ERR_MISALIGNED;
  return rmsnorm_quantize_launch(x, rows, cols, ld, gamma, eps, dst_row, k, out_rows, codes, sf,
                                 gs, compute_gs, ws, dev_status,
                                 reinterpret_cast<cudaStream_t>(stream));
}
