// mx.cu — BF16 -> MXFP4 quantization: E2M1 elements, one UE8M0 (power-of-two) scale per 32.
//
// The format the pages contrast with NVFP4 ("May 24, 2026 — Session Start Plan", section 1
// "NVFP4-0": MXFP4 has 32-element blocks and UE8M0 scales, NVFP4 16-element blocks and E4M3
// scales).  The pages give no formula; the OCP Microscaling v1.0 rule is used:
//   e = floor(log2(max|x_i|)) - 2 (2 = the exponent of E2M1's largest value, 6 = 1.5 * 2^2),
//   clamped to [-127, 127] (-127 for an all-zero block); scale byte = e + 127;
//   code_i = E2M1_rn_satfinite(x_i * 2^-e)   (the multiply by a power of two is exact).
// No global scale.  The scale bytes use the same 128-row x 4-column tiled atoms as the NVFP4
// scales, each scale column now covering 32 elements (an atom covers 128 of K).
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kMxThreads = 128;

// Block exponent from the float bits of amax: for a normal amax with biased exponent E,
// floor(log2(amax)) = E - 127, so e = E - 129, clamped below at -127 (a subnormal amax, and 0,
// give -127).  E <= 254, so e <= 125 and the clamp above never binds for float inputs.
__device__ __forceinline__ int mx_block_exponent(float amax) {
  const int E = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  return amax > 0.0f ? max(E - 129, -127) : -127;
}

// One thread per 32-element block on a 2-D grid (row, chunk of blockDim.x blocks): four 16-byte
// loads, the block's exponent, 16 bytes of codes; 4 consecutive lanes (4 scale columns) assemble
// one aligned 4-byte group of the tiled scale layout.
__global__ void __launch_bounds__(kMxThreads) mxfp4_quantize_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  const int64_t nblk_row = cols / 32;
  const int64_t r = blockIdx.x;
  const int64_t c = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
  const bool valid = r < rows && c < nblk_row;
  uint32_t sbyte = 0;
  uint4 packed = make_uint4(0u, 0u, 0u, 0u);
  if (valid) {
    const uint4* src = reinterpret_cast<const uint4*>(x + r * ld + c * 32);
    float v[32];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 u = __ldg(src + q);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
        v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e = mx_block_exponent(amax);
    sbyte = static_cast<uint32_t>(e + 127);
    // 2^-e as a float: biased exponent 127 - e lies in [2, 254] for e in [-127, 125]
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
    uint32_t wds[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        word |= cvt_e2m1x2(__fmul_rn(v[8 * q + 2 * j], inv), __fmul_rn(v[8 * q + 2 * j + 1], inv))
                << (8 * j);
      wds[q] = word;
    }
    packed = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
  uint32_t sword = sbyte;
  sword |= __shfl_down_sync(0xffffffffu, sbyte, 1) << 8;
  sword |= __shfl_down_sync(0xffffffffu, sbyte, 2) << 16;
  sword |= __shfl_down_sync(0xffffffffu, sbyte, 3) << 24;
  if (!valid) return;
  *reinterpret_cast<uint4*>(codes + r * (cols / 2) + c * 16) = packed;
  if ((c & 3) == 0) *reinterpret_cast<uint32_t*>(sf + sf_offset(r, c, nblk_row)) = sword;
}

}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status_t mxfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                         uint8_t* codes, uint8_t* sf, int32_t* dev_status,
                                         nvfp4_stream_t stream) {
  using namespace nvfp4;
  (void)dev_status;
  if (rows < 0 || cols <= 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
  if (cols % 128 != 0 || ld % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows > 0x7FFFFFFF || cols / 32 > 65535LL * kMxThreads) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0) return NVFP4_OK;
  if (x == nullptr || codes == nullptr || sf == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(sf)) return NVFP4_ERR_MISALIGNED;
  const int64_t nblk = cols / 32;
  const int64_t chunks = (nblk + kMxThreads - 1) / kMxThreads;
  const int64_t per = (nblk + chunks - 1) / chunks;
  const dim3 block(static_cast<unsigned>((per + 31) / 32 * 32));
  const dim3 grid(static_cast<unsigned>(rows), static_cast<unsigned>(chunks));
  mxfp4_quantize_kernel<<<grid, block, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(x), rows, cols, ld, codes, sf);
  return check_launch("mxfp4_quantize_kernel");
}
