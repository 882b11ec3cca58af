// route.cu — top-k softmax routing and the expert-bucketed row map ("slot mapping").
//
// The pages name "the MoE routing logic (top-k selection, slot mapping)" as work around the
// grouped GEMM ("NVFP4 MegaMoE Kernel Rewrite — CuTeDSL", section "Our Adaptation").  Reading
// used here: top-k of the logits (ties to the lower id; -inf = dropped slot), weights
// softmax(logits)[e] renormalized over the k; rows bucketed by expert in ascending id, every
// segment padded to a multiple of 128 rows (the GEMM's M tile), slots inside a segment in
// ascending (token, j); each row records its slot t*k + j.  Everything stays on the device: no
// host sync between routing and the GEMMs (the commit log's zero-.item() rule).
#include <float.h>

#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kMaxE = 256;
constexpr int kMaxK = 32;
constexpr int kPerLane = kMaxE / 32;

// One warp per token.  Lane l holds experts l, l+32, ..., and lane j < k ends up holding the
// j-th selected expert.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                   int k, int renorm, int32_t* __restrict__ ids,
                                                   float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  float v[kPerLane];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(logits + (int64_t)t * E + e) : -INFINITY;
    if (e < E) m = fmaxf(m, v[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));

  uint32_t taken = 0;
  int my_id = -1;
  float my_v = -INFINITY;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = INT_MAX;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !((taken >> i) & 1u) && (v[i] > bv || (v[i] == bv && e < be))) {
        bv = v[i];
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (ov > bv || (ov == bv && oe < be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be != INT_MAX && (be & 31) == lane) taken |= 1u << (be >> 5);
    if (lane == j) {
      my_id = be;
      my_v = bv;
    }
  }
  const bool live = lane < k && my_id != INT_MAX && my_v > -INFINITY && m > -INFINITY;
  const float ex = live ? expf(my_v - m) : 0.0f;
  float denom = 0.0f;
  if (renorm) {
    denom = ex;
  } else {
#pragma unroll
    for (int i = 0; i < kPerLane; ++i)
      if (lane + 32 * i < E && v[i] > -INFINITY && m > -INFINITY) denom += expf(v[i] - m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, o);
  if (lane < k) {
    ids[(int64_t)t * k + lane] = live ? my_id : -1;
    w[(int64_t)t * k + lane] = live ? ex / denom : 0.0f;
  }
}

// Single CTA of 32 warps.  Warp w owns the contiguous slot range [w*chunk, (w+1)*chunk), so a
// per-warp histogram plus an exclusive scan over warps gives every slot a stable rank inside
// its expert; __match_any_sync ranks the slots of one 32-slot step that share an expert.  Both
// passes over the slots load kUnroll steps ahead (independent loads in flight), and one warp
// scans the expert counts.
constexpr int kUnroll = 8;

__global__ void __launch_bounds__(1024) permute_kernel(
    const int32_t* __restrict__ ids, const float* __restrict__ w, int S, int k, int E,
    int64_t R_max, int32_t* __restrict__ offs_out, int32_t* __restrict__ dst_row,
    int32_t* __restrict__ row_slot, float* __restrict__ row_w, int32_t* __restrict__ dev_status) {
  __shared__ int hist[32][kMaxE];
  __shared__ int cnt[kMaxE];
  __shared__ int offs[kMaxE + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 32 * kMaxE; i += blockDim.x) (&hist[0][0])[i] = 0;
  __syncthreads();
  const int chunk = (S + 31) / 32;
  const int lo = min(S, warp * chunk), hi = min(S, lo + chunk);
  bool bad = false;
  for (int base = lo; base < hi; base += 32 * kUnroll) {
    int e[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = base + 32 * u + lane;
      e[u] = s < hi ? __ldg(ids + s) : -1;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (e[u] >= E) bad = true;
      else if (e[u] >= 0) atomicAdd(&hist[warp][e[u]], 1);
    }
  }
  if (bad) report(dev_status, NVFP4_DEVERR_BAD_INDEX);
  __syncthreads();
  if (tid < E) {
    int run = 0;
    for (int ww = 0; ww < 32; ++ww) {
      const int c = hist[ww][tid];
      hist[ww][tid] = run;
      run += c;
    }
    cnt[tid] = run;
  }
  __syncthreads();
  if (warp == 0) {  // offs = exclusive scan of the 128-padded counts (lane l: experts 8l..8l+7)
    int p[kMaxE / 32];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i) {
      const int e = lane * (kMaxE / 32) + i;
      p[i] = e < E ? (cnt[e] + 127) & ~127 : 0;
      sum += p[i];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i) {
      const int e = lane * (kMaxE / 32) + i;
      if (e <= E) offs[e] = run;
      run += p[i];
    }
    if (lane == 31 && E == kMaxE) offs[E] = run;
  }
  __syncthreads();
  if (tid <= E) offs_out[tid] = offs[tid];
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32 * kUnroll) {
    int e[kUnroll];
    float wv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = base + 32 * u + lane;
      e[u] = s < hi ? __ldg(ids + s) : -1;
      wv[u] = s < hi ? __ldg(w + s) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = base + 32 * u + lane;
      const bool valid = s < hi;
      const int eu = (e[u] >= E) ? -1 : e[u];
      const unsigned peers = __match_any_sync(0xffffffffu, eu);
      const int rank = __popc(peers & lt_mask);
      if (valid) {
        if (eu >= 0) {
          const int row = offs[eu] + hist[warp][eu] + rank;
          dst_row[s] = row;
          row_slot[row] = s;
          row_w[row] = wv[u];
        } else {
          dst_row[s] = -1;
        }
      }
      __syncwarp();
      if (eu >= 0 && rank == 0) hist[warp][eu] += __popc(peers);
      __syncwarp();
    }
  }
  // padding rows of every segment, then the unused tail up to R_max
  for (int e = warp; e < E; e += 32) {
    for (int r = offs[e] + cnt[e] + lane; r < offs[e + 1]; r += 32) {
      row_slot[r] = -1;
      row_w[r] = 0.0f;
    }
  }
  for (int64_t r = offs[E] + tid; r < R_max; r += blockDim.x) {
    row_slot[r] = -1;
    row_w[r] = 0.0f;
  }
}

}  // namespace

nvfp4_status_t permute_launch(const float* logits, int T, int E, int k, int renorm,
                              int32_t* topk_ids, float* topk_w, int32_t* offs, int32_t* dst_row,
                              int32_t* row_slot, float* row_w, int64_t R_max,
                              int32_t* dev_status, cudaStream_t s) {
  if (logits != nullptr && T > 0) {
    topk_kernel<<<(T + 7) / 8, 256, 0, s>>>(logits, T, E, k, renorm, topk_ids, topk_w);
    nvfp4_status_t st = check_launch("topk_kernel");
    if (st != NVFP4_OK) return st;
  }
  permute_kernel<<<1, 1024, 0, s>>>(topk_ids, topk_w, T * k, k, E, R_max, offs, dst_row,
                                    row_slot, row_w, dev_status);
  return check_launch("permute_kernel");
}

}  // namespace nvfp4

extern "C" int64_t moe_rows_max(int T, int E, int k) {
  if (T <= 0 || E <= 0 || k <= 0) return 0;
  const int64_t S = (int64_t)T * k;
  const int64_t busy = S < E ? S : E;
  return nvfp4::round_up(S + 127 * busy, 128);
}

extern "C" size_t moe_permute_workspace_size(int, int, int) { return 0; }

extern "C" nvfp4_status_t moe_permute(const float* logits, int T, int E, int k, int renormalize,
                                      int32_t* topk_ids, float* topk_w, int32_t* offs,
                                      int32_t* dst_row, int32_t* row_slot, float* row_w, void*,
                                      size_t, int32_t* dev_status, nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || k > E) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)T * k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (offs == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (T > 0 && (topk_ids == nullptr || topk_w == nullptr || dst_row == nullptr ||
                row_slot == nullptr || row_w == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  const void* ptrs[] = {logits, topk_ids, topk_w, offs, dst_row, row_slot, row_w};
  for (const void* p : ptrs)
    if (reinterpret_cast<uintptr_t>(p) & 3u) return NVFP4_ERR_MISALIGNED;
  return permute_launch(logits, T, E, k, renormalize, topk_ids, topk_w, offs, dst_row, row_slot,
                        row_w, moe_rows_max(T, E, k), dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}
