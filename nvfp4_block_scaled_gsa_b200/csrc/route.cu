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

// Top-k of token t by one warp.  Lane l holds experts l, l+32, ..., and lane j < k ends up
// holding the j-th selected expert.
__device__ __forceinline__ void topk_token(const float* __restrict__ logits, int t, int E, int k,
                                           int renorm, int lane, int32_t* ids, float* w) {
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

// One warp per token.
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                   int k, int renorm, int32_t* __restrict__ ids,
                                                   float* __restrict__ w) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t < T) topk_token(logits, t, E, k, renorm, threadIdx.x & 31, ids, w);
}

// Slots [lo, hi) of one CTA of 32 warps.  Warp w owns a contiguous part of the range, so a
// per-warp histogram plus an exclusive scan over warps gives every slot a stable rank inside its
// expert; __match_any_sync ranks the slots of one 32-slot step that share an expert.  Both passes
// over the slots load kUnroll steps ahead (independent loads in flight).
constexpr int kUnroll = 8;
// From this many slots the row map is built by many CTAs (two launches: per-chunk expert
// histograms, then ranks and writes): one SM issuing every scattered row store was the limit.
constexpr int kMultiMinSlots = 4096;
constexpr int kChunkSlots = 2048;  // slots per CTA in the multi-CTA form

// ids is read with plain loads: in the single-CTA form the same kernel has just written it.
__device__ __forceinline__ void warp_histogram(const int32_t* ids, int lo, int hi, int E, int lane,
                                               int* __restrict__ hist_w, bool& bad) {
  for (int base = lo; base < hi; base += 32 * kUnroll) {
    int e[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = base + 32 * u + lane;
      e[u] = s < hi ? ids[s] : -1;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (e[u] >= E) bad = true;
      else if (e[u] >= 0) atomicAdd(&hist_w[e[u]], 1);
    }
  }
}

// Per-chunk expert histograms of the multi-CTA form: hist_g[c][e] = slots of chunk c routed to e.
__global__ void __launch_bounds__(1024) permute_count_kernel(const int32_t* __restrict__ ids, int S,
                                                              int E, int32_t* __restrict__ hist_g,
                                                              int32_t* __restrict__ dev_status) {
  __shared__ int hist[kMaxE];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kMaxE; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int c0 = blockIdx.x * kChunkSlots, c1 = min(S, c0 + kChunkSlots);
  const int per = (c1 - c0 + 31) / 32;
  const int lo = min(c1, c0 + warp * per), hi = min(c1, lo + per);
  bool bad = false;
  warp_histogram(ids, lo, hi, E, lane, hist, bad);
  if (bad) report(dev_status, NVFP4_DEVERR_BAD_INDEX);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) hist_g[(int64_t)blockIdx.x * E + e] = hist[e];
}

// kMulti = false: one CTA over all S slots; with logits given, it first takes the top-k of the
// T = S / k tokens itself (one warp per token) and writes ids and w, so that a small batch routes
// in one launch.  kMulti = true: CTA c over chunk c, with the expert totals and the chunk's base
// per expert taken from hist_g (nch chunks).
template <bool kMulti>
__global__ void __launch_bounds__(1024) permute_kernel(
    const float* __restrict__ logits, int k, int renorm, int32_t* ids, float* w, int S, int E,
    int64_t R_max, const int32_t* __restrict__ hist_g, int nch, int32_t* __restrict__ offs_out,
    int32_t* __restrict__ dst_row, int32_t* __restrict__ row_slot, float* __restrict__ row_w,
    int32_t* __restrict__ dev_status) {
  __shared__ int hist[32][kMaxE];
  __shared__ int cnt[kMaxE];
  __shared__ int offs[kMaxE + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (!kMulti && logits != nullptr)
    for (int t = warp; t < S / k; t += 32) topk_token(logits, t, E, k, renorm, lane, ids, w);
  for (int i = tid; i < 32 * kMaxE; i += blockDim.x) (&hist[0][0])[i] = 0;
  __syncthreads();  // also: this CTA's ids and w writes are visible to all its threads
  const int c0 = kMulti ? blockIdx.x * kChunkSlots : 0;
  const int c1 = kMulti ? min(S, c0 + kChunkSlots) : S;
  const int per = (c1 - c0 + 31) / 32;
  const int lo = min(c1, c0 + warp * per), hi = min(c1, lo + per);
  bool bad = false;
  warp_histogram(ids, lo, hi, E, lane, hist[warp], bad);
  if (bad && !kMulti) report(dev_status, NVFP4_DEVERR_BAD_INDEX);  // multi: the count kernel
  __syncthreads();
  if (tid < E) {
    int run = 0;
    if (kMulti) {  // this chunk's base and the expert's total over all chunks
      int before = 0, total = 0;
      for (int c = 0; c < nch; ++c) {
        const int v = __ldg(hist_g + (int64_t)c * E + tid);
        if (c < (int)blockIdx.x) before += v;
        total += v;
      }
      run = before;
      cnt[tid] = total;
    }
    for (int ww = 0; ww < 32; ++ww) {
      const int c = hist[ww][tid];
      hist[ww][tid] = run;
      run += c;
    }
    if (!kMulti) cnt[tid] = run;
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
  if (blockIdx.x == 0 && tid <= E) offs_out[tid] = offs[tid];
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32 * kUnroll) {
    int e[kUnroll];
    float wv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = base + 32 * u + lane;
      e[u] = s < hi ? ids[s] : -1;
      wv[u] = s < hi ? w[s] : 0.0f;
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
  // padding rows of every segment, then the unused tail up to R_max (spread over the CTAs)
  const int nwarps = 32 * gridDim.x;
  const int gwarp = blockIdx.x * 32 + warp;
  for (int e = gwarp; e < E; e += nwarps) {
    for (int r = offs[e] + cnt[e] + lane; r < offs[e + 1]; r += 32) {
      row_slot[r] = -1;
      row_w[r] = 0.0f;
    }
  }
  for (int64_t r = offs[E] + blockIdx.x * (int64_t)blockDim.x + tid; r < R_max;
       r += (int64_t)gridDim.x * blockDim.x) {
    row_slot[r] = -1;
    row_w[r] = 0.0f;
  }
}

}  // namespace

int permute_chunks(int T, int k) {
  const int64_t S = (int64_t)T * k;
  return S >= kMultiMinSlots ? static_cast<int>((S + kChunkSlots - 1) / kChunkSlots) : 0;
}

size_t permute_workspace_bytes(int T, int E, int k) {
  return (size_t)permute_chunks(T, k) * (size_t)E * sizeof(int32_t);
}

nvfp4_status_t permute_launch(const float* logits, int T, int E, int k, int renorm,
                              int32_t* topk_ids, float* topk_w, int32_t* offs, int32_t* dst_row,
                              int32_t* row_slot, float* row_w, int64_t R_max, int32_t* hist_ws,
                              int32_t* dev_status, cudaStream_t s) {
  const int S = T * k;
  const int nch = permute_chunks(T, k);
  const bool multi = nch > 0 && hist_ws != nullptr;
  if (logits != nullptr && T > 0 && multi) {
    topk_kernel<<<(T + 7) / 8, 256, 0, s>>>(logits, T, E, k, renorm, topk_ids, topk_w);
    nvfp4_status_t st = check_launch("topk_kernel");
    if (st != NVFP4_OK) return st;
  }
  if (multi) {
    permute_count_kernel<<<nch, 1024, 0, s>>>(topk_ids, S, E, hist_ws, dev_status);
    nvfp4_status_t st = check_launch("permute_count_kernel");
    if (st != NVFP4_OK) return st;
    permute_kernel<true><<<nch, 1024, 0, s>>>(nullptr, k, renorm, topk_ids, topk_w, S, E, R_max,
                                              hist_ws, nch, offs, dst_row, row_slot, row_w,
                                              dev_status);
    return check_launch("permute_kernel");
  }
  // a small batch: top-k and the row map in one CTA, one launch
  permute_kernel<false><<<1, 1024, 0, s>>>(T > 0 ? logits : nullptr, k, renorm, topk_ids,
                                           topk_w, S, E, R_max, nullptr, 0, offs, dst_row,
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

extern "C" size_t moe_permute_workspace_size(int T, int E, int k) {
  if (T <= 0 || E <= 0 || k <= 0) return 0;
  return nvfp4::permute_workspace_bytes(T, E, k);
}

extern "C" nvfp4_status_t moe_permute(const float* logits, int T, int E, int k, int renormalize,
                                      int32_t* topk_ids, float* topk_w, int32_t* offs,
                                      int32_t* dst_row, int32_t* row_slot, float* row_w, void* ws,
                                      size_t ws_bytes, int32_t* dev_status,
                                      nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > kMaxK || k > E) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((int64_t)T * k > (int64_t)1 << 30) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (offs == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (T > 0 && (topk_ids == nullptr || topk_w == nullptr || dst_row == nullptr ||
                row_slot == nullptr || row_w == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  const void* ptrs[] = {logits, topk_ids, topk_w, offs, dst_row, row_slot, row_w, ws};
  for (const void* p : ptrs)
    if (reinterpret_cast<uintptr_t>(p) & 3u) return NVFP4_ERR_MISALIGNED;
  // the multi-CTA form needs the workspace; without it one CTA builds the map (same result)
  int32_t* hist_ws = ws != nullptr && ws_bytes >= permute_workspace_bytes(T, E, k)
                         ? static_cast<int32_t*>(ws)
                         : nullptr;
  return permute_launch(logits, T, E, k, renormalize, topk_ids, topk_w, offs, dst_row, row_slot,
                        row_w, moe_rows_max(T, E, k), hist_ws, dev_status,
                        reinterpret_cast<cudaStream_t>(stream));
}
