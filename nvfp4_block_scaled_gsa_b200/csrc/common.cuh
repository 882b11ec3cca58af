// common.cuh — sm_100a device helpers: bounded mbarrier waits, TMA / bulk copies, tcgen05
// (tensor memory, block-scaled MMA), FP4/FP8 conversions, and host-side error plumbing.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/nvfp4_moe.h"

#ifndef NVFP4_WAIT_TIMEOUT_NS
#define NVFP4_WAIT_TIMEOUT_NS 2000000000ull  // a bounded wait gives up after 2 s
#endif

namespace nvfp4 {

// ------------------------------------------------------------------------------ host errors
void set_last_error(const char* msg);
nvfp4_status_t check_launch(const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// ------------------------------------------------------------------------------ device misc
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report(int32_t* dev_status, int32_t bits) {
  if (dev_status) atomicOr(dev_status, bits);
}

// ------------------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (this CTA's or the peer's).  The
// default (CTA-scope release) semantics: what the arrival publishes is tensor-memory work,
// ordered by tcgen05.fence::before_thread_sync; a cluster-scope release would add a full memory
// barrier to every arrival.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// ------------------------------------------------------------------------------ clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the variable at shared::cta address `addr` in cluster CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Bounded wait on phase `parity` of an mbarrier.  Returns false (and raises *abort) when the
// wait ran out of time or another role of the CTA already gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_flag,
                                                  uint64_t limit_ns = NVFP4_WAIT_TIMEOUT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// ------------------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
// Pair form: this CTA's box lands in its own shared memory and its bytes complete the
// transaction on `cluster_bar` (the pair's leader barrier, a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t cluster_bar, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// *p += v, elementwise, as one vector reduction performed at L2 (no return value).
__device__ __forceinline__ void red_add_v4(float* p, float4 v) {
  asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

// ------------------------------------------------------------------------------ registers
// Per-warpgroup register budget (setmaxnreg): every thread of a warpgroup executes the same one.
// An increase waits until other warpgroups have released enough of the registers the block was
// launched with, so the budgets of all warpgroups must add up to at most that total.
template <uint32_t N>
__device__ __forceinline__ void regs_release_to() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N) : "memory");
}
template <uint32_t N>
__device__ __forceinline__ void regs_raise_to() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Pair (cta_group::2) forms: one warp of each CTA of the pair issues them together.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor (sm_100 format): start>>4 in [0,14), LBO>>4 in [16,30),
// SBO>>4 in [32,46), version 1 in [46,48), layout type in [61,64) (0 none, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}
// D(tmem) (+)= A(smem) * B(smem)^T with E2M1 operands and UE4M3 scales per 16 elements (K = 64),
// from tensor memory addresses of the scales.
// Pair form: M = 256 rows, 128 from each CTA's shared memory; B's N columns split in halves,
// the first from the leader's shared memory; every CTA keeps its 128 rows x N accumulator and
// reads its own scale factors (its A rows, all N of B) from its own tensor memory.
// Whole-warp forms: every lane of the warp executes them and elect.sync picks the one lane that
// issues (the lowest active lane, so MMAs and their commits come from the same thread).  A loop
// that issues MMAs from a single divergent lane costs about twice as many cycles per MMA.
__device__ __forceinline__ void tc_mma_nvf4_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t sfa_tmem,
                                                 uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X"
      " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void tc_mma_nvf4_pair_warp(uint32_t d_tmem, uint64_t adesc,
                                                      uint64_t bdesc, uint32_t idesc,
                                                      uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                      uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X"
      " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// MXFP4 forms: E2M1 operands with one UE8M0 scale per 32 elements (K = 64: 2 scales per row).
// The scale operands are tensor-memory addresses whose bits 30-31 select the byte of each
// 32-bit column where the MMA's 2 scales start (0 or 2); the instruction descriptor repeats
// that byte index in its A and B scale-factor id fields.
__device__ __forceinline__ void tc_mma_mxf4_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t sfa_tmem,
                                                 uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X"
      " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void tc_mma_mxf4_pair_warp(uint32_t d_tmem, uint64_t adesc,
                                                      uint64_t bdesc, uint32_t idesc,
                                                      uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                      uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X"
      " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void tc_commit_warp(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          bar)
      : "memory");
}
__device__ __forceinline__ void tc_commit_pair_warp(uint32_t cluster_bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          cluster_bar)
      : "memory");
}
// Instruction descriptor: E2M1 x E2M1, UE4M3 scales, K-major A and B, M rows (128, or 256 for
// the pair form).
__host__ __device__ constexpr uint32_t idesc_nvf4(int n, int m = 128) {
  return (1u << 7)                               // A format E2M1
         | (1u << 10)                            // B format E2M1
         | (static_cast<uint32_t>(n >> 3) << 17)  // N / 8
         | (0u << 23)                            // scale format UE4M3
         | (static_cast<uint32_t>(m >> 4) << 24);  // M / 16
}
// Instruction descriptor of the MXFP4 form: as above with scale format UE8M0 (bit 23); the
// per-MMA scale byte index goes to bits 29-30 (A) and 4-5 (B), see idesc_sf_byte.
__host__ __device__ constexpr uint32_t idesc_mxf4(int n, int m = 128) {
  return idesc_nvf4(n, m) | (1u << 23);
}
__host__ __device__ constexpr uint32_t idesc_sf_byte(uint32_t idesc, uint32_t byte) {
  return idesc | (byte << 29) | (byte << 4);
}

// 32 lanes x 32 consecutive 32-bit columns from tensor memory (one value per column per lane).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 lanes x 16 / 32 consecutive 32-bit columns into tensor memory (one value per column per lane).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
      "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]),
      "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Scale factors of one stage from shared memory into tensor memory, for the calling warp's lane
// quadrant.  The tensor-core layout for a 128-row operand (and for each 128-row half of a 256-row
// one) puts, for K step a, the 4 scales of row i + 32*m at lane i of every quadrant, column
// 4a + m; in the shared-memory atom those 16 bytes (m = 0..3) are line i, bytes 16i..16i+15.
// So lane i writes, per 128-row atom, one 16-byte line of its own index as 4 columns.
template <int NA = 4>
__device__ __forceinline__ void sf_rows128_to_tmem(uint32_t taddr, const uint8_t* atoms, int lane) {
  uint32_t r[4 * NA];
#pragma unroll
  for (int a = 0; a < NA; ++a) {
    const uint4 v = *reinterpret_cast<const uint4*>(atoms + a * 512 + lane * 16);
    r[4 * a] = v.x;
    r[4 * a + 1] = v.y;
    r[4 * a + 2] = v.z;
    r[4 * a + 3] = v.w;
  }
  if constexpr (NA == 4) tmem_st16(taddr, r);
  else tmem_st8(taddr, r);
}
// 256-row operand: columns 8a + 4h + m, h = which 128-row half (atoms of half h at
// +h*NA*512).
template <int NA = 4>
__device__ __forceinline__ void sf_rows256_to_tmem(uint32_t taddr, const uint8_t* atoms, int lane) {
  uint32_t r[8 * NA];
#pragma unroll
  for (int a = 0; a < NA; ++a) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 v = *reinterpret_cast<const uint4*>(atoms + h * NA * 512 + a * 512 + lane * 16);
      r[8 * a + 4 * h] = v.x;
      r[8 * a + 4 * h + 1] = v.y;
      r[8 * a + 4 * h + 2] = v.z;
      r[8 * a + 4 * h + 3] = v.w;
    }
  }
  if constexpr (NA == 4) tmem_st32(taddr, r);
  else tmem_st16(taddr, r);
}

// ------------------------------------------------------------------------------ conversions
// E4M3 (round to nearest even, saturate to +-448) of one float; result in the low byte.
__device__ __forceinline__ uint32_t cvt_e4m3(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}
// Decode a non-negative E4M3 byte (no NaN) exactly.
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xFu, m = b & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));    // 2^(e-7) * (1 + m/8)
}
// Two floats -> one byte of E2M1 codes (round to nearest even, saturate to +-6):
// `lo` goes to the low nibble, `hi` to the high nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// NVFP4 scale of one 16-element block given its amax:
//   s = (amax / 6) * gs ; byte = E4M3(s) ; d = decode(byte) ; r = gs / d (0 when d == 0).
// Each step is one IEEE float32 operation (no contraction, no fast-math).
// `s` returns the unrounded scale (for counting scales the E4M3 format clips).
__device__ __forceinline__ uint32_t nvfp4_block_scale(float amax, float gs, float& r, float& s) {
  s = __fmul_rn(__fdiv_rn(amax, 6.0f), gs);
  const uint32_t b = cvt_e4m3(s);
  const float d = e4m3_to_float(b);
  r = (d == 0.0f) ? 0.0f : __fdiv_rn(gs, d);
  return b;
}
__device__ __forceinline__ uint32_t nvfp4_block_scale(float amax, float gs, float& r) {
  float s;
  return nvfp4_block_scale(amax, gs, r, s);
}

// x * r for the E2M1 converter; a zero element stays (signed) zero even when r overflowed.
__device__ __forceinline__ float scaled(float x, float r) { return x == 0.0f ? x : __fmul_rn(x, r); }

// 8 values -> 4 bytes of packed codes (element 2j low nibble), using scale reciprocal r.
// A block whose decoded scale is 0 (r == 0) gets all-zero codes.
__device__ __forceinline__ uint32_t nvfp4_pack8(const float* v, float r) {
  if (r == 0.0f) return 0u;
  uint32_t out = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    out |= cvt_e2m1x2(scaled(v[2 * j], r), scaled(v[2 * j + 1], r)) << (8 * j);
  }
  return out;
}

// Global scale from the amax (float bits): 2688 / amax, 1.0 when not finite and positive.
__device__ __forceinline__ float gs_from_amax(float amax) {
  const float g = __fdiv_rn(2688.0f, amax);
  return (isfinite(g) && g > 0.0f) ? g : 1.0f;
}

// Byte offset of block scale (row r, scale column c) in the tiled layout with n_sf scale
// columns per row (n_sf % 4 == 0).
__host__ __device__ __forceinline__ int64_t sf_offset(int64_t r, int64_t c, int64_t n_sf) {
  return ((r >> 7) * (n_sf >> 2) + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

}  // namespace nvfp4
