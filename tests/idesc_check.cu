// Host program for tests/test_idesc_cutlass.py: prints the tcgen05 block-scaled instruction
// descriptors the library builds (common.cuh) next to CUTLASS's own construction of the same
// descriptors (cute/arch/mma_sm100_desc.hpp), one "name ours cutlass" line each.
#include <cstdio>

#include <cute/arch/mma_sm100_desc.hpp>
#include <cute/numeric/numeric_types.hpp>

#include "../nvfp4_block_scaled_gsa_b200/csrc/common.cuh"

template <class SF, int M, int N>
uint32_t cutlass_desc() {
  using namespace cute;
  return static_cast<uint32_t>(UMMA::make_instr_desc_block_scaled<
      float_e2m1_t, float_e2m1_t, float, SF, M, N, UMMA::Major::K, UMMA::Major::K>());
}

template <int M, int N>
uint32_t cutlass_mx_with_byte(uint32_t byte) {
  using namespace cute;
  auto d = UMMA::make_instr_desc_block_scaled<float_e2m1_t, float_e2m1_t, float, float_ue8m0_t,
                                              M, N, UMMA::Major::K, UMMA::Major::K>();
  // scale-factor tensor-memory addresses whose top two bits hold the byte index
  const uint64_t r = UMMA::make_runtime_instr_desc_block_scaled(d, byte << 30, byte << 30);
  return static_cast<uint32_t>(r >> 32);
}

int main() {
  using namespace cute;
  std::printf("nvf4_m128_n256 %08x %08x\n", nvfp4::idesc_nvf4(256, 128),
              cutlass_desc<float_ue4m3_t, 128, 256>());
  std::printf("nvf4_m256_n256 %08x %08x\n", nvfp4::idesc_nvf4(256, 256),
              cutlass_desc<float_ue4m3_t, 256, 256>());
  std::printf("nvf4_m128_n128 %08x %08x\n", nvfp4::idesc_nvf4(128, 128),
              cutlass_desc<float_ue4m3_t, 128, 128>());
  std::printf("mxf4_m128_n256 %08x %08x\n", nvfp4::idesc_mxf4(256, 128),
              cutlass_desc<float_ue8m0_t, 128, 256>());
  std::printf("mxf4_m256_n256 %08x %08x\n", nvfp4::idesc_mxf4(256, 256),
              cutlass_desc<float_ue8m0_t, 256, 256>());
  for (uint32_t byte = 0; byte < 4; byte += 2) {
    std::printf("mxf4_m128_n256_byte%u %08x %08x\n", byte,
                nvfp4::idesc_sf_byte(nvfp4::idesc_mxf4(256, 128), byte),
                cutlass_mx_with_byte<128, 256>(byte));
    std::printf("mxf4_m256_n256_byte%u %08x %08x\n", byte,
                nvfp4::idesc_sf_byte(nvfp4::idesc_mxf4(256, 256), byte),
                cutlass_mx_with_byte<256, 256>(byte));
  }
  return 0;
}
