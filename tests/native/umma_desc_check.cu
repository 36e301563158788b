// Host-only check: the library's tcgen05 descriptor packing equals the
// bitfield definitions of CUTLASS/CuTe (cute/arch/mma_sm100_desc.hpp).
#include <cstdio>
#include <cute/arch/mma_sm100_desc.hpp>
#include <cute/numeric/numeric_types.hpp>

#include "umma_desc.h"

int main() {
  int bad = 0;
  for (uint32_t addr : {0x0u, 0x400u, 0x2420u, 0x1FC60u, 0x3FFF0u}) {
    cute::UMMA::SmemDescriptor d;
    d.desc_ = 0;
    d.start_address_ = (addr & 0x3FFFFu) >> 4;
    d.leading_byte_offset_ = 1;
    d.stride_byte_offset_ = 1024 >> 4;
    d.version_ = 1;
    d.base_offset_ = 0;
    d.lbo_mode_ = 0;
    d.layout_type_ = uint8_t(cute::UMMA::LayoutType::SWIZZLE_128B);
    if (d.desc_ != qsa::sw128_desc(addr)) {
      std::printf("smem desc mismatch at 0x%x: %llx vs %llx\n", addr,
                  (unsigned long long)d.desc_, (unsigned long long)qsa::sw128_desc(addr));
      ++bad;
    }
  }
  using K = cute::UMMA::Major;
  const uint32_t a16 = uint32_t(cute::UMMA::make_instr_desc<cute::bfloat16_t, cute::bfloat16_t,
                                                              float, 128, 16, K::K, K::K>());
  const uint32_t a32 = uint32_t(cute::UMMA::make_instr_desc<cute::bfloat16_t, cute::bfloat16_t,
                                                              float, 128, 32, K::K, K::K>());
  if (a16 != qsa::f16_idesc(128, 16)) { std::printf("idesc N=16 mismatch %x vs %x\n", a16, qsa::f16_idesc(128, 16)); ++bad; }
  if (a32 != qsa::f16_idesc(128, 32)) { std::printf("idesc N=32 mismatch %x vs %x\n", a32, qsa::f16_idesc(128, 32)); ++bad; }
  std::printf(bad ? "FAIL\n" : "OK\n");
  return bad ? 1 : 0;
}
