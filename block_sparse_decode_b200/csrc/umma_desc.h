// Bit packing of the two tcgen05.mma descriptors used by the scoring kernel
// (PTX ISA, "tcgen05 matrix descriptors" and "instruction descriptor" for
// .kind::f16). Host- and device-callable so a host test can compare them
// with an independent definition of the same bitfields.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define QSA_HD __host__ __device__
#else
#define QSA_HD
#endif

namespace qsa {

// Shared-memory matrix descriptor for a K-major operand in the 128-byte
// swizzled layout: start address in 16-byte units (bits 0-13), leading byte
// offset 16 B (bits 16-29; not used by this layout), stride byte offset 1024 B
// between 8-row groups (bits 32-45), descriptor version 1 (bits 46-47), base
// offset 0, swizzle mode 2 = 128 B (bits 61-63).
QSA_HD inline uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16 >> 4) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of .kind::f16: dense, fp32 accumulator (bits 4-5 =
// 1), A and B bf16 (bits 7-9 and 10-12 = 1), no negation, both K-major (bits
// 15, 16 = 0), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
QSA_HD constexpr uint32_t f16_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

}  // namespace qsa
