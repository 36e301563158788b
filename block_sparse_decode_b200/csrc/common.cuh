// Shared device helpers of the QSA library: error word, bf16 packing, and the
// inline-PTX wrappers (cp.async, ldmatrix, movmatrix, mma.sync) the kernels
// use. Host-side launchers are declared in launch.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qsa {

// Bits of the device error word (mirrors the flags of qsa_check_device_errors).
enum : unsigned {
  ERR_SEQ = 1u,      // sequence row out of range
  ERR_PAGE = 2u,     // page id out of range
  ERR_BT = 4u,       // block-table column out of range
  ERR_SEL = 8u,      // selected block id out of range
  ERR_LEN = 16u,     // sequence length out of range
  ERR_TIMEOUT = 32u  // bounded wait gave up
};

__device__ __forceinline__ void raise_err(unsigned *err, unsigned bit) {
  atomicOr(err, bit);
}

// ---------------------------------------------------------------- PDL
// Every kernel is launched as a programmatic dependent of the kernel before
// it on the stream (launch_pdl). It may run its prologue while that kernel
// finishes, but every CTA executes pdl_wait() before it touches anything an
// earlier kernel wrote (and before it exits), so the completion of a grid
// still implies the completion of all work before it. pdl_trigger() lets the
// next kernel start launching (its CTAs then wait in pdl_wait for this whole
// grid). A kernel whose CTAs occupy the SMs calls it only once its main work
// is done: dependents placed on the SMs of early finishers slowed the step.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// ---------------------------------------------------------------- bf16

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // RNE, lo in the low half
  return *reinterpret_cast<uint32_t *>(&h);
}

// ---------------------------------------------------------------- cp.async

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global->shared copy; src_bytes = 0 writes 16 zero bytes instead.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- ldmatrix

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                          uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose of one 8x8 b16 matrix held in the m8n8 fragment layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Shared-memory tile of bf16 rows with a 16-byte-chunk XOR swizzle: chunk c of
// row r lives at chunk (c ^ (r & 7)). With rows of 8 or 16 chunks this keeps
// every ldmatrix (8 rows, one chunk column) free of bank conflicts.
__device__ __forceinline__ uint32_t swz(int row, int chunk, int row_bytes) {
  return static_cast<uint32_t>(row * row_bytes + ((chunk ^ (row & 7)) << 4));
}

}  // namespace qsa
