// qsa_merge: log-sum-exp combine of R partial attention results.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes" (second bullet: attention results
// are combined after the split read) and "Questions worth answering
// directly" (partial attention results are merged afterwards). The
// LSE-weighted form is this library's reading:
//   m = max_r LSE_r,  O = sum_r e^(LSE_r - m) O_r / sum_r e^(LSE_r - m),
//   LSE = m + ln sum_r e^(LSE_r - m); slices with LSE_r = -inf are skipped.
// One warp per (sequence, query head). Lane r holds the weight of slices r
// and r + 32 (R <= 64), so the LSEs cost one load round trip; the partial
// outputs are then read MG slices at a time, all loads of a group issued
// before any is used. Traffic is R * (D + 1) * 4 bytes per row; the kernel is
// latency-bound.
#include "common.cuh"
#include "launch.h"

namespace qsa {
namespace {

constexpr int MG = 8;  // slices whose partial outputs are loaded together

__global__ void __launch_bounds__(256) merge_kernel(int R, int rows, int D, const float *o_part,
                                                    const float *lse_part, void *out,
                                                    int out_is_bf16, float *lse_out) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  pdl_wait();
  if (row >= rows) return;
  const float l0 = lane < R ? lse_part[(size_t)lane * rows + row] : -INFINITY;
  const float l1 = lane + 32 < R ? lse_part[(size_t)(lane + 32) * rows + row] : -INFINITY;
  float M = fmaxf(l0, l1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w0 = (M == -INFINITY || l0 == -INFINITY) ? 0.f : __expf(l0 - M);
  const float w1 = (M == -INFINITY || l1 == -INFINITY) ? 0.f : __expf(l1 - M);
  float wsum = w0 + w1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  for (int d0 = lane * 4; d0 < D; d0 += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r0 = 0; r0 < R; r0 += MG) {
      float4 v[MG];
#pragma unroll
      for (int u = 0; u < MG; ++u) {
        const int r = min(r0 + u, R - 1);
        v[u] = *reinterpret_cast<const float4 *>(o_part + ((size_t)r * rows + row) * D + d0);
      }
#pragma unroll
      for (int u = 0; u < MG; ++u) {
        const int r = r0 + u;
        const float f = __shfl_sync(0xffffffffu, r < 32 ? w0 : w1, r & 31);
        if (r < R && f != 0.f) {  // skipped slices (LSE -inf) may hold anything
          acc.x += f * v[u].x;
          acc.y += f * v[u].y;
          acc.z += f * v[u].z;
          acc.w += f * v[u].w;
        }
      }
    }
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
    if (out_is_bf16) {
      uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(out) + (size_t)row * D + d0) = pk;
    } else {
      *reinterpret_cast<float4 *>(static_cast<float *>(out) + (size_t)row * D + d0) = acc;
    }
  }
  if (lane == 0 && lse_out != nullptr) lse_out[row] = wsum > 0.f ? M + logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge(int R, int B, int Hq, int D, const float *o_part, const float *lse_part,
                         void *out, int out_is_bf16, float *lse_out, cudaStream_t st) {
  const int rows = B * Hq;
  if (rows == 0) return cudaSuccess;
  return launch_pdl(merge_kernel, (rows + 7) / 8, 256, 0, st, R, rows, D, o_part, lse_part, out,
                    out_is_bf16, lse_out);
}

}  // namespace qsa
