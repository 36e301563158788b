// qsa_merge: log-sum-exp combine of R partial attention results.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes" (second bullet: attention results
// are combined after the split read) and "Questions worth answering
// directly" (partial attention results are merged afterwards). The
// LSE-weighted form is this library's reading:
//   m = max_r LSE_r,  O = sum_r e^(LSE_r - m) O_r / sum_r e^(LSE_r - m),
//   LSE = m + ln sum_r e^(LSE_r - m); slices with LSE_r = -inf are skipped.
// One warp per (sequence, query head); each lane owns D/32 consecutive dims.
// Traffic is R * (D + 1) * 4 bytes per row; launch-bound in practice.
#include "common.cuh"
#include "launch.h"

namespace qsa {
namespace {

__global__ void __launch_bounds__(256) merge_kernel(int R, int rows, int D, const float *o_part,
                                                    const float *lse_part, void *out,
                                                    int out_is_bf16, float *lse_out) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  pdl_wait();
  if (row >= rows) return;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) M = fmaxf(M, lse_part[(size_t)r * rows + row]);
  float wsum = 0.f;
  for (int d0 = lane * 4; d0 < D; d0 += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    wsum = 0.f;
    if (M != -INFINITY) {
      for (int r = 0; r < R; ++r) {
        const float lse = lse_part[(size_t)r * rows + row];
        if (lse == -INFINITY) continue;
        const float f = __expf(lse - M);
        const float4 v =
            *reinterpret_cast<const float4 *>(o_part + ((size_t)r * rows + row) * D + d0);
        acc.x += f * v.x;
        acc.y += f * v.y;
        acc.z += f * v.z;
        acc.w += f * v.w;
        wsum += f;
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
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
  if (lane == 0 && lse_out != nullptr) {
    if (M == -INFINITY) {
      lse_out[row] = -INFINITY;
    } else {
      float s = 0.f;
      for (int r = 0; r < R; ++r) {
        const float lse = lse_part[(size_t)r * rows + row];
        if (lse != -INFINITY) s += __expf(lse - M);
      }
      lse_out[row] = M + logf(s);
    }
  }
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
