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
// and r + 32 (R <= 64; merge_row.cuh), so the LSEs cost one load round trip; the partial
// outputs are then read MERGE_BATCH slices at a time, all loads of a group issued
// before any is used. Traffic is R * (D + 1) * 4 bytes per row; the kernel is
// latency-bound.
#include "common.cuh"
#include "launch.h"
#include "merge_row.cuh"

namespace qsa {
namespace {

__global__ void __launch_bounds__(256) merge_kernel(int R, int rows, int D, const float *o_part,
                                                    const float *lse_part, void *out,
                                                    int out_is_bf16, float *lse_out) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  pdl_wait();
  if (row >= rows) return;
  merge_row(R, rows, D, o_part, lse_part, row, out, out_is_bf16, lse_out);
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
