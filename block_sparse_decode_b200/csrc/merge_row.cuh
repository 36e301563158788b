// LSE-weighted combine of one row over R partials, by one warp. Shared by
// the merge kernel and the decode step's fused merge (the last combine CTA
// of a row group), so both produce the same bits.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "Questions worth answering directly": the partial attention results of the
// split read are merged afterwards. With m = max_r LSE_r:
//   O = sum_r e^(LSE_r - m) O_r / sum_r e^(LSE_r - m),  LSE = m + ln sum_r e^(LSE_r - m);
// slices with LSE_r = -inf contribute nothing.
#pragma once

#include "common.cuh"

namespace qsa {

constexpr int MERGE_BATCH = 8;  // slices whose partial outputs are loaded together

// The combine of output row `row` (out [rows, D] bf16 or fp32, lse_out
// [rows] or nullptr) from R partials that the two loaders fetch:
// load_o(r, d0) gives dims d0..d0+3 of slice r's partial output (d0 < D, a
// multiple of 4), load_lse(r) its LSE. The arithmetic does not depend on
// where the partials live, so every caller gets the same bits from the same
// values. Lane r holds the weights of slices r and r + 32 (R <= 64).
template <class LoadO, class LoadL>
__device__ __forceinline__ void merge_row_with(int R, int D, int row, LoadO load_o,
                                               LoadL load_lse, void *out, int out_is_bf16,
                                               float *lse_out) {
  const int lane = threadIdx.x & 31;
  const int passes = (D + 127) / 128;
  // the first batch of partial outputs is requested together with the LSEs
  // (one round trip instead of two when R <= MERGE_BATCH and D <= 128)
  float4 v0[MERGE_BATCH];
  {
    const int d0 = lane * 4;
    const bool live = d0 < D;
#pragma unroll
    for (int u = 0; u < MERGE_BATCH; ++u) {
      const int r = min(u, R - 1);
      v0[u] = live ? load_o(r, d0) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  const float l0 = lane < R ? load_lse(lane) : -INFINITY;
  const float l1 = lane + 32 < R ? load_lse(lane + 32) : -INFINITY;
  float M = fmaxf(l0, l1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w0 = (M == -INFINITY || l0 == -INFINITY) ? 0.f : __expf(l0 - M);
  const float w1 = (M == -INFINITY || l1 == -INFINITY) ? 0.f : __expf(l1 - M);
  float wsum = w0 + w1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  // every lane runs the same number of passes over the head dims (the weight
  // shuffles below need the whole warp); a lane past D loads and stores nothing
  for (int it = 0; it < passes; ++it) {
    const int d0 = it * 128 + lane * 4;
    const bool live = d0 < D;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r0 = 0; r0 < R; r0 += MERGE_BATCH) {
      float4 v[MERGE_BATCH];
#pragma unroll
      for (int u = 0; u < MERGE_BATCH; ++u) {
        const int r = min(r0 + u, R - 1);
        v[u] = it == 0 && r0 == 0 ? v0[u] : live ? load_o(r, d0) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < MERGE_BATCH; ++u) {
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
    if (!live) continue;
    if (out_is_bf16) {
      uint2 pk = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
      *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(out) + (size_t)row * D + d0) = pk;
    } else {
      *reinterpret_cast<float4 *>(static_cast<float *>(out) + (size_t)row * D + d0) = acc;
    }
  }
  if (lane == 0 && lse_out != nullptr) lse_out[row] = wsum > 0.f ? M + logf(wsum) : -INFINITY;
}

// o_part [R, rows, D] and lse_part [R, rows] fp32 in global memory (read
// through L2: they may come from other CTAs of the running grid).
__device__ __forceinline__ void merge_row(int R, int rows, int D, const float *o_part,
                                          const float *lse_part, int row, void *out,
                                          int out_is_bf16, float *lse_out) {
  merge_row_with(
      R, D, row,
      [&](int r, int d0) {
        return __ldcg(reinterpret_cast<const float4 *>(o_part + ((size_t)r * rows + row) * D + d0));
      },
      [&](int r) { return __ldcg(lse_part + (size_t)r * rows + row); }, out, out_is_bf16, lse_out);
}

}  // namespace qsa
