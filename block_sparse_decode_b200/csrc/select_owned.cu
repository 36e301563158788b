// qsa_select_owned: the share of a selection that one rank of a decode
// context-parallel group holds.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": under DCP a rank reads just its
// own part of the main KV cache, the selector is kept whole on every rank,
// and the partial attention results are merged at the end ("Questions worth
// answering directly"). This library's reading of the slice: page p of every sequence
// is held by rank p mod W, so each rank keeps about 1/W of every sequence and
// the split does not move as a sequence grows. Every rank scores and selects
// on the replicated side cache; this kernel keeps the selected blocks whose
// page the rank holds, in the selection's order. One warp per sequence,
// ballot compaction; -1 padded to k.
#include "common.cuh"
#include "launch.h"

namespace qsa {
namespace {

__global__ void __launch_bounds__(128) select_owned_kernel(const int32_t *sel, int B, int k,
                                                           int P, int W, int r, int32_t *out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * 4 + warp;
  pdl_wait();  // the selection comes from the kernel before this one
  if (b >= B) return;
  const int32_t *src = sel + (size_t)b * k;
  int32_t *dst = out + (size_t)b * k;
  const unsigned lower = (1u << lane) - 1u;
  int pos = 0;
  for (int i0 = 0; i0 < k; i0 += 32) {
    const int i = i0 + lane;
    const int j = i < k ? src[i] : -1;
    const bool own = j >= 0 && ((4 * (long long)j) / P) % W == r;
    const unsigned m = __ballot_sync(0xffffffffu, own);
    if (own) dst[pos + __popc(m & lower)] = j;
    pos += __popc(m);
  }
  for (int i = pos + lane; i < k; i += 32) dst[i] = -1;
}

}  // namespace

cudaError_t launch_select_owned(const int32_t *sel, int B, int k, int P, int W, int r,
                                int32_t *out, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  return launch_pdl(select_owned_kernel, (B + 3) / 4, 128, 0, st, sel, B, k, P, W, r, out);
}

}  // namespace qsa
