// qsa_topk_select: per sequence, the k best micro-blocks by (score desc,
// block index asc), written in ascending block order and padded with -1.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": the indexer "keeps the best 512
// blocks, roughly 2,048 token positions". The lower-index tie-break and the
// ascending output order are this library's reading.
//
// Design: one thread-block cluster of 8 CTAs per sequence. Each CTA holds a
// contiguous eighth of the sequence's scores in shared memory as
// order-preserving 32-bit keys (read from global once). An exact radix select
// over the key bits (4 passes of 8 bits, most significant first) finds the
// k-th largest key T and how many keys equal to T are taken: every pass
// counts the digits of the keys still matching the prefix into a per-CTA
// histogram (per-warp shared histograms), the 8 histograms are summed
// through distributed shared memory, and every CTA picks the same digit. The
// compaction then writes each selected block at position
//   (#keys > T before it) + min(#keys == T before it, ties taken),
// which is ascending index order; the per-CTA counts are exchanged through
// distributed shared memory again. No global scratch, no atomics on global
// memory and no inter-CTA waits other than cluster barriers.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace qsa {
namespace {

constexpr int TK_THREADS = 512;
constexpr int TK_WARPS = TK_THREADS / 32;
constexpr int TK_LOADS = 16;  // score loads per thread issued together

struct TopkArgs {
  const float *scores;
  const int32_t *seq_lens;
  int32_t *sel;
  int ld, k;
  unsigned *err;
};

// Order-preserving map of fp32 onto uint32 (larger float -> larger key);
// -0.0 maps like +0.0.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(TK_THREADS, 1) topk_kernel(TopkArgs a) {
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const int b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  extern __shared__ uint32_t keys[];
  __shared__ unsigned whist[TK_WARPS][256];  // per-warp digit counts
  __shared__ unsigned hist[2][256];          // this CTA's counts (double-buffered)
  __shared__ unsigned wtot[TK_WARPS];
  __shared__ int pick[3];                    // digit, keys above it, keys in it
  __shared__ unsigned ctot[2];               // this CTA's (#keys > T, #keys == T)
  __shared__ unsigned wgt[TK_WARPS], weq[TK_WARPS];

  const int L = a.seq_lens[b];
  const int nb = L < 0 ? 0 : (L + 3) >> 2;
  int32_t *out = a.sel + (size_t)b * a.k;
  pdl_wait();  // the scores come from the kernel before this one
  if (L < 0 || nb > a.ld) {  // uniform over the cluster
    if (crank == 0 && tid == 0) raise_err(a.err, ERR_LEN);
    for (int i = crank * TK_THREADS + tid; i < a.k; i += TOPK_CLUSTER * TK_THREADS) out[i] = -1;
    return;
  }
  if (nb <= a.k) {  // every block is kept
    for (int i = crank * TK_THREADS + tid; i < a.k; i += TOPK_CLUSTER * TK_THREADS)
      out[i] = i < nb ? i : -1;
    return;
  }

  const int chunk = (nb + TOPK_CLUSTER - 1) / TOPK_CLUSTER;
  const int lo = min(nb, crank * chunk);
  const int n = min(nb, lo + chunk) - lo;
  const float *src = a.scores + (size_t)b * a.ld + lo;
  // TK_LOADS loads per thread in flight before any is used
  for (int i0 = 0; i0 < n; i0 += TK_THREADS * TK_LOADS) {
    float v[TK_LOADS];
#pragma unroll
    for (int u = 0; u < TK_LOADS; ++u) {
      const int i = i0 + u * TK_THREADS + tid;
      v[u] = i < n ? src[i] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < TK_LOADS; ++u) {
      const int i = i0 + u * TK_THREADS + tid;
      if (i < n) keys[i] = score_key(v[u]);
    }
  }
  if (tid == 0) { pick[0] = 0; pick[1] = 0; pick[2] = 0; }

  // contiguous per-warp segments of the CTA's range
  const int seg = (n + TK_WARPS - 1) / TK_WARPS;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);

  uint32_t prefix = 0u, mask = 0u;
  int need = a.k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass, buf = pass & 1;
    // (hist[buf] was last read by the other CTAs before the previous cluster
    // barrier, so it can be rewritten now)
    for (int i = lane; i < 256; i += 32) whist[warp][i] = 0u;
    __syncthreads();  // keys loaded (first pass), pick[] of the last pass read
    for (int i = s0 + lane; i < s1; i += 32) {
      const uint32_t key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&whist[warp][(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 256) {
      unsigned c = 0u;
#pragma unroll
      for (int w = 0; w < TK_WARPS; ++w) c += whist[w][tid];
      hist[buf][tid] = c;
    }
    cluster.sync();
    // sum the 8 histograms; thread t takes digit 255 - t (descending order)
    unsigned c = 0u, cum = 0u;
    if (tid < 256) {
      unsigned v[TOPK_CLUSTER];
#pragma unroll
      for (int r = 0; r < TOPK_CLUSTER; ++r)
        v[r] = cluster.map_shared_rank(&hist[buf][0], r)[255 - tid];
#pragma unroll
      for (int r = 0; r < TOPK_CLUSTER; ++r) c += v[r];
      cum = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        unsigned y = __shfl_up_sync(0xffffffffu, cum, o);
        if (lane >= o) cum += y;
      }
      if (lane == 31) wtot[warp] = cum;
    }
    __syncthreads();
    if (tid < 256) {
      for (int w = 0; w < warp; ++w) cum += wtot[w];
      if (cum >= (unsigned)need && cum - c < (unsigned)need) {
        pick[0] = 255 - tid;
        pick[1] = (int)(cum - c);  // keys with a larger digit under the prefix
        pick[2] = (int)c;          // keys with this digit under the prefix
      }
    }
    __syncthreads();
    prefix |= (uint32_t)pick[0] << shift;
    mask |= 255u << shift;
    need -= pick[1];
    if (pick[2] == need) break;  // every key left under the prefix is kept
  }
  pdl_trigger();
  // Selection: keys whose masked value is above the prefix, plus the first
  // `need` (lowest index) keys equal to it under the mask.
  const int take_eq = need;

  unsigned gt = 0u, eq = 0u;
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const uint32_t key = (i < s1 ? keys[i] : 0u) & mask;
    gt += __popc(__ballot_sync(0xffffffffu, i < s1 && key > prefix));
    eq += __popc(__ballot_sync(0xffffffffu, i < s1 && key == prefix));
  }
  if (lane == 0) { wgt[warp] = gt; weq[warp] = eq; }
  __syncthreads();
  unsigned run_gt = 0u, run_eq = 0u;
  for (int w = 0; w < warp; ++w) { run_gt += wgt[w]; run_eq += weq[w]; }
  if (tid == 0) {
    unsigned tg = 0u, te = 0u;
    for (int w = 0; w < TK_WARPS; ++w) { tg += wgt[w]; te += weq[w]; }
    ctot[0] = tg;
    ctot[1] = te;
  }
  cluster.sync();
  {
    // the counts of every lower-ranked CTA, all loads in flight together
    unsigned rg[TOPK_CLUSTER], re[TOPK_CLUSTER];
#pragma unroll
    for (int r = 0; r < TOPK_CLUSTER; ++r) {
      const unsigned *rt = cluster.map_shared_rank(&ctot[0], r < crank ? r : crank);
      rg[r] = rt[0];
      re[r] = rt[1];
    }
#pragma unroll
    for (int r = 0; r < TOPK_CLUSTER; ++r) {
      if (r < crank) {
        run_gt += rg[r];
        run_eq += re[r];
      }
    }
  }
  cluster.sync();  // no CTA leaves while another still reads its counts

  const unsigned lower = (1u << lane) - 1u;
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const uint32_t key = (i < s1 ? keys[i] : 0u) & mask;
    const bool is_gt = i < s1 && key > prefix, is_eq = i < s1 && key == prefix;
    const unsigned bg = __ballot_sync(0xffffffffu, is_gt);
    const unsigned be = __ballot_sync(0xffffffffu, is_eq);
    const unsigned gb = run_gt + __popc(bg & lower), eb = run_eq + __popc(be & lower);
    // positions stay below k by construction; the bound only guards the buffer
    const unsigned pos = is_gt ? gb + min(eb, (unsigned)take_eq) : gb + eb;
    if ((is_gt || (is_eq && eb < (unsigned)take_eq)) && pos < (unsigned)a.k) out[pos] = lo + i;
    run_gt += __popc(bg);
    run_eq += __popc(be);
  }
}

}  // namespace

cudaError_t launch_topk(int B, const int32_t *seq_lens, const float *scores, int ld, int k,
                        int32_t *sel, unsigned *err, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  TopkArgs a{scores, seq_lens, sel, ld, k, err};
  const int per_cta = (ld + TOPK_CLUSTER - 1) / TOPK_CLUSTER;
  const size_t smem = (size_t)per_cta * 4;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(topk_kernel), smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(TOPK_CLUSTER, B, 1);
  cfg.blockDim = dim3(TK_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = TOPK_CLUSTER;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, topk_kernel, a);
}

}  // namespace qsa
