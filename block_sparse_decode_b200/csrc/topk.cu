// qsa_topk_select: per sequence, the k best micro-blocks by (score desc,
// block index asc), written in ascending block order and padded with -1.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": the indexer retains the top 512
// micro-blocks of a sequence (near 2,048 tokens). The lower-index tie-break
// and the ascending output order are this library's reading.
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

#include <algorithm>

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
  // decode step only (cluster kernel): for every sequence, the R + 1 slice
  // starts of the selection, st[r] = number of selected blocks below
  // floor(r nb / R) (st[R] = all of them), [B, R + 1]; nullptr: none
  int32_t *starts;
  int R;
};

// Order-preserving map of fp32 onto uint32 (larger float -> larger key);
// -0.0 maps like +0.0.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// CS CTAs per sequence (a cluster of 8 or 4): the host picks the larger one
// that keeps every cluster of the batch resident at two CTAs per SM.
template <int CS, bool WS>  // WS: write the decode step's slice starts
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
  int32_t *st_row = WS ? a.starts + (size_t)b * (a.R + 1) : nullptr;
  if (L < 0 || nb > a.ld) {  // uniform over the cluster
    if (crank == 0 && tid == 0) raise_err(a.err, ERR_LEN);
    for (int i = crank * TK_THREADS + tid; i < a.k; i += CS * TK_THREADS) out[i] = -1;
    if (WS && crank == 0)
      for (int r = tid; r <= a.R; r += TK_THREADS) st_row[r] = 0;
    return;
  }
  if (nb <= a.k) {  // every block is kept
    for (int i = crank * TK_THREADS + tid; i < a.k; i += CS * TK_THREADS)
      out[i] = i < nb ? i : -1;
    if (WS && crank == 0)  // block j sits at position j
      for (int r = tid; r <= a.R; r += TK_THREADS) st_row[r] = (int)(((long long)r * nb) / a.R);
    return;
  }

  const int chunk = (nb + CS - 1) / CS;
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
      unsigned v[CS];
#pragma unroll
      for (int r = 0; r < CS; ++r)
        v[r] = cluster.map_shared_rank(&hist[buf][0], r)[255 - tid];
#pragma unroll
      for (int r = 0; r < CS; ++r) c += v[r];
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
    unsigned rg[CS], re[CS];
#pragma unroll
    for (int r = 0; r < CS; ++r) {
      const unsigned *rt = cluster.map_shared_rank(&ctot[0], r < crank ? r : crank);
      rg[r] = rt[0];
      re[r] = rt[1];
    }
#pragma unroll
    for (int r = 0; r < CS; ++r) {
      if (r < crank) {
        run_gt += rg[r];
        run_eq += re[r];
      }
    }
  }
  cluster.sync();  // no CTA leaves while another still reads its counts

  const unsigned lower = (1u << lane) - 1u;
  // slice boundaries floor(r nb / R), 0 < r < R, in this warp's segment (the
  // first one at or past its start): the lane holding that block writes the
  // number of winners before it
  int rc = 1, jb = 0x7fffffff;  // next boundary index and its block (none: INT_MAX)
  if (WS) {
    while (rc < a.R && (rc * nb) / a.R < lo + s0) ++rc;
    if (rc < a.R) jb = (rc * nb) / a.R;
    if (crank == 0 && tid == 0) {
      st_row[0] = 0;
      st_row[a.R] = a.k;  // nb > k: exactly k winners
    }
  }
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
    // (warp-uniform; a division only per boundary passed; r * nb < 2^25)
    while (WS && jb < lo + min(base + 32, s1)) {
      if (lo + i == jb) st_row[rc] = (int)(gb + min(eb, (unsigned)take_eq));
      ++rc;
      jb = rc < a.R ? (rc * nb) / a.R : 0x7fffffff;
    }
    run_gt += __popc(bg);
    run_eq += __popc(be);
  }
}

// ---------------------------------------------------------------------------
// One CTA per sequence (rows of a prefill, or any batch whose score rows fit):
// the upper 16 bits of every key in shared memory (2 bytes per block), two
// 8-bit radix passes over them, then two over the low 16 bits of only the
// keys equal to the 16-bit threshold, re-read from global memory (the score
// row is L2-resident right after scoring). The passes synchronise with block
// barriers only; a pass over a whole row costs a few microseconds of issue
// time on one SM, so the kernel makes three: the load (with the first
// digit's counts), the second digit's counts, and a gather of every key at
// or above the 16-bit threshold into a list (the k winners plus the keys
// tied with the threshold on the upper half, a few hundred beyond k). The
// low-half passes and the index tie-break run on that list, and the winners
// reach the output in ascending order through a bitmap of the row and one
// block-wide scan of its word counts. A list that overflows TR_GATHER (a
// row of largely equal scores) takes the slow path: the tied keys' low
// halves are listed (or, beyond TR_CAND, re-read from global memory in every
// pass) and two more passes over the row count and compact the winners;
// each warp owns a contiguous segment of the row, so that compaction writes
// ascending indices with one block-wide count exchange.
constexpr int TR_THREADS = 1024;
constexpr int TR_WARPS = TR_THREADS / 32;
constexpr int TR_LOADS = 16;   // score loads per lane issued together
constexpr int TR_CAND = 2048;    // keys tied on the upper half kept as a list (slow path)
constexpr int TR_GATHER = 4096;  // keys at or above the upper-half threshold (fast path)

__host__ __device__ inline size_t tr_k16_bytes(int ld) { return ((size_t)ld * 2 + 15) / 16 * 16; }
__host__ __device__ inline size_t tr_bit_bytes(int ld) {
  return (((size_t)ld + 31) / 32 * 4 + 15) / 16 * 16;
}

// Digit with cum >= need > cum - count over 256 descending bins, chosen by
// the CTA's first 256 threads from the per-warp histograms; every thread
// returns (digit, keys above it, keys in it) through pick.
__device__ __forceinline__ void tr_pick(unsigned (*whist)[256], unsigned *wtot, int *pick,
                                        int need) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned c = 0u, cum = 0u;
  if (tid < 256) {
#pragma unroll 8
    for (int w = 0; w < TR_WARPS; ++w) c += whist[w][255 - tid];
    cum = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, cum, o);
      if (lane >= o) cum += y;
    }
    if (lane == 31) wtot[warp] = cum;
  }
  __syncthreads();
  if (tid < 256) {
    for (int w = 0; w < warp; ++w) cum += wtot[w];
    if (cum >= (unsigned)need && cum - c < (unsigned)need) {
      pick[0] = 255 - tid;
      pick[1] = (int)(cum - c);
      pick[2] = (int)c;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(TR_THREADS, 1) topk_row_kernel(TopkArgs a) {
  // dynamic: [upper key halves of the row][bitmap of the row][gather list:
  // indices, keys] (the slow path's tied-key list reuses the indices)
  extern __shared__ __align__(16) unsigned char tr_dyn[];
  __shared__ unsigned whist[TR_WARPS][256];     // per-warp digit counts
  __shared__ unsigned wtot[8];
  __shared__ int pick[3];
  __shared__ unsigned wgt[TR_WARPS], weq[TR_WARPS];
  __shared__ int ncand;
  const int b = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const unsigned lower = (1u << lane) - 1u;
  const int L = a.seq_lens[b];
  const int nb = L < 0 ? 0 : (L + 3) >> 2;
  int32_t *out = a.sel + (size_t)b * a.k;
  uint16_t *k16 = reinterpret_cast<uint16_t *>(tr_dyn);
  uint32_t *cbit = reinterpret_cast<uint32_t *>(tr_dyn + tr_k16_bytes(a.ld));
  int *gidx = reinterpret_cast<int *>(tr_dyn + tr_k16_bytes(a.ld) + tr_bit_bytes(a.ld));
  uint32_t *gkey = reinterpret_cast<uint32_t *>(gidx + TR_GATHER);
  int *clist = gidx;
  pdl_wait();  // the scores come from the kernel before this one
  if (L < 0 || nb > a.ld) {
    if (tid == 0) raise_err(a.err, ERR_LEN);
    for (int i = tid; i < a.k; i += TR_THREADS) out[i] = -1;
    return;
  }
  if (nb <= a.k) {
    for (int i = tid; i < a.k; i += TR_THREADS) out[i] = i < nb ? i : -1;
    return;
  }
  const float *src = a.scores + (size_t)b * a.ld;
  // warp segments: whole 32-key rounds, so every ballot sees a full warp
  const int seg = ((nb + TR_WARPS - 1) / TR_WARPS + 31) & ~31;
  const int s0 = min(nb, warp * seg), s1 = min(nb, s0 + seg);
  for (int i = lane; i < 256; i += 32) whist[warp][i] = 0u;
  __syncwarp();
  // load: keys' upper halves to shared memory, first-digit counts
  for (int i0 = s0; i0 < s1; i0 += 32 * TR_LOADS) {
    float v[TR_LOADS];
#pragma unroll
    for (int u = 0; u < TR_LOADS; ++u) {
      const int i = i0 + 32 * u + lane;
      v[u] = i < s1 ? src[i] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < TR_LOADS; ++u) {
      const int i = i0 + 32 * u + lane;
      if (i < s1) {
        const uint32_t key = score_key(v[u]);
        k16[i] = (uint16_t)(key >> 16);
        atomicAdd(&whist[warp][key >> 24], 1u);
      }
    }
  }
  __syncthreads();
  int need = a.k;
  tr_pick(whist, wtot, pick, need);
  const uint32_t d1 = (uint32_t)pick[0];
  need -= pick[1];
  uint32_t prefix = d1 << 24, mask = 0xFF000000u;
  bool done = pick[2] == need;
  if (!done) {  // second digit: bits 23..16
    for (int i = lane; i < 256; i += 32) whist[warp][i] = 0u;
    __syncwarp();
    // two keys per lane per round (s0 is even; a read past s1 stays inside
    // the shared buffer and is ignored)
    for (int i = s0 + 2 * lane; i < s1; i += 64) {
      const uint32_t x = *reinterpret_cast<const uint32_t *>(k16 + i);
      const uint32_t h0 = x & 0xFFFFu, h1 = x >> 16;
      if ((h0 >> 8) == d1) atomicAdd(&whist[warp][h0 & 255u], 1u);
      if (i + 1 < s1 && (h1 >> 8) == d1) atomicAdd(&whist[warp][h1 & 255u], 1u);
    }
    __syncthreads();
    tr_pick(whist, wtot, pick, need);
    prefix |= (uint32_t)pick[0] << 16;
    mask = 0xFFFF0000u;
    need -= pick[1];
    done = pick[2] == need;
  }
  const uint32_t t16 = prefix >> 16;
  {
    // ---- fast path: the keys whose upper bits (under the mask) are at or
    // above the threshold's: every winner, plus the ties still open
    const uint32_t pm = prefix & 0xFFFF0000u, mu = mask & 0xFFFF0000u;
    const int nw = (nb + 31) / 32;
    for (int i = tid; i < nw; i += TR_THREADS) cbit[i] = 0u;
    if (tid == 0) ncand = 0;
    __syncthreads();
    for (int base = s0; base < s1; base += 64) {  // two keys per lane per round
      const int i = base + 2 * lane;
      const uint32_t x = i < s1 ? *reinterpret_cast<const uint32_t *>(k16 + i) : 0u;
      const bool c0 = i < s1 && ((x << 16) & mu) >= pm;
      const bool c1 = i + 1 < s1 && ((x & 0xFFFF0000u) & mu) >= pm;
      const unsigned m0 = __ballot_sync(0xffffffffu, c0), m1 = __ballot_sync(0xffffffffu, c1);
      if ((m0 | m1) != 0u) {
        int off = 0;
        if (lane == 0) off = atomicAdd(&ncand, __popc(m0) + __popc(m1));
        off = __shfl_sync(0xffffffffu, off, 0);
        const int p0 = off + __popc(m0 & lower), p1 = off + __popc(m0) + __popc(m1 & lower);
        if (c0 && p0 < TR_GATHER) gidx[p0] = i;
        if (c1 && p1 < TR_GATHER) gidx[p1] = i + 1;
      }
    }
    __syncthreads();
    const int ng = ncand;
    if (ng <= TR_GATHER) {
      const bool open = !done;  // ties on the upper half still to resolve
      if (open) {
        for (int j = tid; j < ng; j += TR_THREADS) {
          const int i = gidx[j];
          gkey[j] = k16[i] == t16 ? score_key(src[i]) : 0xFFFFFFFFu;
        }
        __syncthreads();
        for (int pass = 0; pass < 2 && !done; ++pass) {  // bits 15..8, then 7..0
          const int shift = 8 - 8 * pass;
          for (int i = lane; i < 256; i += 32) whist[warp][i] = 0u;
          __syncwarp();
          for (int j = tid; j < ng; j += TR_THREADS) {
            if (k16[gidx[j]] != t16) continue;
            const uint32_t key = gkey[j];
            if ((key & mask) == prefix) atomicAdd(&whist[warp][(key >> shift) & 255u], 1u);
          }
          __syncthreads();
          tr_pick(whist, wtot, pick, need);
          prefix |= (uint32_t)pick[0] << shift;
          mask |= 255u << shift;
          need -= pick[1];
          done = pick[2] == need;
        }
      }
      pdl_trigger();
      // winners: every listed key above the threshold under the final mask,
      // and the first `need` (by index) equal to it
      auto state = [&](int j) -> int {  // +1 above, 0 equal, -1 below
        if (!open || k16[gidx[j]] != t16) return 1;
        const uint32_t m = gkey[j] & mask;
        return m > prefix ? 1 : (m == prefix ? 0 : -1);
      };
      // the equal keys' indices listed once (the per-warp histograms are
      // free now), each ranked against that short list only
      int *eql = reinterpret_cast<int *>(&whist[0][0]);
      if (tid == 0) ncand = 0;
      __syncthreads();
      for (int j = tid; j < ng; j += TR_THREADS) {
        const int st = state(j);
        if (st > 0) atomicOr(&cbit[gidx[j] >> 5], 1u << (gidx[j] & 31));
        if (st == 0) eql[atomicAdd(&ncand, 1)] = gidx[j];
      }
      __syncthreads();
      const int ne = ncand;
      for (int e = tid; e < ne; e += TR_THREADS) {
        const int i = eql[e];
        int before = 0;  // equal keys with a lower index
        for (int f = 0; f < ne; ++f) before += eql[f] < i ? 1 : 0;
        if (before < need) atomicOr(&cbit[i >> 5], 1u << (i & 31));
      }
      __syncthreads();
      // the bitmap's words in contiguous runs per thread, one scan of counts
      const int wpt = (nw + TR_THREADS - 1) / TR_THREADS;
      const int w0 = min(nw, tid * wpt), w1 = min(nw, w0 + wpt);
      unsigned cnt = 0u;
      for (int w = w0; w < w1; ++w) cnt += __popc(cbit[w]);
      unsigned incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) wgt[warp] = incl;
      __syncthreads();
      unsigned pos = incl - cnt;
      for (int w = 0; w < warp; ++w) pos += wgt[w];
      for (int w = w0; w < w1; ++w) {
        unsigned bits = cbit[w];
        while (bits != 0u) {
          const int bit = __ffs(bits) - 1;
          if (pos < (unsigned)a.k) out[pos] = 32 * w + bit;
          ++pos;
          bits &= bits - 1u;
        }
      }
      return;
    }
  }
  // ---- slow path (more than TR_GATHER keys at or above the upper threshold)
  bool have_low = false;  // the tied keys' low halves are in k16 (marked in cbit)
  int nc = 0;
  if (!done) {
    for (int i = tid; i < (nb + 31) / 32; i += TR_THREADS) cbit[i] = 0u;
    if (tid == 0) ncand = 0;
    __syncthreads();
    for (int base = s0; base < s1; base += 32) {
      const int i = base + lane;
      const bool c = i < s1 && k16[i] == t16;
      const unsigned m = __ballot_sync(0xffffffffu, c);
      if (m != 0u) {
        int off = 0;
        if (lane == 0) off = atomicAdd(&ncand, __popc(m));
        off = __shfl_sync(0xffffffffu, off, 0);
        const int p = off + __popc(m & lower);
        if (c && p < TR_CAND) clist[p] = i;
      }
    }
    __syncthreads();
    nc = ncand;
    if (nc <= TR_CAND) {
      for (int j = tid; j < nc; j += TR_THREADS) {
        const int i = clist[j];
        k16[i] = (uint16_t)(score_key(src[i]) & 0xFFFFu);
        atomicOr(&cbit[i >> 5], 1u << (i & 31));
      }
      have_low = true;
    }
    __syncthreads();
  }
  for (int pass = 0; pass < 2 && !done; ++pass) {  // bits 15..8, then 7..0
    const int shift = 8 - 8 * pass;
    for (int i = lane; i < 256; i += 32) whist[warp][i] = 0u;
    __syncwarp();
    if (have_low) {
      for (int j = tid; j < nc; j += TR_THREADS) {
        const uint32_t key = (t16 << 16) | k16[clist[j]];
        if ((key & mask) == prefix) atomicAdd(&whist[warp][(key >> shift) & 255u], 1u);
      }
    } else {
      for (int i = s0 + lane; i < s1; i += 32) {
        if (k16[i] == t16) {
          const uint32_t key = score_key(src[i]);
          if ((key & mask) == prefix) atomicAdd(&whist[warp][(key >> shift) & 255u], 1u);
        }
      }
    }
    __syncthreads();
    tr_pick(whist, wtot, pick, need);
    prefix |= (uint32_t)pick[0] << shift;
    mask |= 255u << shift;
    need -= pick[1];
    done = pick[2] == need;
  }
  pdl_trigger();
  const int take_eq = need;
  // (masked key vs prefix) of block i: +1 above, 0 equal, -1 below; the
  // low half is read from global memory only when the upper halves tie
  auto cmp = [&](int i) -> int {
    if (have_low && ((cbit[i >> 5] >> (i & 31)) & 1u)) {
      const uint32_t m = ((t16 << 16) | k16[i]) & mask;
      return m > prefix ? 1 : (m == prefix ? 0 : -1);
    }
    const uint32_t hm = ((uint32_t)k16[i] << 16) & mask, pm = prefix & 0xFFFF0000u;
    if (hm != pm) return hm > pm ? 1 : -1;
    if ((mask & 0xFFFFu) == 0u) return 0;
    const uint32_t m = score_key(src[i]) & mask;
    return m > prefix ? 1 : (m == prefix ? 0 : -1);
  };
  unsigned gt = 0u, eq = 0u;
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const int c = i < s1 ? cmp(i) : -1;
    gt += __popc(__ballot_sync(0xffffffffu, c > 0));
    eq += __popc(__ballot_sync(0xffffffffu, c == 0));
  }
  if (lane == 0) { wgt[warp] = gt; weq[warp] = eq; }
  __syncthreads();
  unsigned run_gt = 0u, run_eq = 0u;
  for (int w = 0; w < warp; ++w) { run_gt += wgt[w]; run_eq += weq[w]; }
  for (int base = s0; base < s1; base += 32) {
    const int i = base + lane;
    const int c = i < s1 ? cmp(i) : -1;
    const unsigned bg = __ballot_sync(0xffffffffu, c > 0);
    const unsigned be = __ballot_sync(0xffffffffu, c == 0);
    const unsigned gb = run_gt + __popc(bg & lower), eb = run_eq + __popc(be & lower);
    const unsigned pos = c > 0 ? gb + min(eb, (unsigned)take_eq) : gb + eb;
    if ((c > 0 || (c == 0 && eb < (unsigned)take_eq)) && pos < (unsigned)a.k) out[pos] = i;
    run_gt += __popc(bg);
    run_eq += __popc(be);
  }
}

}  // namespace

cudaError_t launch_topk(int B, const int32_t *seq_lens, const float *scores, int ld, int k,
                        int32_t *sel, unsigned *err, cudaStream_t st, int32_t *starts, int R,
                        bool *wrote_starts) {
  if (wrote_starts != nullptr) *wrote_starts = false;
  if (B == 0) return cudaSuccess;
  TopkArgs a{scores, seq_lens, sel, ld, k, err, nullptr, R};
  // clusters of CS CTAs while the batch's clusters all fit at two CTAs per SM
  // (largest CS first, each CTA's keys within its shared memory); beyond
  // that, one CTA per sequence for rows it can hold, else clusters of 8
  // (clusters of 2 were measured slower than one CTA per row: 25.6 against
  // 20.5 us for 128 rows of 16,384 blocks)
  int cs = 0;
  for (int c = TOPK_CLUSTER; c >= 4 && cs == 0; c >>= 1) {
    const long long keys_b = (long long)((ld + c - 1) / c) * 4;
    // CTAs per SM: two by registers (512 threads), fewer if the keys need it
    // (the kernel's own shared arrays and 1 KiB reserved per CTA besides)
    const long long per_sm = std::min<long long>(2, (228 * 1024) / (keys_b + 20 * 1024));
    if (keys_b <= (long long)TOPK_MAX_KEYS_PER_CTA * 4 && per_sm > 0 &&
        (long long)B * c <= per_sm * device_sm_count())
      cs = c;
  }
  if (cs == 0 && B >= TOPK_ROW_MIN_B && ld <= TOPK_ROW_MAX_KEYS) {
    const size_t smem = tr_k16_bytes(ld) + tr_bit_bytes(ld) + (size_t)TR_GATHER * 8;
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void *>(topk_row_kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_row_kernel, B, TR_THREADS, smem, st, a);
  }
  if (cs == 0) cs = TOPK_CLUSTER;
  a.starts = starts;  // the cluster kernel writes the slice starts
  if (wrote_starts != nullptr) *wrote_starts = starts != nullptr;
  const bool ws = starts != nullptr;
  const void *kern = cs == 8 ? (ws ? reinterpret_cast<const void *>(topk_kernel<8, true>)
                                   : reinterpret_cast<const void *>(topk_kernel<8, false>))
                             : (ws ? reinterpret_cast<const void *>(topk_kernel<4, true>)
                                   : reinterpret_cast<const void *>(topk_kernel<4, false>));
  const int per_cta = (ld + cs - 1) / cs;
  const size_t smem = (size_t)per_cta * 4;
  cudaError_t e = ensure_dynamic_smem(kern, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, B, 1);
  cfg.blockDim = dim3(TK_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cs == 8)
    return ws ? cudaLaunchKernelEx(&cfg, topk_kernel<8, true>, a)
              : cudaLaunchKernelEx(&cfg, topk_kernel<8, false>, a);
  return ws ? cudaLaunchKernelEx(&cfg, topk_kernel<4, true>, a)
            : cudaLaunchKernelEx(&cfg, topk_kernel<4, false>, a);
}

}  // namespace qsa
