// Sparse prefill for QSA: the indexer scores of every query row of an
// appended chunk.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "Why a serving PR about an unreleased architecture is still worth your
// time": the engine work around the decode path includes a native sparse
// prefill kernel for the QSA path (for Hopper); the page gives none of its
// steps. This library's reading: every token of an appended chunk queries
// like a decode step over its own causal prefix. Sequence s holds the rows
// [row_start[s], row_start[s+1]) (its T_s newest tokens, already appended, so
// L_s = seq_lens[s] counts them); row i of it is the token at position
// L_s - T_s + i and sees the first L_s - T_s + i + 1 tokens.
//
// Scoring shares the side-cache tiles between rows: up to QG = 256 / Hi
// consecutive rows of one sequence form a group, and one tcgen05.mma of
// M = 128 blocks x N = 256 (QG rows x Hi heads) x K = di scores a tile of
// the group's blocks for all of its rows (the decode kernel's N is Hi alone).
// Per tile that is 8x the decode kernel's tensor work on the same 32 KiB of
// side cache, so the kernel is about balanced between the tensor pipe and
// the side-cache stream.
//
// Three kernels, chained by programmatic dependent launch:
//   plan     one CTA: validates the chunk layout, writes every row's causal
//            length (row_len, the top-k's sequence lengths) and sequence, the
//            group list {sequence, first row, rows, complete blocks of its
//            last row} and the groups' tile prefix;
//   partial  one warp per row whose length is not a multiple of 4: the score
//            of its trailing partial block, on CUDA cores;
//   score    persistent, one CTA per SM over a contiguous range of the
//            flattened (group, 128-block tile) list:
//              warps 0-2 producers (tiles round-robin): TMA boxes of the
//                        tile's page pieces into a ring of stages
//              warp 3    TMEM owner; lane 0 loads the group's 256 indexer
//                        query rows into one shared buffer when the group
//                        changes (after the MMAs on the old rows completed)
//                        and issues the MMAs into one of two accumulators
//              warps 4-19 epilogue: four warps per TMEM lane quadrant, each
//                        tcgen05.ld of 32 blocks x 64 columns (a quarter of
//                        the group's rows), per row the head-weighted ReLU
//                        sum, one coalesced store per (row, 32 blocks),
//                        masked to the blocks complete within the row's own
//                        prefix. (With fewer warps the epilogue's TMEM-load
//                        and arithmetic latencies, not the tensor pipe, set
//                        the tile time.)
// Every mbarrier wait is bounded, with the drain of the decode scoring kernel.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"
#include "umma_desc.h"

namespace qsa {
namespace {

constexpr int PF_M = 128;  // blocks per tile
constexpr int PF_N = 256;  // group rows x indexer heads
constexpr int PF_MAX_STAGES = 6;
constexpr int PF_PROD_WARPS = 3;
constexpr int PF_MMA_WARP = PF_PROD_WARPS;
constexpr int PF_EPI0 = PF_PROD_WARPS + 1;
constexpr int PF_EPI_WARPS = 16;  // four per TMEM lane quadrant, each a quarter of the columns
constexpr int PF_EPI_PARTS = PF_EPI_WARPS / 4;
constexpr int PF_EPI_COLS = PF_N / PF_EPI_PARTS;
constexpr int PF_THREADS = 32 * (PF_PROD_WARPS + 1 + PF_EPI_WARPS);
constexpr int PL_THREADS = 1024;

struct PfArgs {
  const __nv_bfloat16 *kidx_pool, *q_idx;  // q_idx [Nq, Hi, DI]
  const float *w;                          // [Nq, Hi]
  const int32_t *block_table, *seq_lens, *row_start;
  int32_t *row_len;  // [Nq] causal length of each row (written by the plan)
  int32_t *row_seq;  // [Nq] its sequence, -1 for a row outside every chunk
  int *hdr;          // [0] groups, [1] tiles
  int *gtile;        // [Gmax + 1] tile prefix over groups
  int4 *ginfo;       // [Gmax] {sequence, first row, rows, complete blocks of the last row}
  float *scores;
  int S, Nq, Gmax, QG, ld, P, rpp, max_pages, num_pages, Hi, stages;
  int box;  // rows per page piece: min(P/4, 128); a tile holds 128 / box pieces
  unsigned *err;
};

struct PfCtrl {
  uint64_t full[PF_MAX_STAGES];
  uint64_t empty[PF_MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t qfull;  // the group's query rows landed
  uint64_t qfree;  // the MMAs on the previous group's rows completed
  uint32_t tmem_base;
  int abort_flag;
  int q_pending;  // parity of a query-row load not yet seen landed, else -1
  int issued[PF_PROD_WARPS];
  int consumed;
  int done;
};

// Block-wide exclusive scan of one value per thread (PL_THREADS threads);
// returns the thread's offset and the block total in *total.
__device__ int plan_scan(int v, int *wsum, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  int off = 0, tot = 0;
  for (int i = 0; i < PL_THREADS / 32; ++i) {
    if (i < warp) off += wsum[i];
    tot += wsum[i];
  }
  __syncthreads();  // wsum is reused by the next call
  *total = tot;
  return off + x - v;
}

__global__ void __launch_bounds__(PL_THREADS) prefill_plan_kernel(PfArgs a) {
  __shared__ int wsum[PL_THREADS / 32];
  const int tid = threadIdx.x;
  pdl_wait();  // the outputs may still be read by the kernel before this one
  // groups of every sequence, in sequence order
  int gbase = 0;
  for (int base = 0; base < a.S; base += PL_THREADS) {
    const int s = base + tid;
    int ng = 0, r0 = 0, T = 0, L = 0;
    if (s < a.S) {
      r0 = a.row_start[s];
      const int r1 = a.row_start[s + 1];
      L = a.seq_lens[s];
      T = r1 - r0;
      // (a chunk past Nq or longer than its sequence, or a context whose
      // blocks do not fit a score row, is skipped: its rows get length 0)
      if (r0 < 0 || T < 0 || r1 > a.Nq || T > L || (long long)L > 4LL * a.ld) {
        raise_err(a.err, ERR_LEN);
      } else {
        ng = (T + a.QG - 1) / a.QG;
      }
    }
    int tot;
    const int off = gbase + plan_scan(ng, wsum, &tot);
    for (int gi = 0; gi < ng; ++gi) {
      const int g = off + gi;
      if (g >= a.Gmax) {  // only overlapping chunks can need more groups than rows allow
        raise_err(a.err, ERR_LEN);
        break;
      }
      const int nr = min(a.QG, T - gi * a.QG);
      const int nfull = (L - T + gi * a.QG + nr) >> 2;
      a.ginfo[g] = make_int4(s, r0 + gi * a.QG, nr, nfull);
      a.gtile[g] = (nfull + PF_M - 1) / PF_M;
    }
    gbase += tot;
  }
  const int G = min(gbase, a.Gmax);
  __syncthreads();  // every group's tile count is written
  int tbase = 0;
  for (int base = 0; base < G; base += PL_THREADS) {
    const int g = base + tid;
    const int n = g < G ? a.gtile[g] : 0;
    int tot;
    const int off = tbase + plan_scan(n, wsum, &tot);  // (its barriers order the reads first)
    if (g < G) a.gtile[g] = off;
    tbase += tot;
  }
  if (tid == 0) {
    a.gtile[G] = tbase;
    a.hdr[0] = G;
    a.hdr[1] = tbase;
  }
  // every row: its sequence (the chunk holding it) and causal length
  for (int r = tid; r < a.Nq; r += PL_THREADS) {
    int lo = 0, hi = a.S - 1;  // last s with row_start[s] <= r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (a.row_start[mid] <= r) lo = mid; else hi = mid - 1;
    }
    int seq = -1, len = 0;
    if (a.S > 0) {
      const int r0 = a.row_start[lo], r1 = a.row_start[lo + 1], L = a.seq_lens[lo];
      if (r0 >= 0 && r0 <= r && r < r1 && r1 <= a.Nq && r1 - r0 <= L &&
          (long long)L <= 4LL * a.ld) {
        seq = lo;
        len = L - (r1 - r0) + (r - r0) + 1;
      }
    }
    a.row_seq[r] = seq;
    a.row_len[r] = len;
  }
}

// The trailing partial block of every row whose length is not a multiple of
// 4 (one warp per row). The scoring kernel never writes that block's score.
template <int DI>
__global__ void __launch_bounds__(256) prefill_partial_kernel(PfArgs a) {
  pdl_wait();  // row_len and row_seq come from the plan kernel
  pdl_trigger();  // the scoring kernel does not touch these blocks
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= a.Nq) return;
  const int L = a.row_len[r], s = a.row_seq[r];
  if (L <= 0 || (L & 3) == 0 || s < 0) return;
  bool ok;
  const float sp = partial_block_score_row<DI>(
      a.kidx_pool, a.P, a.block_table + (size_t)s * a.max_pages, a.max_pages, a.num_pages, L,
      a.q_idx + (size_t)r * a.Hi * DI, a.w + (size_t)r * a.Hi, a.Hi, a.err, &ok);
  if (lane == 0 && ok) a.scores[(size_t)r * a.ld + (L >> 2)] = sp;
}

// group of flattened tile t, searching forward from group g
__device__ __forceinline__ int pf_advance(const int *gtile, int g, int t) {
  while (__ldg(gtile + g + 1) <= t) ++g;
  return g;
}

template <int DI, int HI>
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_score_kernel(const __grid_constant__ CUtensorMap side_map,
                         const __grid_constant__ CUtensorMap q_map, PfArgs a) {
  constexpr int KH = DI / 64;          // 128-byte K halves
  constexpr int QG = PF_N / HI;        // rows per group
  constexpr int A_HALF = PF_M * 128;   // bytes of one A half
  constexpr int Q_HALF = PF_N * 128;   // bytes of one half of the group's query rows
  constexpr int STAGE = KH * A_HALF;
  constexpr int QBYTES = KH * Q_HALF;
  constexpr int KSTEPS = DI / 16;
  constexpr uint32_t IDESC = f16_idesc(PF_M, PF_N);

  extern __shared__ unsigned char smem_raw[];
  __shared__ PfCtrl ctl;
  __shared__ float w_s[PF_EPI_WARPS][PF_EPI_COLS];  // per epilogue warp: its rows' head weights
  __shared__ int nf_s[PF_EPI_WARPS][QG / PF_EPI_PARTS];  // and their complete blocks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;

  // dynamic smem: [pad to 1024][query rows QBYTES][stages x STAGE]
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  const uint32_t q_s = raw_s + pad;
  const uint32_t ring_s = q_s + QBYTES;
  const uint32_t full0 = smem_u32(&ctl.full[0]), empty0 = smem_u32(&ctl.empty[0]);
  const uint32_t tfull0 = smem_u32(&ctl.tfull[0]), tempty0 = smem_u32(&ctl.tempty[0]);
  const uint32_t qfull = smem_u32(&ctl.qfull), qfree = smem_u32(&ctl.qfree);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, PF_EPI_WARPS * 32);
    }
    mbar_init(qfull, 1);
    mbar_init(qfree, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    ctl.abort_flag = 0;
    ctl.q_pending = -1;
    ctl.consumed = ctl.done = 0;
    for (int w = 0; w < PF_PROD_WARPS; ++w) ctl.issued[w] = w;
  }
  if (warp == PF_MMA_WARP) {  // two accumulators of 256 fp32 columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ctl.tmem_base)),
                 "r"(2 * PF_N)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();  // the group list and row lengths come from the kernels before this one
  const uint32_t tmem = ctl.tmem_base;
  volatile int *abort_flag = &ctl.abort_flag;

  // this CTA's contiguous range of the flattened tile list
  const int G = a.hdr[0], total = a.hdr[1];
  const int per = total / (int)gridDim.x, extra = total % (int)gridDim.x;
  const int t0 = (int)blockIdx.x * per + min((int)blockIdx.x, extra);
  const int my_tiles = G > 0 ? per + ((int)blockIdx.x < extra ? 1 : 0) : 0;
  int g_first = 0;
  if (my_tiles > 0) {  // last group whose first tile is <= t0
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(a.gtile + mid) <= t0) lo = mid; else hi = mid - 1;
    }
    g_first = pf_advance(a.gtile, lo, t0);
  }

  if (warp < PF_PROD_WARPS) {
    // ------------------------------------------------------------ producers
    int g = g_first;
    int ti = warp;
    // page ids of a tile's pieces (lane k: piece k), loaded one tile ahead
    auto tile_page = [&](int t, int gg, int &page, int &rip) {
      const int4 gi = __ldg(a.ginfo + gg);
      const int j0 = (t - __ldg(a.gtile + gg)) * PF_M;
      const int rows = max(0, min(PF_M, gi.w - j0));
      const int npiece = (rows + a.box - 1) / a.box;
      page = -1;
      rip = (j0 + lane * a.box) % a.rpp;  // row in page (P > 512 only)
      if (lane < npiece) {
        const int col = (j0 + lane * a.box) / a.rpp;
        if (col >= a.max_pages) {
          raise_err(a.err, ERR_BT);
        } else {
          page = __ldg(a.block_table + (size_t)gi.x * a.max_pages + col);
          if (page < 0 || page >= a.num_pages) {
            if (page != -1) raise_err(a.err, ERR_PAGE);
            page = -1;
          }
        }
      }
    };
    int page = -1, rip = 0;
    if (ti < my_tiles) {
      g = pf_advance(a.gtile, g, t0 + ti);
      tile_page(t0 + ti, g, page, rip);
    }
    for (; ti < my_tiles; ti += PF_PROD_WARPS) {
      int npage = -1, nrip = 0;
      const int tn = ti + PF_PROD_WARPS;
      if (tn < my_tiles) {  // the next tile's page ids, in flight while this one waits
        const int gn = pf_advance(a.gtile, g, t0 + tn);
        tile_page(t0 + tn, gn, npage, nrip);
        g = gn;
      }
      const int s = ti % S;
      const uint32_t ph = (uint32_t)((ti / S) & 1);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, a.err);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      __syncwarp();
      const unsigned live = __ballot_sync(0xffffffffu, page >= 0);
      const uint32_t stage_s = ring_s + (uint32_t)s * STAGE;
      const uint32_t bar = full0 + 8 * s;
      if (lane == 0) mbar_arrive_expect(bar, (uint32_t)(__popc(live) * a.box * 128 * KH));
      __syncwarp();
      if (page >= 0) {
#pragma unroll
        for (int h = 0; h < KH; ++h)
          tma_load_3d(stage_s + h * A_HALF + lane * a.box * 128, &side_map, bar, h * 64, rip,
                      page);
      }
      page = npage;
      rip = nrip;
    }
    if (lane == 0) ctl.issued[warp] = ti;
  } else if (warp == PF_MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0, acc = 0, g = g_first, cur_g = -1;
      uint32_t ph = 0, aph = 0, qph = 0, fph = 0;
      int consumed = 0;
      for (int ti = 0; ti < my_tiles; ++ti) {
        g = pf_advance(a.gtile, g, t0 + ti);
        if (g != cur_g) {  // load the group's 256 query rows
          if (cur_g >= 0) {
            tc_commit(qfree);
            if (!mbar_wait(qfree, fph, abort_flag, a.err)) break;
            fph ^= 1u;
          }
          const int row0 = __ldg(a.ginfo + g).y;
          mbar_arrive_expect(qfull, (uint32_t)QBYTES);
#pragma unroll
          for (int h = 0; h < KH; ++h)
            tma_load_2d(q_s + h * Q_HALF, &q_map, qfull, h * 64, row0 * HI);
          ctl.q_pending = (int)qph;
          if (!mbar_wait(qfull, qph, abort_flag, a.err)) break;
          ctl.q_pending = -1;
          qph ^= 1u;
          cur_g = g;
        }
        if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, abort_flag, a.err)) break;
        if (!mbar_wait(full0 + 8 * s, ph, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t stage_s = ring_s + (uint32_t)s * STAGE;
        const uint32_t d = tmem + (uint32_t)(acc * PF_N);
        const uint64_t da0 = sw128_desc(stage_s), db0 = sw128_desc(q_s);
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const int h = ks >> 2, kk = (ks & 3) * 32;
          tc_mma(d, da0 + (uint64_t)((h * A_HALF + kk) >> 4),
                 db0 + (uint64_t)((h * Q_HALF + kk) >> 4), IDESC, ks > 0 ? 1u : 0u);
        }
        tc_commit(empty0 + 8 * s);
        tc_commit(tfull0 + 8 * acc);
        ++consumed;
        if (++s == S) { s = 0; ph ^= 1u; }
        if (++acc == 2) { acc = 0; aph ^= 1u; }
      }
      ctl.consumed = consumed;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - PF_EPI0;
    const int q4 = warp & 3;             // TMEM lane quadrant this warp may access
    const int half = e >> 2;             // columns [half * 64, half * 64 + 64)
    constexpr int QH = QG / PF_EPI_PARTS;  // group rows per warp
    int acc = 0, g = g_first, cur_g = -1, row0 = 0;
    uint32_t aph = 0;
    int done = 0;
    for (int ti = 0; ti < my_tiles; ++ti) {
      g = pf_advance(a.gtile, g, t0 + ti);
      if (g != cur_g) {
        const int4 gi = __ldg(a.ginfo + g);
        row0 = gi.y + half * QH;  // first row of this warp's half
        const int nr = gi.z - half * QH;
        for (int i = lane; i < PF_EPI_COLS; i += 32) {
          const int qi = i / HI, h = i % HI;
          const float wv = qi < nr ? __ldg(a.w + (size_t)(row0 + qi) * HI + h) : 0.f;
          if constexpr (HI <= 16)  // (row 2p, row 2p + 1) pairs, head by head
            w_s[e][((qi >> 1) * HI + h) * 2 + (qi & 1)] = wv;
          else
            w_s[e][i] = wv;
        }
        for (int i = lane; i < QH; i += 32) nf_s[e][i] = i < nr ? a.row_len[row0 + i] >> 2 : 0;
        __syncwarp();
        cur_g = g;
      }
      const int j = (t0 + ti - __ldg(a.gtile + g)) * PF_M + q4 * 32 + lane;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, a.err);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(q4 * 32) << 16) +
                             (uint32_t)(acc * PF_N + half * PF_EPI_COLS);
      float part = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < PF_EPI_COLS; c0 += 32) {
        uint32_t r0[32];
        tc_ld32_nowait(taddr + c0, r0);
        tc_wait_ld();
        if (c0 + 32 == PF_EPI_COLS) {  // every column read: the accumulator may be overwritten
          tc_fence_before();
          mbar_arrive(tempty0 + 8 * acc);
        }
        if constexpr (HI <= 16) {
          // the chunk holds 32 / HI whole rows: two rows advance together in
          // one paired fp32 FMA, each in head order from 0 (the same bits
          // as one FMA per column)
          constexpr int QC = 32 / HI;
#pragma unroll
          for (int pr = 0; pr < QC / 2; ++pr) {
            const int qa = c0 / HI + 2 * pr;
            unsigned long long s2;
            asm("mov.b64 %0, {%1, %1};" : "=l"(s2) : "f"(0.f));
#pragma unroll
            for (int h = 0; h < HI; ++h) {
              const float va = fmaxf(__uint_as_float(r0[2 * pr * HI + h]), 0.f);
              const float vb = fmaxf(__uint_as_float(r0[(2 * pr + 1) * HI + h]), 0.f);
              const float2 w2 =
                  *reinterpret_cast<const float2 *>(&w_s[e][((qa >> 1) * HI + h) * 2]);
              unsigned long long v2, ww;
              asm("mov.b64 %0, {%1, %2};" : "=l"(v2) : "f"(va), "f"(vb));
              asm("mov.b64 %0, {%1, %2};" : "=l"(ww) : "f"(w2.x), "f"(w2.y));
              asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(s2) : "l"(ww), "l"(v2));
            }
            float pa, pb;
            asm("mov.b64 {%0, %1}, %2;" : "=f"(pa), "=f"(pb) : "l"(s2));
            if (j < nf_s[e][qa]) a.scores[(size_t)(row0 + qa) * a.ld + j] = pa;
            if (j < nf_s[e][qa + 1]) a.scores[(size_t)(row0 + qa + 1) * a.ld + j] = pb;
          }
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u) {
            const int col = c0 + u;
            const float v = __uint_as_float(r0[u]);
            part = fmaf(w_s[e][col], fmaxf(v, 0.f), part);
            if (col % HI == HI - 1) {
              const int qi = col / HI;
              if (j < nf_s[e][qi]) a.scores[(size_t)(row0 + qi) * a.ld + j] = part;
              part = 0.f;
            }
          }
        }
      }
      ++done;
      if (++acc == 2) { acc = 0; aph ^= 1u; }
    }
    if (threadIdx.x == 32 * PF_EPI0) ctl.done = done;
  }

  __syncthreads();
  pdl_trigger();
  if (ctl.abort_flag) {
    // drain: stages whose copies were issued but never consumed, MMAs whose
    // accumulators were never read, the last query-row load
    if (threadIdx.x == 0) {
      for (int i = ctl.consumed; i < my_tiles; ++i)
        if (i < ctl.issued[i % PF_PROD_WARPS])
          mbar_wait(full0 + 8 * (i % S), (uint32_t)((i / S) & 1), abort_flag, a.err,
                    TC_DRAIN_LIMIT, false);
    }
    if (threadIdx.x == 32 * PF_MMA_WARP) {
      for (int i = ctl.done; i < ctl.consumed; ++i)
        mbar_wait(tfull0 + 8 * (i & 1), (uint32_t)((i >> 1) & 1), abort_flag, a.err,
                  TC_DRAIN_LIMIT, false);
      if (ctl.q_pending >= 0)
        mbar_wait(qfull, (uint32_t)ctl.q_pending, abort_flag, a.err, TC_DRAIN_LIMIT, false);
    }
    __syncthreads();
  }
  if (warp == PF_MMA_WARP) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(2 * PF_N)
                 : "memory");
  }
}

template <int DI, int HI>
cudaError_t launch_pf_t(const qsa_cache &c, PfArgs a, cudaStream_t st) {
  cudaError_t e;
  EncodeTiledFn enc = encode_tiled_fn(&e);
  if (e != cudaSuccess) return e;
  if (enc == nullptr) return cudaErrorNotSupported;
  CUtensorMap side_map, q_map;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)DI, (cuuint64_t)a.rpp, (cuuint64_t)c.num_pages};
    const cuuint64_t strides[2] = {(cuuint64_t)DI * 2, (cuuint64_t)a.rpp * DI * 2};
    const cuuint32_t box[3] = {64u, (cuuint32_t)a.box, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    if (enc(&side_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, c.side_pool, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // q_idx as [Nq * Hi rows][DI]; a group's 256 rows in one box per K half
    // (rows past the end read as zeros)
    const cuuint64_t dims[2] = {(cuuint64_t)DI, (cuuint64_t)a.Nq * HI};
    const cuuint64_t strides[1] = {(cuuint64_t)DI * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)PF_N};
    const cuuint32_t estr[2] = {1u, 1u};
    if (enc(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(a.q_idx),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  constexpr size_t STAGE = (size_t)(DI / 64) * PF_M * 128;
  constexpr size_t QBYTES = (size_t)(DI / 64) * PF_N * 128;
  const size_t limit = 200 * 1024;  // dynamic part; the static part holds the epilogue tables
  a.stages = (int)std::min<size_t>(PF_MAX_STAGES, (limit - 1024 - QBYTES) / STAGE);
  if (a.stages < 4) return cudaErrorInvalidValue;  // fewer would let a producer run two laps ahead
  const size_t smem = 1024 + QBYTES + (size_t)a.stages * STAGE;

  a.QG = PF_N / HI;
  e = launch_pdl(prefill_plan_kernel, 1, PL_THREADS, 0, st, a);
  if (e != cudaSuccess) return e;
  e = launch_pdl(prefill_partial_kernel<DI>, (a.Nq + 7) / 8, 256, 0, st, a);
  if (e != cudaSuccess) return e;
  auto kern = prefill_score_kernel<DI, HI>;
  e = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, device_sm_count(), PF_THREADS, smem, st, side_map, q_map, a);
}

}  // namespace

int prefill_group_rows(const qsa_dims &d) { return PF_N / d.Hi; }

bool prefill_supported(const qsa_dims &d) {
  return index_score_supported(d) && (d.Hi == 4 || d.Hi == 8 || d.Hi == 16 || d.Hi == 32);
}

size_t prefill_plan_ws_bytes(const qsa_dims &d, int S, int Nq) {
  const size_t QG = (size_t)(PF_N / d.Hi);
  const size_t gmax = (size_t)S + ((size_t)Nq + QG - 1) / QG;
  size_t bytes = 16;                                // header
  bytes += ((size_t)Nq * 4 + 15) / 16 * 16;         // row_seq
  bytes += ((gmax + 1) * 4 + 15) / 16 * 16;         // tile prefix
  bytes += gmax * 16;                               // group list
  return bytes;
}

cudaError_t launch_prefill_index_score(const qsa_dims &d, const qsa_cache &c, int S,
                                       const int32_t *seq_lens, const int32_t *row_start, int Nq,
                                       const void *q_idx, const float *w, float *scores, int ld,
                                       int32_t *row_len, void *ws, unsigned *err,
                                       cudaStream_t st) {
  if (S == 0 || Nq == 0) return cudaSuccess;
  PfArgs a;
  a.kidx_pool = static_cast<const __nv_bfloat16 *>(c.kidx_pool);
  a.q_idx = static_cast<const __nv_bfloat16 *>(q_idx);
  a.w = w;
  a.block_table = c.block_table;
  a.seq_lens = seq_lens;
  a.row_start = row_start;
  a.row_len = row_len;
  const int QG = PF_N / d.Hi;
  a.Gmax = S + (Nq + QG - 1) / QG;
  unsigned char *p = static_cast<unsigned char *>(ws);
  a.hdr = reinterpret_cast<int *>(p);
  p += 16;
  a.row_seq = reinterpret_cast<int32_t *>(p);
  p += ((size_t)Nq * 4 + 15) / 16 * 16;
  a.gtile = reinterpret_cast<int *>(p);
  p += ((size_t)(a.Gmax + 1) * 4 + 15) / 16 * 16;
  a.ginfo = reinterpret_cast<int4 *>(p);
  a.scores = scores;
  a.S = S;
  a.Nq = Nq;
  a.QG = QG;
  a.ld = ld;
  a.P = d.P;
  a.rpp = d.P / 4;
  a.box = std::min(a.rpp, PF_M);
  a.max_pages = c.max_pages_per_seq;
  a.num_pages = c.num_pages;
  a.Hi = d.Hi;
  a.stages = 0;
  a.err = err;
  if (d.di == 128) {
    switch (d.Hi) {
      case 4: return launch_pf_t<128, 4>(c, a, st);
      case 8: return launch_pf_t<128, 8>(c, a, st);
      case 16: return launch_pf_t<128, 16>(c, a, st);
      default: return launch_pf_t<128, 32>(c, a, st);
    }
  }
  switch (d.Hi) {
    case 4: return launch_pf_t<64, 4>(c, a, st);
    case 8: return launch_pf_t<64, 8>(c, a, st);
    case 16: return launch_pf_t<64, 16>(c, a, st);
    default: return launch_pf_t<64, 32>(c, a, st);
  }
}

}  // namespace qsa
