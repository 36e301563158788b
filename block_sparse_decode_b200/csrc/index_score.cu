// qsa_index_score on 5th-generation tensor cores: side-cache tiles moved by
// TMA into shared memory, tcgen05.mma into TMEM, and an epilogue that reads
// the accumulators back with tcgen05.ld.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": the indexer scores the
// micro-blocks. Score of block b: s_b = sum_h w_h * max(0, q_idx_h . kc_b)
// (this library's reading; the page prints no formula).
//
// Why this shape: the contraction is [blocks x di] . [di x Hi], 8 MAC per
// side-cache byte at di = 128, Hi = 16; at HBM speed that is ~50 TMAC/s,
// beyond fp32 CUDA cores. One thread issues the MMAs (M = 128 blocks, N = 16
// or 32 heads, K = di in steps of 16) into TMEM, so the tensor work costs a
// few instructions per tile. The side cache is paged (P/4 rows per page): a
// 128-row tile is a gather of 128/(P/4) page pieces. Each piece is one TMA
// box per 128-byte K half, landing in the 128-byte-swizzled K-major layout
// the MMA descriptors expect; the data never passes through the load/store
// pipe, so the producer's own bookkeeping never queues behind it.
//
// Page ids: under full HBM load a block-table read waits several
// microseconds behind the in-flight tile data, so per-tile lookups would
// stall the producer. Instead the CTA copies the page ids of its tiles into
// a shared table first (4-byte cp.async by every warp, before any tile
// traffic; two halves, the second refilled hundreds of tiles ahead when a
// CTA has that many tiles), and the producer reads the table.
//
// CTA = 8 warps, persistent over the flattened (sequence, 128-block tile) list:
//   warps 0-2  producers (tiles round-robin): expect-tx, TMA boxes of the
//              tile's page pieces and, when the stage holds another
//              sequence's, of the indexer query, into a ring of stages
//   warp 3     TMEM owner; lane 0 issues the MMAs into one of two TMEM
//              accumulators and commits to the stage's empty barrier and the
//              accumulator's full barrier
//   warps 4-7  epilogue: tcgen05.ld of 32 rows x N columns each, ReLU, head
//              weights, one coalesced fp32 store per block; the trailing
//              partial block (key built from its L mod 4 indexer keys) is
//              scored on CUDA cores by the warp that owns its row.
// Every mbarrier wait is bounded: on timeout the kernel sets the TIMEOUT bit,
// stops all roles, drains what it issued (bounded) and frees TMEM.
//
// Page pieces: a tile's rows are cut into pieces of gcd(P/4, 128) rows, so a
// piece never spans two pages and pieces tile the 128 rows exactly; with P a
// multiple of 32 a piece is a multiple of 8 rows and every box starts on a
// 1 KiB swizzle atom. Supported: P a multiple of 32 in [32, 1024], di in
// {64, 128}, Hi <= 32; other page sizes (P a multiple of 4) are scored by the
// warp-level MMA kernel of index_score_warp.cu.
// Roofline: HBM-bound; algorithmic bytes = nb * di * 2 per sequence.
#include <cuda.h>

#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"
#include "umma_desc.h"

namespace qsa {
namespace {

constexpr int TC_M = 128;  // blocks per tile (MMA M)
constexpr int TC_MAX_STAGES = 8;
constexpr int TC_EPI_WARPS = 4;
constexpr int TC_PROD_WARPS = 3;                          // producers take tiles round-robin
constexpr int TC_MMA_WARP = TC_PROD_WARPS;                // warp 3
constexpr int TC_EPI0 = TC_PROD_WARPS + 1;                // first epilogue warp
constexpr int TC_THREADS = 32 * (TC_PROD_WARPS + 1 + TC_EPI_WARPS);
constexpr int TBL = 2048;  // shared page-table entries (two halves)
__device__ const int32_t k_no_page = -1;

struct TcArgs {
  const __nv_bfloat16 *kidx_pool, *q_idx;
  const float *w;
  const int32_t *block_table, *seq_lens;
  float *scores;
  int B, ld, P, rpp, max_pages, num_pages, Hi, stages;
  int box;  // tile rows per page piece: gcd(P/4, 128)
  int ept;  // page pieces per tile: 128 / box
  int tpc;  // tiles per half of the shared page table
  uint32_t spin_limit;  // try_wait rounds before a role gives up
  int stall;            // failure injection: producers issue nothing (debug_stall_score())
  unsigned *err;
};

struct TcCtrl {
  uint64_t full[TC_MAX_STAGES];
  uint64_t empty[TC_MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t tbl0;    // first page-table half filled (every CTA thread)
  uint64_t tbl[2];  // later refills of a half (producer warp)
  uint32_t tmem_base;
  int abort_flag;
  int issued[TC_PROD_WARPS];  // per producer warp: first tile index it did not issue
  int qseq[TC_MAX_STAGES];    // sequence whose indexer query a stage holds
  int consumed;  // tiles the MMA warp consumed
  int done;      // tiles the epilogue finished
};

__device__ __forceinline__ int tc_find_seq(const int *prefix, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Score of the trailing partial block of sequence b (whole warp; every lane
// returns it).
template <int DI, int N>
__device__ float partial_block_score(const TcArgs &a, int b, int L, bool *ok_out) {
  return partial_block_score_row<DI, N>(a.kidx_pool, a.P, a.block_table + (size_t)b * a.max_pages,
                                     a.max_pages, a.num_pages, L, a.q_idx + (size_t)b * a.Hi * DI,
                                     a.w + (size_t)b * a.Hi, a.Hi, a.err, ok_out);
}

template <int DI, int N>
__global__ void __launch_bounds__(TC_THREADS, 1)
    index_score_tc_kernel(const __grid_constant__ CUtensorMap side_map,
                          const __grid_constant__ CUtensorMap q_map, TcArgs a) {
  constexpr int KH = DI / 64;         // 128-byte K halves
  constexpr int A_HALF = TC_M * 128;  // bytes of one A half (128 rows)
  constexpr int B_HALF = N * 128;     // bytes of one B half (N rows)
  constexpr int STAGE = KH * (A_HALF + B_HALF);
  constexpr int KSTEPS = DI / 16;
  constexpr uint32_t IDESC = f16_idesc(TC_M, N);

  extern __shared__ unsigned char smem_raw[];
  __shared__ TcCtrl ctl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;

  // dynamic smem: [pad to 1024][stages][page table TBL][prefix B+1][lens B]
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  const uint32_t ring_s = raw_s + pad;
  int *prefix = reinterpret_cast<int *>(smem_raw + pad + (size_t)S * STAGE + TBL * 4);
  int *lens = prefix + (a.B + 1);

  // the CTAs pull the block-table rows of the batch into L2 together, so the
  // page-table fill below (which first needs the tile prefix) hits L2
  {
    const char *bt = reinterpret_cast<const char *>(a.block_table);
    const long long lines = ((long long)a.B * a.max_pages * 4 + 127) >> 7;
    for (long long i = blockIdx.x + (long long)gridDim.x * threadIdx.x; i < lines;
         i += (long long)gridDim.x * blockDim.x)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(bt + (i << 7)));
  }

  // ---- per-CTA tile prefix over sequences
  __shared__ int carry;
  __shared__ int wsum[TC_THREADS / 32];
  if (threadIdx.x == 0) {
    carry = 0;
    prefix[0] = 0;
    ctl.abort_flag = 0;
    ctl.consumed = ctl.done = 0;
    for (int w = 0; w < TC_PROD_WARPS; ++w) ctl.issued[w] = w;
    for (int i = 0; i < TC_MAX_STAGES; ++i) ctl.qseq[i] = -1;
  }
  __syncthreads();
  for (int base = 0; base < a.B; base += TC_THREADS) {
    const int b = base + threadIdx.x;
    int n = 0;
    if (b < a.B) {
      int L = a.seq_lens[b];
      int nb = L < 0 ? 0 : (L + 3) >> 2;
      if (L < 0 || nb > a.ld) {
        if (blockIdx.x == 0) raise_err(a.err, ERR_LEN);
        nb = 0;
        L = 0;
      }
      lens[b] = L;
      n = (nb + TC_M - 1) / TC_M;
    }
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int off = carry;
    for (int i = 0; i < warp; ++i) off += wsum[i];
    if (b < a.B) prefix[b + 1] = off + x;
    __syncthreads();
    if (threadIdx.x == TC_THREADS - 1) carry = off + x;
    __syncthreads();
  }
  const int total = prefix[a.B];
  const int my_tiles =
      total > (int)blockIdx.x ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  // Shared page table: half h holds, for tpc consecutive tiles of this CTA,
  // the page ids of the tile's ept page pieces (-1: the piece holds no
  // complete block). Warps fill tiles round-robin with 4-byte cp.async; every
  // filling thread arrives on the half's barrier when its copies land.
  int *table = reinterpret_cast<int *>(smem_raw + pad + (size_t)S * STAGE);
  auto tile_start = [&](int ti, int &b, int &j0) {
    const int t = blockIdx.x + ti * gridDim.x;
    b = tc_find_seq(prefix, a.B, t);
    j0 = (t - prefix[b]) * TC_M;
  };
  auto fill_table = [&](int chunk, int wfirst, int nwarps) {
    int *half = table + (chunk & 1) * (TBL / 2);
    const int ntiles = min(a.tpc, my_tiles - chunk * a.tpc);
    for (int til = warp - wfirst; til < ntiles; til += nwarps) {
      int b, j0;
      tile_start(chunk * a.tpc + til, b, j0);
      const int nfull = lens[b] >> 2;
      for (int k = lane; k < a.ept; k += 32) {
        const int col = (j0 + k * a.box) / a.rpp;  // a piece never spans two pages
        const bool live = (j0 + k * a.box) < nfull && col < a.max_pages;
        if ((j0 + k * a.box) < nfull && col >= a.max_pages) raise_err(a.err, ERR_BT);
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                         smem_u32(half + til * a.ept + k)),
                     "l"(live ? a.block_table + (size_t)b * a.max_pages + col : &k_no_page)
                     : "memory");
      }
    }
  };
  const uint32_t full0 = smem_u32(&ctl.full[0]), empty0 = smem_u32(&ctl.empty[0]);
  const uint32_t tfull0 = smem_u32(&ctl.tfull[0]), tempty0 = smem_u32(&ctl.tempty[0]);
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull0 + 8 * i, 1);
      mbar_init(tempty0 + 8 * i, TC_EPI_WARPS * 32);
      mbar_init(smem_u32(&ctl.tbl[i]), 32);
    }
    mbar_init(smem_u32(&ctl.tbl0), TC_THREADS);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();  // barriers initialised before the first table copy arrives
  fill_table(0, 0, TC_THREADS / 32);
  cp_async_arrive(smem_u32(&ctl.tbl0));
  if (warp == TC_MMA_WARP) {  // TMEM: two accumulators of N fp32 columns (64 allocated)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&ctl.tmem_base)),
                 "r"(64)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // everything above reads inputs only; the side cache and the per-token
  // indexer keys come from the append kernel before this one
  pdl_wait();
  const uint32_t tmem = ctl.tmem_base;
  volatile int *abort_flag = &ctl.abort_flag;

  if (warp < TC_PROD_WARPS) {
    // ------------------------------------------------------------ producers
    // Warp w issues tiles w, w + 3, ...; stage and phase follow from the tile
    // index, so the MMA warp consumes tiles in order. One warp's bookkeeping
    // overlaps the other's TMA issue.
    int last_chunk = -1, refilled = 0;
    int ti = warp;
    for (; ti < my_tiles && !a.stall; ti += TC_PROD_WARPS) {
      const int chunk = ti / a.tpc, tl = ti - chunk * a.tpc;
      if (chunk != last_chunk) {  // this half of the page table must have landed
        bool ok = true;
        if (lane == 0)
          ok = chunk == 0 ? mbar_wait(smem_u32(&ctl.tbl0), 0u, abort_flag, a.err, a.spin_limit)
                          : mbar_wait(smem_u32(&ctl.tbl[chunk & 1]),
                                      (uint32_t)(((chunk - 1) >> 1) & 1), abort_flag, a.err,
                                      a.spin_limit);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        __syncwarp();
        last_chunk = chunk;
      }
      // Refill the other half for the next chunk once every producer is past
      // the previous one: a producer at tile ti has seen the stage of tile
      // ti - S consumed, and the MMA consumes in order, so every other
      // producer has issued beyond ti - S - TC_PROD_WARPS.
      if (warp == 0 && refilled <= chunk && tl >= S + TC_PROD_WARPS &&
          (chunk + 1) * a.tpc < my_tiles) {
        fill_table(chunk + 1, 0, 1);
        cp_async_arrive(smem_u32(&ctl.tbl[(chunk + 1) & 1]));
        refilled = chunk + 1;
      }
      int b, j0;
      tile_start(ti, b, j0);
      const int rows = max(0, min(TC_M, (lens[b] >> 2) - j0));  // complete blocks
      const int npiece = (rows + a.box - 1) / a.box;
      int page = -1;
      if (lane < npiece) {
        page = table[(chunk & 1) * (TBL / 2) + tl * a.ept + lane];
        if (page < 0 || page >= a.num_pages) {
          if (page != -1) raise_err(a.err, ERR_PAGE);
          page = -1;
        }
      }
      const int s = ti % S;
      const uint32_t ph = (uint32_t)((ti / S) & 1);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, a.err, a.spin_limit);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      __syncwarp();
      const unsigned live = __ballot_sync(0xffffffffu, page >= 0);
      const bool new_q = ctl.qseq[s] != b;  // the stage's query buffer holds another sequence
      const uint32_t stage_s = ring_s + (uint32_t)s * STAGE;
      const uint32_t bar = full0 + 8 * s;
      if (lane == 0) {
        mbar_arrive_expect(bar, (uint32_t)(__popc(live) * a.box * 128 * KH + (new_q ? B_HALF * KH : 0)));
        ctl.qseq[s] = b;
      }
      __syncwarp();
      if (page >= 0) {
        const int rip = (j0 + lane * a.box) % a.rpp;  // row in page (P > 512 only)
#pragma unroll
        for (int h = 0; h < KH; ++h)
          tma_load_3d(stage_s + h * A_HALF + lane * a.box * 128, &side_map, bar, h * 64, rip, page);
      }
      if (new_q && lane < KH)
        tma_load_2d(stage_s + KH * A_HALF + lane * B_HALF, &q_map, bar, lane * 64, b * a.Hi);
    }
    if (lane == 0) ctl.issued[warp] = ti;
  } else if (warp == TC_MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      int consumed = 0;
      for (int ti = 0; ti < my_tiles; ++ti) {
        if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, abort_flag, a.err, a.spin_limit)) break;
        if (!mbar_wait(full0 + 8 * s, ph, abort_flag, a.err, a.spin_limit)) break;
        tc_fence_after();
        const uint32_t stage_s = ring_s + (uint32_t)s * STAGE;
        const uint32_t d = tmem + (uint32_t)(acc * 32);
        // descriptors of the stage base; each k-step adds its byte offset / 16 to
        // the start-address field (no carry: shared addresses stay below 256 KiB)
        const uint64_t da0 = sw128_desc(stage_s), db0 = sw128_desc(stage_s + KH * A_HALF);
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          const int h = ks >> 2, kk = (ks & 3) * 32;
          tc_mma(d, da0 + (uint64_t)((h * A_HALF + kk) >> 4),
                 db0 + (uint64_t)((h * B_HALF + kk) >> 4), IDESC, ks > 0 ? 1u : 0u);
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
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    int acc = 0;
    uint32_t aph = 0;
    int done = 0;
    for (int ti = 0; ti < my_tiles; ++ti) {
      const int t = blockIdx.x + ti * gridDim.x;
      const int b = tc_find_seq(prefix, a.B, t);
      const int j0 = (t - prefix[b]) * TC_M;
      const int L = lens[b];
      const int nfull = L >> 2, nb = (L + 3) >> 2;
      float wv[N];  // head weights, loaded before the wait so their latency hides
#pragma unroll
      for (int h = 0; h < N; ++h) wv[h] = h < a.Hi ? __ldg(a.w + (size_t)b * a.Hi + h) : 0.f;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, a.err, a.spin_limit);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      __syncwarp();
      tc_fence_after();
      float v[16];
      float score = 0.f;
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 32);
      tc_ld16(taddr, v);
#pragma unroll
      for (int h = 0; h < 16; ++h) score = fmaf(wv[h], fmaxf(v[h], 0.f), score);
      if (N == 32) {
        tc_ld16(taddr + 16, v);
#pragma unroll
        for (int h = 0; h < 16; ++h) score = fmaf(wv[(16 + h) % N], fmaxf(v[h], 0.f), score);
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * acc);  // the accumulator may be overwritten
      const int j = j0 + q * 32 + lane;
      if (j < nfull) a.scores[(size_t)b * a.ld + j] = score;
      if (nfull < nb && nfull >= j0 + q * 32 && nfull < j0 + q * 32 + 32) {
        bool ok;
        const float sp = partial_block_score<DI, N>(a, b, L, &ok);
        if (lane == 0 && ok) a.scores[(size_t)b * a.ld + nfull] = sp;
      }
      ++done;
      if (++acc == 2) { acc = 0; aph ^= 1u; }
    }
    if (threadIdx.x == 32 * TC_EPI0) ctl.done = done;
  }

  asm volatile("cp.async.wait_all;" ::: "memory");  // page-table copies, even after an abort
  __syncthreads();
  pdl_trigger();
  if (ctl.abort_flag) {
    // drain: stages whose copies were issued but never consumed, MMAs whose
    // accumulators were never read
    if (threadIdx.x == 0) {
      for (int i = ctl.consumed; i < my_tiles; ++i)
        if (i < ctl.issued[i % TC_PROD_WARPS])
          mbar_wait(full0 + 8 * (i % S), (uint32_t)((i / S) & 1), abort_flag, a.err,
                    TC_DRAIN_LIMIT, false);
    }
    if (threadIdx.x == 32 * TC_MMA_WARP) {
      for (int i = ctl.done; i < ctl.consumed; ++i)
        mbar_wait(tfull0 + 8 * (i & 1), (uint32_t)((i >> 1) & 1), abort_flag, a.err,
                  TC_DRAIN_LIMIT, false);
    }
    __syncthreads();
  }
  if (warp == TC_MMA_WARP) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(64)
                 : "memory");
  }
}

}  // namespace

bool debug_stall_score() {
  const char *v = std::getenv("QSA_DEBUG_STALL_SCORE");
  return v != nullptr && v[0] == '1' && v[1] == '\0';
}

EncodeTiledFn encode_tiled_fn(cudaError_t *status) {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  static cudaError_t st = cudaSuccess;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    st = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (st == cudaSuccess && q != cudaDriverEntryPointSuccess) st = cudaErrorNotSupported;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  *status = st;
  return fn;
}

namespace {

template <int DI, int N>
cudaError_t launch_tc_t(const qsa_cache &c, TcArgs a, cudaStream_t st) {
  cudaError_t e;
  EncodeTiledFn enc = encode_tiled_fn(&e);
  if (e != cudaSuccess) return e;
  if (enc == nullptr) return cudaErrorNotSupported;
  // side pool viewed as [num_pages][rpp rows][DI]; q_idx as [B*Hi][DI]
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
    const cuuint64_t dims[2] = {(cuuint64_t)DI, (cuuint64_t)a.B * a.Hi};
    const cuuint64_t strides[1] = {(cuuint64_t)DI * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)N};
    const cuuint32_t estr[2] = {1u, 1u};
    if (enc(&q_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(a.q_idx),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  constexpr int KH = DI / 64;
  constexpr size_t STAGE = (size_t)KH * (TC_M * 128 + N * 128);
  const size_t meta = (size_t)TBL * 4 + (size_t)(2 * a.B + 1) * 4;
  const size_t limit = 227 * 1024;
  if (1024 + 2 * STAGE + meta > limit) return cudaErrorInvalidValue;
  // a multiple of the producer count keeps each stage with one producer warp
  a.stages = (int)std::min<size_t>(6, (limit - 1024 - meta) / STAGE);
  a.stages -= a.stages % TC_PROD_WARPS;
  if (a.stages < TC_PROD_WARPS || a.tpc < a.stages + TC_PROD_WARPS + 1)
    return cudaErrorInvalidValue;
  const size_t smem = 1024 + (size_t)a.stages * STAGE + meta;
  auto kern = index_score_tc_kernel<DI, N>;
  e = ensure_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
  if (e != cudaSuccess) return e;
  const long long tiles_bound = (long long)a.B * ((a.ld + TC_M - 1) / TC_M);
  const int grid =
      (int)std::max<long long>(1, std::min<long long>(device_sm_count(), tiles_bound));
  return launch_pdl(kern, grid, TC_THREADS, smem, st, side_map, q_map, a);
}

}  // namespace

int piece_rows(int rpp) {
  int x = rpp, y = TC_M;  // gcd(rows per page, rows per tile)
  while (y != 0) {
    const int t = x % y;
    x = y;
    y = t;
  }
  return x;
}

bool index_score_supported(const qsa_dims &d) {
  // a page piece of gcd(P/4, 128) rows must start on a 1 KiB swizzle atom
  const bool pages = d.P >= 32 && d.P <= 1024 && d.P % 32 == 0;
  return pages && (d.di == 64 || d.di == 128) && d.Hi <= 32;
}

cudaError_t launch_index_score(const qsa_dims &d, const qsa_cache &c, int B,
                               const int32_t *seq_lens, const void *q_idx, const float *w,
                               float *scores, int ld, unsigned *err, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  if (!index_score_supported(d))  // page pieces off the swizzle atoms: warp-level MMA path
    return launch_index_score_warp(d, c, B, seq_lens, q_idx, w, scores, ld, err, st);
  TcArgs a;
  a.kidx_pool = static_cast<const __nv_bfloat16 *>(c.kidx_pool);
  a.q_idx = static_cast<const __nv_bfloat16 *>(q_idx);
  a.w = w;
  a.block_table = c.block_table;
  a.seq_lens = seq_lens;
  a.scores = scores;
  a.B = B;
  a.ld = ld;
  a.P = d.P;
  a.rpp = d.P / 4;
  a.box = piece_rows(a.rpp);
  a.ept = TC_M / a.box;
  a.tpc = (TBL / 2) / a.ept;
  a.max_pages = c.max_pages_per_seq;
  a.num_pages = c.num_pages;
  a.Hi = d.Hi;
  a.stages = 2;
  a.stall = debug_stall_score() ? 1 : 0;
  a.spin_limit = a.stall ? TC_STALL_LIMIT : TC_SPIN_LIMIT;
  a.err = err;
  if (d.di == 128)
    return d.Hi <= 16 ? launch_tc_t<128, 16>(c, a, st) : launch_tc_t<128, 32>(c, a, st);
  return d.Hi <= 16 ? launch_tc_t<64, 16>(c, a, st) : launch_tc_t<64, 32>(c, a, st);
}

}  // namespace qsa
