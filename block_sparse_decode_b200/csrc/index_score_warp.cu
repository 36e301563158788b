// qsa_index_score for page sizes the TMA page-piece gather cannot address
// (P a multiple of 4 but not of 32: a piece of a page would start inside a
// 1 KiB swizzle atom of the tensor-core tile).
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": the indexer scores the
// micro-blocks, s_b = sum_h w_h * max(0, q_idx_h . kc_b) (this library's
// reading). Same scores as the tcgen05 kernel within fp32 rounding (the dot
// products accumulate in a different order).
//
// Design: each warp scores 16 blocks at a time with warp-level tensor-core
// MMAs (mma.sync m16n8k16: the 16 rows are blocks, the 8 columns indexer
// heads, K = di). The 16 side-cache rows of a tile are gathered row by row
// (any page size: a row is one block's compressed key, di * 2 bytes) with
// 16-byte cp.async into XOR-swizzled shared memory, two tiles in flight per
// warp; the query fragments stay in registers for the warp's whole range.
// The trailing partial block is scored on CUDA cores by the warp whose tile
// holds it, with the tcgen05 kernel's code. Roofline: HBM-bound, nb * di * 2
// bytes per sequence; this path trades some of it for generality.
#include "common.cuh"
#include "launch.h"
#include "tc_util.cuh"

namespace qsa {
namespace {

constexpr int SW_WARPS = 4;
constexpr int SW_ROWS = 16;                 // blocks per warp tile (MMA M)
constexpr int SW_TILES_PER_WARP = 8;        // consecutive tiles a warp walks
constexpr int SW_BLOCKS_PER_CTA = SW_WARPS * SW_TILES_PER_WARP * SW_ROWS;  // 512
constexpr int SW_STAGES = 2;

struct SwArgs {
  const __nv_bfloat16 *side_pool, *kidx_pool, *q_idx;
  const float *w;
  const int32_t *block_table, *seq_lens;
  float *scores;
  int B, ld, P, rpp, max_pages, num_pages, Hi;
  unsigned *err;
};

template <int DI, int NT>  // NT: 8-head column tiles (Hi <= 8 * NT)
__global__ void __launch_bounds__(SW_WARPS * 32) index_score_warp_kernel(SwArgs a) {
  constexpr int ROWB = DI * 2;                 // bytes per side-cache row
  constexpr int CHUNKS = ROWB / 16;            // 16-byte chunks per row
  constexpr int TILEB = SW_ROWS * ROWB;        // bytes per tile
  constexpr int KSTEPS = DI / 16;
  __shared__ __align__(1024) unsigned char ring[SW_WARPS][SW_STAGES][TILEB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int gq = lane >> 2, tq = lane & 3;

  int L = a.seq_lens[b];
  int nb = L < 0 ? 0 : (L + 3) >> 2;
  if (L < 0 || nb > a.ld) {  // the sequence is skipped (no score written)
    if (threadIdx.x == 0 && blockIdx.x == 0) raise_err(a.err, ERR_LEN);
    L = nb = 0;
  }
  const int nfull = L >> 2;
  const int32_t *bt = a.block_table + (size_t)b * a.max_pages;
  // query fragments (B operand, k = dims, n = heads): head nt*8 + gq
  uint32_t qf[NT][KSTEPS][2];
  float wv[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int h = nt * 8 + gq;
    const bool hv = h < a.Hi;
    const uint32_t *qrow =
        reinterpret_cast<const uint32_t *>(a.q_idx + ((size_t)b * a.Hi + (hv ? h : 0)) * DI);
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      qf[nt][ks][0] = hv ? qrow[ks * 8 + tq] : 0u;
      qf[nt][ks][1] = hv ? qrow[ks * 8 + 4 + tq] : 0u;
    }
    // weights of the heads this lane's accumulator columns hold: 2tq, 2tq+1
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int hc = nt * 8 + 2 * tq + c;
      wv[nt][c] = hc < a.Hi ? a.w[(size_t)b * a.Hi + hc] : 0.f;
    }
  }
  pdl_wait();  // the side cache comes from the append kernel before this one

  const int j_warp = blockIdx.x * SW_BLOCKS_PER_CTA + warp * SW_TILES_PER_WARP * SW_ROWS;
  const uint32_t ring_s = smem_u32(&ring[warp][0][0]);
  // one tile: rows j0 .. j0+15; lane copies chunks (row, chunk) = (i / CHUNKS, i % CHUNKS)
  auto issue = [&](int t) {
    if (t < SW_TILES_PER_WARP) {
      const int j0 = j_warp + t * SW_ROWS;
      const uint32_t dst = ring_s + (t % SW_STAGES) * TILEB;
#pragma unroll
      for (int i0 = 0; i0 < SW_ROWS * CHUNKS; i0 += 32) {
        const int i = i0 + lane;
        const int row = i / CHUNKS, ch = i % CHUNKS;
        const int j = j0 + row;
        bool ok = j < nfull;
        const __nv_bfloat16 *src = a.side_pool;
        if (ok) {
          const int col = (4 * j) / a.P;
          const int page = col < a.max_pages ? __ldg(bt + col) : -1;
          if (page < 0 || page >= a.num_pages) {
            if (ch == 0) raise_err(a.err, col < a.max_pages ? ERR_PAGE : ERR_BT);
            ok = false;
          } else {
            src = a.side_pool + ((size_t)page * a.rpp + (j - col * a.rpp)) * DI + ch * 8;
          }
        }
        cp_async16(dst + swz(row, ch, ROWB), src, ok ? 16 : 0);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int t = 0; t < SW_STAGES - 1; ++t) issue(t);
  const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int akc = lane >> 4;
  for (int t = 0; t < SW_TILES_PER_WARP; ++t) {
    const int j0 = j_warp + t * SW_ROWS;
    if (j0 >= nb) break;  // warp-uniform
    __syncwarp();
    issue(t + SW_STAGES - 1);
    cp_async_wait<SW_STAGES - 1>();
    __syncwarp();
    const uint32_t base = ring_s + (t % SW_STAGES) * TILEB;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(base + swz(arow, 2 * ks + akc, ROWB), a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        mma_bf16_16816(acc[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
    }
    // acc[nt][0..1]: block gq, heads nt*8 + 2tq (+1); acc[nt][2..3]: block gq + 8
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s0 = fmaf(wv[nt][0], fmaxf(acc[nt][0], 0.f), s0);
      s0 = fmaf(wv[nt][1], fmaxf(acc[nt][1], 0.f), s0);
      s1 = fmaf(wv[nt][0], fmaxf(acc[nt][2], 0.f), s1);
      s1 = fmaf(wv[nt][1], fmaxf(acc[nt][3], 0.f), s1);
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, o);
      s1 += __shfl_xor_sync(0xffffffffu, s1, o);
    }
    if (tq == 0) {
      if (j0 + gq < nfull) a.scores[(size_t)b * a.ld + j0 + gq] = s0;
      if (j0 + gq + 8 < nfull) a.scores[(size_t)b * a.ld + j0 + gq + 8] = s1;
    }
    if (nfull < nb && nfull >= j0 && nfull < j0 + SW_ROWS) {  // the trailing partial block
      bool ok;
      const float sp = partial_block_score_row<DI, NT * 8>(a.kidx_pool, a.P, bt, a.max_pages, a.num_pages,
                                                   L, a.q_idx + (size_t)b * a.Hi * DI,
                                                   a.w + (size_t)b * a.Hi, a.Hi, a.err, &ok);
      if (lane == 0 && ok) a.scores[(size_t)b * a.ld + nfull] = sp;
    }
  }
  cp_async_wait<0>();
  pdl_trigger();
}

template <int DI, int NT>
cudaError_t launch_t(const SwArgs &a, cudaStream_t st) {
  const int nbmax = a.ld;  // every block index a sequence may have
  const dim3 grid((nbmax + SW_BLOCKS_PER_CTA - 1) / SW_BLOCKS_PER_CTA, a.B);
  return launch_pdl(index_score_warp_kernel<DI, NT>, grid, SW_WARPS * 32, 0, st, a);
}

}  // namespace

cudaError_t launch_index_score_warp(const qsa_dims &d, const qsa_cache &c, int B,
                                    const int32_t *seq_lens, const void *q_idx, const float *w,
                                    float *scores, int ld, unsigned *err, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  SwArgs a;
  a.side_pool = static_cast<const __nv_bfloat16 *>(c.side_pool);
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
  a.max_pages = c.max_pages_per_seq;
  a.num_pages = c.num_pages;
  a.Hi = d.Hi;
  a.err = err;
  const int nt = (d.Hi + 7) / 8;
  if (d.di == 128) {
    switch (nt) {
      case 1: return launch_t<128, 1>(a, st);
      case 2: return launch_t<128, 2>(a, st);
      case 3: return launch_t<128, 3>(a, st);
      default: return launch_t<128, 4>(a, st);
    }
  }
  switch (nt) {
    case 1: return launch_t<64, 1>(a, st);
    case 2: return launch_t<64, 2>(a, st);
    case 3: return launch_t<64, 3>(a, st);
    default: return launch_t<64, 4>(a, st);
  }
}

}  // namespace qsa
