// qsa_index_score: s_b = sum_h w_h * max(0, q_idx_h . kc_b) for every
// micro-block b of every sequence.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": the indexer compresses keys into
// micro-blocks at ratio 4 and "scores them". The weighted-ReLU head sum is
// this library's reading of that step (the page prints no formula).
//
// Work: a dense [blocks x di] . [di x Hi] contraction per sequence, 8 MAC per
// side-cache byte (di = 128, Hi = 16), above what fp32 CUDA cores sustain at
// HBM speed, so the dot products run on tensor cores (m16n8k16, bf16 in,
// fp32 out). Each warp streams tiles of 16 side-cache rows (one per block)
// through a 3-stage cp.async ring in shared memory (XOR-swizzled rows, so
// ldmatrix is conflict-free) and keeps the indexer query of its current
// sequence in registers as mma B fragments. The epilogue applies ReLU and
// the head weights to the fp32 accumulators and reduces over heads with two
// shuffles. The trailing partial block's key is built in the warp from the
// per-token indexer-key pool and written into its tile row before the MMA.
// The grid is persistent (2 CTAs of 8 warps per SM) over the flattened list
// of (sequence, 16-block tile), so ragged batches stay balanced.
//
// Roofline: HBM-bound; algorithmic bytes = nb * di * 2 per sequence.
#include "common.cuh"
#include "launch.h"

namespace qsa {
namespace {

constexpr int SC_WARPS = 8;
constexpr int SC_STAGES = 3;
constexpr int SC_ROWS = 16;  // blocks per warp tile

struct ScoreArgs {
  const __nv_bfloat16 *side_pool, *kidx_pool, *q_idx;
  const float *w;
  const int32_t *block_table, *seq_lens;
  float *scores;
  int B, ld, P, max_pages, num_pages, Hi;
  unsigned *err;
};

// Index of the sequence whose tile range [prefix[b], prefix[b+1]) holds t.
__device__ __forceinline__ int find_seq(const int *prefix, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int DI, int NT>
__global__ void __launch_bounds__(SC_WARPS * 32, 2) index_score_kernel(ScoreArgs a) {
  constexpr int ROWB = DI * 2;            // bytes per side-cache row
  constexpr int CH = ROWB / 16;           // 16-byte chunks per row
  constexpr int TILEB = SC_ROWS * ROWB;   // bytes per warp tile
  constexpr int KS = DI / 16;             // mma k-steps
  extern __shared__ __align__(128) unsigned char smem[];
  int *prefix = reinterpret_cast<int *>(smem);  // [B + 1] tiles before sequence b
  int *lens = prefix + (a.B + 1);               // [B] sequence lengths
  unsigned char *tiles = smem + (((2 * a.B + 1) * 4 + 127) & ~127);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- per-CTA prefix of tiles per sequence
  __shared__ int carry;
  __shared__ int wsum[SC_WARPS];
  if (threadIdx.x == 0) { carry = 0; prefix[0] = 0; }
  __syncthreads();
  for (int base = 0; base < a.B; base += blockDim.x) {
    int b = base + threadIdx.x, n = 0;
    if (b < a.B) {
      int L = a.seq_lens[b];
      int nb = L < 0 ? 0 : (L + 3) >> 2;
      if (L < 0 || nb > a.ld) {
        if (blockIdx.x == 0) raise_err(a.err, ERR_LEN);
        nb = 0;
        L = 0;
      }
      lens[b] = L;
      n = (nb + SC_ROWS - 1) / SC_ROWS;
    }
    int x = n;  // inclusive warp scan
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    int off = carry;
    for (int i = 0; i < warp; ++i) off += wsum[i];
    if (b < a.B) prefix[b + 1] = off + x;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = off + x;
    __syncthreads();
  }
  const int total = prefix[a.B];

  unsigned char *ring = tiles + warp * (SC_STAGES * TILEB);
  const uint32_t ring_s = smem_u32(ring);
  // contiguous tile range per warp: consecutive tiles stay in one sequence
  const int nwarps = gridDim.x * SC_WARPS, gwarp = blockIdx.x * SC_WARPS + warp;
  const int t_begin = (int)(((long long)gwarp * total) / nwarps);
  const int t_end = (int)(((long long)(gwarp + 1) * total) / nwarps);
  const int rows_per_page = a.P >> 2;
  const int32_t *bt_all = a.block_table;

  // Page of row (lane & 15) of tile t: one independent load per lane, issued a
  // tile ahead of its use. -1: no complete block there; -2: bounds error.
  auto lookup = [&](int t) -> int {
    if (t >= t_end) return -1;
    const int b = find_seq(prefix, a.B, t);
    const int j = (t - prefix[b]) * SC_ROWS + (lane & 15);
    if (j >= (lens[b] >> 2)) return -1;
    const int col = j / rows_per_page;
    if (col >= a.max_pages) return -2;
    const int page = __ldg(bt_all + (size_t)b * a.max_pages + col);
    return (page >= 0 && page < a.num_pages) ? page : -3;
  };
  // cp.async of tile t into stage st, given each row's page (from lookup()).
  auto issue = [&](int t, int st, int pg) {
    if (t >= t_end) return;
    const int j0 = (t - prefix[find_seq(prefix, a.B, t)]) * SC_ROWS;
    if (lane < 16 && pg < -1) raise_err(a.err, pg == -2 ? ERR_BT : ERR_PAGE);
#pragma unroll
    for (int i = 0; i < SC_ROWS * CH / 32; ++i) {
      const int q = lane + 32 * i, r = q / CH, c = q % CH;
      const int page = __shfl_sync(0xffffffffu, pg, r);
      if (page == -1) continue;
      const int j = j0 + r;
      const __nv_bfloat16 *src = a.side_pool;
      int bytes = 0;
      if (page >= 0) {
        src = a.side_pool + ((size_t)page * rows_per_page + (j % rows_per_page)) * DI + c * 8;
        bytes = 16;
      }
      cp_async16(ring_s + st * TILEB + swz(r, c, ROWB), src, bytes);
    }
  };

  // prologue: pages of the first STAGES tiles, copies of the first STAGES-1
  int pg_next[SC_STAGES];
#pragma unroll
  for (int i = 0; i < SC_STAGES; ++i) pg_next[i] = lookup(t_begin + i);
#pragma unroll
  for (int i = 0; i < SC_STAGES - 1; ++i) {
    issue(t_begin + i, i, pg_next[i]);
    cp_async_commit();
  }
  int pg_ahead = pg_next[SC_STAGES - 1];  // pages of tile it + STAGES - 1

  uint32_t qf[NT][KS][2];
  float wv[NT][2];
  int qb = -1;

  for (int it = 0;; ++it) {
    const int t = t_begin + it;
    if (t >= t_end) break;
    issue(t + SC_STAGES - 1, (it + SC_STAGES - 1) % SC_STAGES, pg_ahead);
    cp_async_commit();
    pg_ahead = lookup(t + SC_STAGES);  // consumed by the next iteration
    cp_async_wait<SC_STAGES - 1>();
    __syncwarp();

    const int st = it % SC_STAGES;
    const int b = find_seq(prefix, a.B, t);
    const int j0 = (t - prefix[b]) * SC_ROWS;
    const int L = lens[b];
    const int nfull = L >> 2, nb = (L + 3) >> 2;
    unsigned char *tile = ring + st * TILEB;

    if (b != qb) {  // indexer query of a new sequence -> B fragments, weights
      qb = b;
      const int g = lane >> 2, tq = lane & 3;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int h = nt * 8 + g;
        const uint32_t *qrow =
            reinterpret_cast<const uint32_t *>(a.q_idx + ((size_t)b * a.Hi + h) * DI);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qf[nt][ks][0] = h < a.Hi ? qrow[ks * 8 + tq] : 0u;
          qf[nt][ks][1] = h < a.Hi ? qrow[ks * 8 + 4 + tq] : 0u;
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hw = nt * 8 + 2 * tq + e;
          wv[nt][e] = hw < a.Hi ? a.w[(size_t)b * a.Hi + hw] : 0.f;
        }
      }
    }

    if (nfull < nb && nfull >= j0 && nfull < j0 + SC_ROWS) {
      // trailing partial block: key = bf16_rne(fp32 sum of its n tokens / n)
      const int n = L - 4 * nfull, pos = 4 * nfull;
      const int col = pos / a.P;
      int page = -1;
      if (col < a.max_pages) page = bt_all[(size_t)b * a.max_pages + col];
      const bool ok = page >= 0 && page < a.num_pages;
      if (!ok && lane == 0) raise_err(a.err, col < a.max_pages ? ERR_PAGE : ERR_BT);
      const uint32_t *x = reinterpret_cast<const uint32_t *>(a.kidx_pool) +
                          ((size_t)(ok ? page : 0) * a.P + pos % a.P) * (DI / 2);
      const int r = nfull - j0;
      for (int e = lane; e < DI / 2; e += 32) {
        float lo = 0.f, hi = 0.f;
        if (ok) {
          uint32_t v = x[e];
          lo = bf16lo(v);
          hi = bf16hi(v);
          for (int u = 1; u < n; ++u) {
            v = x[u * (DI / 2) + e];
            lo = __fadd_rn(lo, bf16lo(v));
            hi = __fadd_rn(hi, bf16hi(v));
          }
          lo = __fdiv_rn(lo, (float)n);
          hi = __fdiv_rn(hi, (float)n);
        }
        *reinterpret_cast<uint32_t *>(tile + swz(r, e >> 2, ROWB) + (e & 3) * 4) =
            pack_bf16x2(lo, hi);
      }
      __syncwarp();
    }

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
    const uint32_t ts = ring_s + st * TILEB;
    const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(ts + swz(arow, 2 * ks + (lane >> 4), ROWB), a0, a1, a2, a3);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        mma_bf16_16816(acc[nt], a0, a1, a2, a3, qf[nt][ks][0], qf[nt][ks][1]);
    }
    float s0 = 0.f, s1 = 0.f;  // rows g and g + 8 of the tile
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s0 += wv[nt][0] * fmaxf(acc[nt][0], 0.f) + wv[nt][1] * fmaxf(acc[nt][1], 0.f);
      s1 += wv[nt][0] * fmaxf(acc[nt][2], 0.f) + wv[nt][1] * fmaxf(acc[nt][3], 0.f);
    }
    s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
    s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
    if ((lane & 3) == 0) {
      const int g = lane >> 2;
      float *out = a.scores + (size_t)b * a.ld + j0;
      if (j0 + g < nb) out[g] = s0;
      if (j0 + g + 8 < nb) out[g + 8] = s1;
    }
    __syncwarp();  // the stage is refilled by the next iteration's issue
  }
  cp_async_wait<0>();
}

template <int DI, int NT>
cudaError_t launch_t(const ScoreArgs &a, cudaStream_t st) {
  const size_t smem = (((size_t)(2 * a.B + 1) * 4 + 127) & ~(size_t)127) +
                      (size_t)SC_WARPS * SC_STAGES * SC_ROWS * DI * 2;
  auto kern = index_score_kernel<DI, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = device_sm_count() * 2;
  kern<<<grid, SC_WARPS * 32, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_score(const qsa_dims &d, const qsa_cache &c, int B,
                               const int32_t *seq_lens, const void *q_idx, const float *w,
                               float *scores, int ld, unsigned *err, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  if (index_score_tc_supported(d))
    return launch_index_score_tc(d, c, B, seq_lens, q_idx, w, scores, ld, err, st);
  ScoreArgs a;
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
