// qsa_sparse_decode: exact attention over the selected micro-blocks, read as
// R context slices that each give a partial output and its log-sum-exp.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": softmax attention over the kept
// blocks uses their full-precision K and V; under DCP a rank reads just its
// own part of the main KV cache, the selector is the same on every rank, and
// the attention results are merged after the split read. Here
// the slices are the block ranges [floor(r*nb/R), floor((r+1)*nb/R)) of one
// GPU and the one selection serves all of them.
//
// Work decomposition. The selected blocks of slice r are a contiguous run of
// the ascending selection list; the run is cut into tiles of 4 blocks (16
// tokens), so a tile never spans two slices. The sequence's NT tiles, slice
// after slice, are split into ncb contiguous ranges, one per CTA (grid = ncb x
// head groups x B, ncb picked on the host so that about two CTAs per SM are in
// flight). Each CTA has one warp per KV head (up to 4); all warps walk the
// same tiles, so the heads of a token (1 KiB of K, 1 KiB of V at 4 KV heads)
// are read at about the same time.
//
// Per CTA: (1) copy the selection row to shared memory and read L_b; (2) one
// warp builds the slice table (start and count of each slice's run, tile
// prefix); (3) all threads look up the physical row of every block of the
// CTA's range in one pass of block-table loads; (4) each warp streams its
// head's tiles (8 KiB of K+V per tile) through an ST-stage cp.async ring into
// XOR-swizzled shared memory and runs S^T = K Q^T and O^T += V^T P^T on
// tensor cores (m16n8k16: the 16 MMA rows are tokens / head dims, the 8
// columns the GQA group's query heads) with an online softmax in fp32 (exp2
// domain); P^T moves from the accumulator layout to the B-operand layout with
// movmatrix. (5) At the end of each slice's run the warp holds the partial of
// its range. A slice that lies inside one CTA's range is written to o_part /
// lse_part directly; only the first and the last slice of a range can be
// shared with neighbouring CTAs, and their partials go to scratch, keyed by
// CTA + slice (distinct for all pairs, since ranges and slices are both
// ordered). (6) A second, small kernel, launched as a programmatic dependent
// of the first, combines the partials of each shared slice once all streaming
// is done (every load of a row batched, so it costs a couple of L2 round
// trips). Inside the one-call decode step it also merges the R slices
// (merge_row.cuh, the arithmetic of qsa_merge), in one of three forms: with
// R = 1 each warp merges its own row from registers; with 2 <= R <= 8 and
// every combine CTA resident at once, a CTA holds all R slices of its heads
// (a warp per slice and head) and merges them in shared memory after a
// block barrier; otherwise each CTA counts its arrival per (sequence, group
// of heads) after a fence, and the one that completes the group merges it.
//
// The same kernels serve sparse prefill rows (row_start != nullptr): a row is
// a query of a chunk; it takes its sequence's block-table row and its own
// causal length, and is otherwise a sequence of one query.
//
// Roofline: HBM-bound; algorithmic bytes = selected tokens * Hkv * D * 2 * 2
// (each selected token's K and V rows read once).
#include "common.cuh"
#include "launch.h"
#include "merge_row.cuh"

namespace qsa {
namespace {

constexpr int DV_D = 128;                    // head dim
constexpr int DV_ROWB = DV_D * 2;            // bytes per K or V row of one head
constexpr int DV_TOK = 16;                   // tokens per tile (MMA rows)
constexpr int DV_STAGE = 2 * DV_TOK * DV_ROWB;  // K tile + V tile of one head: 8 KiB
constexpr int DV_WARPS = 4;                  // KV heads per CTA
constexpr int DV_TBL_BLOCKS = 1024;          // blocks per CTA range (host guarantees)
constexpr int DV_TBL_TILES = DV_TBL_BLOCKS / 4;
constexpr int DV_RMAX = 64;
constexpr int DV_CTAS_PER_SM = 2;
constexpr size_t DV_SMEM_LIMIT = 113 * 1024;    // shared memory per CTA so that two fit an SM
constexpr int DV_CB_ROWS = 8;                   // query-head rows per combine CTA
constexpr int DV_CB_BATCH = 16;                 // records' outputs loaded together (combine)
constexpr int DV_CG_WARPS = 8;                  // warps of a combine CTA that also merges (R >= 2)
constexpr int DV_CB_PER_SM = 2;                 // combine CTAs resident per SM (256 threads, ~104 registers)
constexpr int DV_QGROUP = 2;                    // queries of a sequence per pass over K/V
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct DecodeArgs {
  const __nv_bfloat16 *k_pool, *v_pool, *q;  // q [B, Qn, Hq, D]
  const int32_t *block_table, *seq_lens, *sel;
  // [B, R + 1] slice starts of each selection from the top-k kernel of a
  // decode step (st[r] = selected blocks below floor(r nb / R)), nullptr:
  // found here by binary search
  const int32_t *starts;
  // prefill rows (nullptr for decode): row b belongs to the sequence s with
  // row_start[s] <= b < row_start[s+1] and sees L_s - T_s + (b - row_start[s]) + 1
  // tokens (T_s its chunk rows), through block-table row s
  const int32_t *row_start;
  int S;
  float *o_part, *lse_part;  // [R, B, Qn, Hq, D], [R, B, Qn, Hq]
  float *rec_o, *rec_lse;    // [B, rb, QN, Hq, D], [B, rb, QN, Hq]: shared-slice partials
  int2 *span;                // [B, R]: contributors (c_lo, c_hi) of a shared slice
  // fused merge (decode step, one query): the combine CTA that completes a
  // row group's R slices merges them into m_out / m_lse; mcnt counts the
  // arrivals per (sequence, row group). m_out == nullptr: no fused merge.
  int *mcnt;                 // [B, ceil(Hq / DV_CB_ROWS)]
  void *m_out;
  int m_bf16;
  float *m_lse;
  int B, Hq, Hkv, G, P, max_pages, num_pages, k, k_pad, R, ncb, rb;
  int Qn, q0, qn;            // queries per sequence; first query and size of this group
  int ring_bytes;            // DV_WARPS * ST * DV_STAGE
  int bt_smem;               // the block-table row (max_pages entries) is staged in the ring
  float scale_log2;
  unsigned *err;
};

__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}

// First position in the ascending list s[0..n) whose value is >= v.
__device__ __forceinline__ int lower_bound(const int32_t *s, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (s[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Slice holding tile v: the largest r < R with pre[r] <= v (pre ascending,
// pre[R] = NT > v).
__device__ __forceinline__ int slice_of_tile(const int *pre, int R, int v) {
  int lo = 0, hi = R - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// CTA whose tile range [floor(c*NT/ncb), floor((c+1)*NT/ncb)) holds tile v.
__device__ __forceinline__ int cta_of_tile(int v, int NT, int ncb) {
  // 32-bit: (v + 1) * ncb <= NT * ncb, both below 2^11 by the host's bounds
  return (int)(((unsigned)(v + 1) * (unsigned)ncb + (unsigned)NT - 1u) / (unsigned)NT) - 1;
}

// Online-softmax state of one warp: heads 2tq, 2tq+1 of the group (tq = lane
// & 3), accumulators O^T in the m16n8 layout (8 tiles of 16 head dims).
struct Acc {
  float m0, m1, l0, l1;
  float o[8][4];
  __device__ __forceinline__ void reset() {
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
  }
};

// One 16-token tile of one head for QN queries of the same sequence: K rows
// at kbase, V rows at vbase (swizzled); token i valid for query qq iff bit i
// of valid[qq]. Each K and V fragment is loaded once for all queries.
template <int QN>
__device__ __forceinline__ void attend_tile(Acc (&st)[QN], uint32_t kbase, uint32_t vbase,
                                            const unsigned (&valid)[QN],
                                            const uint32_t (&qf)[QN][8][2], float scale_log2,
                                            int lane) {
  const int gq = lane >> 2;
  const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;  // K: non-transposed x4
  const int akc = lane >> 4;
  const int vrow = (lane & 7) + ((lane >> 4) & 1) * 8;  // V: transposed x4
  const int vkc = (lane >> 3) & 1;
  // S^T[16 tokens x 8 heads] per query, in two independent accumulation chains
  float sa[QN][4], sb[QN][4];
#pragma unroll
  for (int qq = 0; qq < QN; ++qq)
#pragma unroll
    for (int i = 0; i < 4; ++i) sa[qq][i] = sb[qq][i] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
    ldsm_x4(kbase + swz(arow, 2 * ks + akc, DV_ROWB), a0, a1, a2, a3);
    ldsm_x4(kbase + swz(arow, 2 * (ks + 4) + akc, DV_ROWB), b0, b1, b2, b3);
#pragma unroll
    for (int qq = 0; qq < QN; ++qq) {
      mma_bf16_16816(sa[qq], a0, a1, a2, a3, qf[qq][ks][0], qf[qq][ks][1]);
      mma_bf16_16816(sb[qq], b0, b1, b2, b3, qf[qq][ks + 4][0], qf[qq][ks + 4][1]);
    }
  }
  float c0[QN], c1[QN];
  uint32_t pb0[QN], pb1[QN];
#pragma unroll
  for (int qq = 0; qq < QN; ++qq) {
    Acc &s_ = st[qq];
    // s[0], s[1]: token gq, heads 2tq, 2tq+1; s[2], s[3]: token gq + 8
    const bool v0 = (valid[qq] >> gq) & 1u, v1 = (valid[qq] >> (gq + 8)) & 1u;
    const float x0 = v0 ? (sa[qq][0] + sb[qq][0]) * scale_log2 : -INFINITY;
    const float x1 = v0 ? (sa[qq][1] + sb[qq][1]) * scale_log2 : -INFINITY;
    const float x2 = v1 ? (sa[qq][2] + sb[qq][2]) * scale_log2 : -INFINITY;
    const float x3 = v1 ? (sa[qq][3] + sb[qq][3]) * scale_log2 : -INFINITY;
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o_));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o_));
    }
    const float mn0 = fmaxf(s_.m0, mx0), mn1 = fmaxf(s_.m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
    c0[qq] = exp2f(s_.m0 - base0);
    c1[qq] = exp2f(s_.m1 - base1);
    const float p0 = exp2f(x0 - base0), p1 = exp2f(x1 - base1);
    const float p2 = exp2f(x2 - base0), p3 = exp2f(x3 - base1);
    float r0 = p0 + p2, r1 = p1 + p3;
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) {
      r0 += __shfl_xor_sync(0xffffffffu, r0, o_);
      r1 += __shfl_xor_sync(0xffffffffu, r1, o_);
    }
    s_.l0 = s_.l0 * c0[qq] + r0;
    s_.l1 = s_.l1 * c1[qq] + r1;
    s_.m0 = mn0;
    s_.m1 = mn1;
    // P^T (tokens x heads) in accumulator layout -> B operand (k = tokens, n = heads)
    pb0[qq] = movmatrix_t(pack_bf16x2(p0, p1));
    pb1[qq] = movmatrix_t(pack_bf16x2(p2, p3));
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    uint32_t a0, a1, a2, a3;
    ldsm_x4_t(vbase + swz(vrow, 2 * mt + vkc, DV_ROWB), a0, a1, a2, a3);
#pragma unroll
    for (int qq = 0; qq < QN; ++qq) {
      Acc &s_ = st[qq];
      s_.o[mt][0] *= c0[qq];
      s_.o[mt][1] *= c1[qq];
      s_.o[mt][2] *= c0[qq];
      s_.o[mt][3] *= c1[qq];
      mma_bf16_16816(s_.o[mt], a0, a1, a2, a3, pb0[qq], pb1[qq]);
    }
  }
}

// Write the normalised partial of heads (2tq, 2tq+1) < G: o [.., D] rows at
// o_rows (row stride D, head h at o_rows + h*D), LSE (natural log) at lse_rows.
__device__ __forceinline__ void store_partial(const Acc &s_, float *o_rows, float *lse_rows, int G,
                                              int lane) {
  const int gq = lane >> 2, tq = lane & 3;
  const int h0 = 2 * tq, h1 = 2 * tq + 1;
  const float inv0 = s_.l0 > 0.f ? 1.f / s_.l0 : 0.f;
  const float inv1 = s_.l1 > 0.f ? 1.f / s_.l1 : 0.f;
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int d = mt * 16 + gq;
    if (h0 < G) {
      o_rows[h0 * DV_D + d] = s_.o[mt][0] * inv0;
      o_rows[h0 * DV_D + d + 8] = s_.o[mt][2] * inv0;
    }
    if (h1 < G) {
      o_rows[h1 * DV_D + d] = s_.o[mt][1] * inv1;
      o_rows[h1 * DV_D + d + 8] = s_.o[mt][3] * inv1;
    }
  }
  if (gq == 0) {
    if (h0 < G) lse_rows[h0] = s_.l0 > 0.f ? (s_.m0 + log2f(s_.l0)) * LN2 : -INFINITY;
    if (h1 < G) lse_rows[h1] = s_.l1 > 0.f ? (s_.m1 + log2f(s_.l1)) * LN2 : -INFINITY;
  }
}

// Tile range [v0, v0 + n) of rank c when NT tiles are split over ncb CTAs.
__device__ __forceinline__ void tile_range(int c, int NT, int ncb, int &v0, int &n) {
  if (c >= ncb) {
    v0 = n = 0;
    return;
  }
  v0 = (int)(((unsigned)c * (unsigned)NT) / (unsigned)ncb);  // products below 2^22
  n = (int)(((unsigned)(c + 1) * (unsigned)NT) / (unsigned)ncb) - v0;
}

template <int ST, int QN>
__global__ void __launch_bounds__(DV_WARPS * 32, DV_CTAS_PER_SM) sparse_decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ int s_st[DV_RMAX], s_ct[DV_RMAX], s_pre[DV_RMAX + 1];
  __shared__ int s_gst[DV_RMAX + 1];  // slice starts given by the top-k kernel
  __shared__ int s_L;
  const int c = blockIdx.x, CL = a.ncb;
  const int hg = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int g = hg * DV_WARPS + warp;  // KV head of this warp
  const bool has_head = g < a.Hkv;
  // shared memory: ring | selection row | page table
  int32_t *s_sel = reinterpret_cast<int32_t *>(smem + a.ring_bytes);
  int32_t *s_row = s_sel + a.k_pad;               // first pool row of a block
  int32_t *s_blk = s_row + DV_TBL_BLOCKS;         // its block index (-1: none)
  uint8_t *s_nv = reinterpret_cast<uint8_t *>(s_blk + DV_TBL_BLOCKS);  // its valid tokens

  // (1) the block-table row (into shared memory when it fits the ring, which
  // is idle until streaming starts; else into L2), L_b and the query: all
  // inputs, so they are read before the wait on the top-k kernel; then the
  // selection row
  int32_t *s_bt = reinterpret_cast<int32_t *>(smem);
  auto copy_bt_row = [&](int row) {
    const int32_t *btr = a.block_table + (size_t)row * a.max_pages;
    int i0 = 0;
    if ((reinterpret_cast<uintptr_t>(btr) & 15u) == 0) {  // 16-byte pieces, then the tail
      const int n4 = a.max_pages >> 2;
      for (int i = tid; i < n4; i += blockDim.x) cp_async16(smem_u32(s_bt + 4 * i), btr + 4 * i, 16);
      i0 = 4 * n4;
    }
    for (int i = i0 + tid; i < a.max_pages; i += blockDim.x) cp_async4(smem_u32(s_bt + i), btr + i);
  };
  int bs = b;  // block-table row
  {
    int L;
    if (a.row_start == nullptr) {
      if (a.bt_smem) copy_bt_row(b);
      L = a.seq_lens[b];
    } else {  // prefill row: the chunk holding it (every thread; S is small)
      int lo = 0, hi = a.S - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(a.row_start + mid) <= b) lo = mid; else hi = mid - 1;
      }
      const int r0 = __ldg(a.row_start + lo), r1 = __ldg(a.row_start + lo + 1);
      const int Ls = __ldg(a.seq_lens + lo);
      L = 0;  // a row outside every chunk attends to nothing
      if (r0 <= b && b < r1 && r1 - r0 <= Ls) {
        L = Ls - (r1 - r0) + (b - r0) + 1;
        bs = lo;
      } else if (tid == 0) {
        raise_err(a.err, ERR_LEN);
      }
    }
    if (tid == 0) s_L = L;
    if (a.row_start != nullptr && a.bt_smem) copy_bt_row(bs);
    if (!a.bt_smem) {
      // the CTAs of a sequence pull its block-table row into L2 together, so
      // the page lookups after the slice search hit L2
      const char *bt_row = reinterpret_cast<const char *>(a.block_table + (size_t)bs * a.max_pages);
      const int lines = (a.max_pages * 4 + 127) >> 7;
      for (int i = c + CL * tid; i < lines; i += CL * (int)blockDim.x)
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(bt_row + ((size_t)i << 7)));
    }
  }
  // query fragments (B operand of S^T = K Q^T): query a.q0 + qq, head g*G + lane/4
  const int gq = lane >> 2, tq = lane & 3;
  uint32_t qf[QN][8][2];
#pragma unroll
  for (int qq = 0; qq < QN; ++qq) {
    const bool hv = has_head && gq < a.G;
    const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
        a.q + (((size_t)b * a.Qn + a.q0 + qq) * a.Hq + (hv ? g * a.G + gq : 0)) * DV_D);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qf[qq][ks][0] = hv ? qrow[ks * 8 + tq] : 0u;
      qf[qq][ks][1] = hv ? qrow[ks * 8 + 4 + tq] : 0u;
    }
  }
  pdl_wait();
  {
    const int32_t *srow = a.sel + (size_t)b * a.k;
    int i0 = 0;
    if ((reinterpret_cast<uintptr_t>(srow) & 15u) == 0) {  // 16-byte pieces, then the tail
      const int n4 = a.k >> 2;
      for (int i = tid; i < n4; i += blockDim.x) cp_async16(smem_u32(s_sel + 4 * i), srow + 4 * i, 16);
      i0 = 4 * n4;
    }
    for (int i = i0 + tid; i < a.k; i += blockDim.x) cp_async4(smem_u32(s_sel + i), srow + i);
    if (a.starts != nullptr)
      for (int r = tid; r <= a.R; r += blockDim.x)
        cp_async4(smem_u32(s_gst + r), a.starts + (size_t)b * (a.R + 1) + r);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  // (2) slice table: slice r's run starts at st[r] and holds ct[r] blocks;
  // its tiles are [pre[r], pre[r+1]) of the sequence's NT = pre[R] tiles
  const int L = s_L;
  const int nb = L <= 0 ? 0 : (L + 3) >> 2;
  int kb = min(a.k, nb);
  if (a.starts == nullptr) {
    // the list ends at its first -1 (a selection may hold fewer than
    // min(k, nb) blocks, e.g. one rank's share): valid ids come first, so the
    // predicate "entry < 0" is monotone over the row
    int lo = 0, hi = kb;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (s_sel[mid] < 0) hi = mid; else lo = mid + 1;
    }
    kb = lo;
  }
  if (warp == 0 && a.starts != nullptr) {  // the starts came with the selection
    int st[2], ct[2], nt[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = lane + 32 * h;
      st[h] = ct[h] = nt[h] = 0;
      if (r < a.R) {
        // clamped: a corrupt start can only shorten a run, never leave the row
        st[h] = min(max(s_gst[r], 0), kb);
        ct[h] = min(max(s_gst[r + 1], st[h]), kb) - st[h];
        nt[h] = (ct[h] + 3) >> 2;
      }
    }
    int inc0 = nt[0], inc1 = nt[1];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y0 = __shfl_up_sync(0xffffffffu, inc0, o), y1 = __shfl_up_sync(0xffffffffu, inc1, o);
      if (lane >= o) {
        inc0 += y0;
        inc1 += y1;
      }
    }
    inc1 += __shfl_sync(0xffffffffu, inc0, 31);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = lane + 32 * h;
      if (r < a.R) {
        s_st[r] = st[h];
        s_ct[r] = ct[h];
        s_pre[r] = (h ? inc1 : inc0) - nt[h];
      }
    }
    const int total = __shfl_sync(0xffffffffu, inc1, 31);
    if (lane == 0) {
      s_pre[a.R] = total;
      if (L < 0 && c == 0 && hg == 0) raise_err(a.err, ERR_LEN);
    }
  } else if (warp == 0) {
    int st[2], ct[2], nt[2];
    // floor(r nb / R) = r q + floor(r m / R) with nb = q R + m: 32-bit, no overflow
    const unsigned qR = (unsigned)nb / (unsigned)a.R, mR = (unsigned)nb - qR * (unsigned)a.R;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = lane + 32 * h;
      st[h] = ct[h] = nt[h] = 0;
      if (r < a.R) {
        const int lo = (int)((unsigned)r * qR + ((unsigned)r * mR) / (unsigned)a.R);
        const int hi = (int)((unsigned)(r + 1) * qR + ((unsigned)(r + 1) * mR) / (unsigned)a.R);
        st[h] = lower_bound(s_sel, kb, lo);
        ct[h] = lower_bound(s_sel, kb, hi) - st[h];
        nt[h] = (ct[h] + 3) >> 2;
      }
    }
    int inc0 = nt[0], inc1 = nt[1];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y0 = __shfl_up_sync(0xffffffffu, inc0, o), y1 = __shfl_up_sync(0xffffffffu, inc1, o);
      if (lane >= o) {
        inc0 += y0;
        inc1 += y1;
      }
    }
    inc1 += __shfl_sync(0xffffffffu, inc0, 31);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = lane + 32 * h;
      if (r < a.R) {
        s_st[r] = st[h];
        s_ct[r] = ct[h];
        s_pre[r] = (h ? inc1 : inc0) - nt[h];
      }
    }
    const int total = __shfl_sync(0xffffffffu, inc1, 31);
    if (lane == 0) {
      s_pre[a.R] = total;
      if (L < 0 && c == 0 && hg == 0) raise_err(a.err, ERR_LEN);
    }
  }
  __syncthreads();

  // (3) this CTA's tiles [v0, v0 + ntile) and the pool row of each of their
  // blocks; at most NT CTAs share the sequence, so every range is non-empty
  const int NT = s_pre[a.R];
  const int ncb = min(CL, NT);
  int v0, ntile;
  tile_range(c, NT, ncb, v0, ntile);
  if (ntile > DV_TBL_TILES) {  // excluded by the host's choice of ncb
    if (tid == 0) raise_err(a.err, ERR_SEL);
    ntile = DV_TBL_TILES;
  }
  const int nslot = 4 * ntile;
  for (int base = 0; base < nslot; base += 4 * (int)blockDim.x) {
    long long idx[4];
    int jj[4], pg[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int slot = base + tid + u * (int)blockDim.x;
      idx[u] = -1;
      jj[u] = 0;
      if (slot < nslot) {
        const int v = v0 + (slot >> 2);
        const int r = slice_of_tile(s_pre, a.R, v);
        const int off = 4 * (v - s_pre[r]) + (slot & 3);
        if (off < s_ct[r]) {
          const int j = s_sel[s_st[r] + off];
          if (j < 0 || j >= nb) {
            raise_err(a.err, ERR_SEL);
          } else {
            const int col = (4 * j) / a.P;
            if (col >= a.max_pages) {
              raise_err(a.err, ERR_BT);
            } else {
              idx[u] = (long long)bs * a.max_pages + col;
              jj[u] = j;
            }
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      pg[u] = idx[u] < 0 ? -1
              : a.bt_smem ? s_bt[idx[u] - (long long)bs * a.max_pages]
                          : __ldg(a.block_table + idx[u]);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int slot = base + tid + u * (int)blockDim.x;
      if (slot < nslot) {
        int row = -1, nv = 0;
        if (idx[u] >= 0) {
          if (pg[u] < 0 || pg[u] >= a.num_pages) {
            raise_err(a.err, ERR_PAGE);
          } else {
            row = pg[u] * a.P + (4 * jj[u]) % a.P;
            nv = min(4, L - 4 * jj[u]);
          }
        }
        s_row[slot] = row;
        s_blk[slot] = nv > 0 ? jj[u] : -1;
        s_nv[slot] = (uint8_t)nv;
      }
    }
  }
  __syncthreads();

  // contributors [c_lo, c_hi] of slice r (non-empty), from the tile split
  auto contributors = [&](int r, int &c_lo, int &c_hi) {
    const int pre = s_pre[r], nt = s_pre[r + 1] - pre;
    c_lo = cta_of_tile(pre, NT, ncb);
    c_hi = cta_of_tile(pre + nt - 1, NT, ncb);
  };
  // which slices the combine kernel must merge, and from which CTAs
  if (c == 0 && hg == 0) {
    for (int r = tid; r < a.R; r += blockDim.x) {
      int2 sp = make_int2(0, -1);
      if (s_ct[r] != 0) contributors(r, sp.x, sp.y);
      a.span[(size_t)b * a.R + r] = sp;
    }
    if (a.m_out != nullptr) {  // the fused merge's arrival counters of this sequence
      const int ng = (a.Hq + DV_CB_ROWS - 1) / DV_CB_ROWS;
      for (int g2 = tid; g2 < ng; g2 += blockDim.x) a.mcnt[(size_t)b * ng + g2] = 0;
    }
  }
  // slices that own no selected block: O_r = 0, LSE_r = -inf (CTA 0 writes them)
  if (has_head && c == 0) {
    for (int r = 0; r < a.R; ++r) {
      if (s_ct[r] != 0) continue;
      for (int qq = 0; qq < QN; ++qq) {
        for (int h = 0; h < a.G; ++h) {
          const size_t row = (((size_t)r * a.B + b) * a.Qn + a.q0 + qq) * a.Hq + g * a.G + h;
          reinterpret_cast<float4 *>(a.o_part + row * DV_D)[lane] =
              make_float4(0.f, 0.f, 0.f, 0.f);
          if (lane == 0) a.lse_part[row] = -INFINITY;
        }
      }
    }
  }

  const uint32_t ring = smem_u32(smem) + warp * ST * DV_STAGE;

  // (4) stream this head's tiles through the ring
  if (has_head && ntile > 0) {
    const int chunk = lane & 15;
    auto issue = [&](int t) {
      if (t < ntile) {
        const uint32_t kbuf = ring + (t % ST) * DV_STAGE, vbuf = kbuf + DV_TOK * DV_ROWB;
#pragma unroll
        for (int i = 0; i < DV_TOK / 2; ++i) {
          const int row = (lane >> 4) + 2 * i;
          const int slot = 4 * t + (row >> 2);
          const int row0 = s_row[slot];
          const bool ok = (row & 3) < (int)s_nv[slot];
          const size_t off = ((size_t)(row0 + (row & 3)) * a.Hkv + g) * DV_D + chunk * 8;
          const uint32_t so = swz(row, chunk, DV_ROWB);
          cp_async16(kbuf + so, ok ? (const void *)(a.k_pool + off) : (const void *)a.k_pool,
                     ok ? 16 : 0);
          cp_async16(vbuf + so, ok ? (const void *)(a.v_pool + off) : (const void *)a.v_pool,
                     ok ? 16 : 0);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int t = 0; t < ST - 1; ++t) issue(t);

    Acc acc[QN];
#pragma unroll
    for (int qq = 0; qq < QN; ++qq) acc[qq].reset();
    int cur = -1;                            // slice of the running segment
    int rs = slice_of_tile(s_pre, a.R, v0);  // slice of the current tile
    // (5) partial of slice r over this CTA's tiles
    auto flush = [&](int r) {
      int c_lo, c_hi;
      contributors(r, c_lo, c_hi);
#pragma unroll
      for (int qq = 0; qq < QN; ++qq) {
        if (c_lo == c_hi) {  // the only contributor: the partial is slice r's result
          const size_t row =
              (((size_t)r * a.B + b) * a.Qn + a.q0 + qq) * a.Hq + g * a.G;
          store_partial(acc[qq], a.o_part + row * DV_D, a.lse_part + row, a.G, lane);
        } else {  // shared with neighbouring CTAs: a record for the combine kernel
          const size_t row = (((size_t)b * a.rb + c + r) * QN + qq) * a.Hq + g * a.G;
          store_partial(acc[qq], a.rec_o + row * DV_D, a.rec_lse + row, a.G, lane);
        }
      }
    };
    for (int t = 0; t < ntile; ++t) {
      const int v = v0 + t;
      while (s_pre[rs + 1] <= v) ++rs;
      if (rs != cur) {
        if (cur >= 0) {
          flush(cur);
#pragma unroll
          for (int qq = 0; qq < QN; ++qq) acc[qq].reset();
        }
        cur = rs;
      }
      __syncwarp();  // every lane is done with the stage the next issue overwrites
      issue(t + ST - 1);
      cp_async_wait<ST - 1>();
      __syncwarp();
      unsigned valid = 0;
      int jlast = -1;
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        valid |= ((1u << s_nv[4 * t + blk]) - 1u) << (4 * blk);
        jlast = max(jlast, s_blk[4 * t + blk]);
      }
      // query q0 + qq sits at position L - Qn + q0 + qq and sees the tokens up
      // to it; only a tile reaching past the group's first query needs masks
      const int lim0 = L - a.Qn + a.q0;
      unsigned vq[QN];
      unsigned any = 0u;
#pragma unroll
      for (int qq = 0; qq < QN; ++qq) {
        vq[qq] = valid;
        if (4 * jlast + 3 > lim0) {
          unsigned m = 0u;
#pragma unroll
          for (int row = 0; row < DV_TOK; ++row) {
            const int j = s_blk[4 * t + (row >> 2)];
            if (j >= 0 && 4 * j + (row & 3) <= lim0 + qq) m |= 1u << row;
          }
          vq[qq] = valid & m;
        }
        any |= vq[qq];
      }
      const uint32_t kbuf = ring + (t % ST) * DV_STAGE;
      if (any) attend_tile<QN>(acc, kbuf, kbuf + DV_TOK * DV_ROWB, vq, qf, a.scale_log2, lane);
    }
    cp_async_wait<0>();
    pdl_trigger();
    flush(cur);
  }
}

// (6) Merge of one slice's records for one row q = (query of the group,
// head), by one warp; lane l owns dims 4l..4l+3. Lane i holds the weight of
// record i of each group of 32 (its LSE loaded in one round trip per 32
// records, the max taken across the warp); the outputs are then read
// DV_CB_BATCH records at a time, their weights broadcast from the lanes.
// Writes the slice partial to o_part / lse_part and returns it in res / lse;
// returns false for a slice the decode kernel wrote itself (inside one CTA's
// range, or empty).
__device__ __forceinline__ bool combine_slice_row(const DecodeArgs &a, int b, int r, int q,
                                                  int lane, float4 &res, float &lse) {
  const int2 sp = a.span[(size_t)b * a.R + r];
  if (sp.y <= sp.x) return false;
  const int n = sp.y - sp.x + 1;
  const size_t stride = (size_t)a.qn * a.Hq;                         // between records
  const size_t row0 = ((size_t)b * a.rb + sp.x + r) * stride + q;    // record i at row0 + i*stride
  // the first DV_CB_BATCH records' outputs are requested together with the
  // LSEs (one round trip instead of two for slices of that many records)
  float4 v[DV_CB_BATCH];
#pragma unroll
  for (int u = 0; u < DV_CB_BATCH; ++u) {
    const size_t rr = row0 + (size_t)min(u, n - 1) * stride;
    v[u] = __ldcg(reinterpret_cast<const float4 *>(a.rec_o + rr * DV_D) + lane);
  }
  float M = -INFINITY;
  for (int i0 = 0; i0 < n; i0 += 32) {
    const float l = i0 + lane < n ? __ldcg(a.rec_lse + row0 + (size_t)(i0 + lane) * stride)
                                  : -INFINITY;
    M = fmaxf(M, l);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, wsum = 0.f;
  if (M != -INFINITY) {
    for (int i0 = 0; i0 < n; i0 += 32) {
      const float l = i0 + lane < n ? __ldcg(a.rec_lse + row0 + (size_t)(i0 + lane) * stride)
                                    : -INFINITY;
      const float wl = l == -INFINITY ? 0.f : __expf(l - M);  // weight of record i0 + lane
      const int m = min(32, n - i0);
      for (int u0 = 0; u0 < m; u0 += DV_CB_BATCH) {
        if (i0 != 0 || u0 != 0) {  // (the first batch is in v already)
#pragma unroll
          for (int u = 0; u < DV_CB_BATCH; ++u) {
            const size_t rr = row0 + (size_t)(i0 + min(u0 + u, m - 1)) * stride;
            v[u] = __ldcg(reinterpret_cast<const float4 *>(a.rec_o + rr * DV_D) + lane);
          }
        }
#pragma unroll
        for (int u = 0; u < DV_CB_BATCH; ++u) {
          const float w = __shfl_sync(0xffffffffu, wl, (u0 + u) & 31);
          if (u0 + u < m && w != 0.f) {  // a record of a query that saw nothing holds zeros
            wsum += w;
            acc[0] += w * v[u].x;
            acc[1] += w * v[u].y;
            acc[2] += w * v[u].z;
            acc[3] += w * v[u].w;
          }
        }
      }
    }
  }
  const int qq = q / a.Hq, h = q % a.Hq;
  const size_t orow = (((size_t)r * a.B + b) * a.Qn + a.q0 + qq) * a.Hq + h;
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  res = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  lse = wsum > 0.f ? M + logf(wsum) : -INFINITY;
  reinterpret_cast<float4 *>(a.o_part + orow * DV_D)[lane] = res;
  if (lane == 0) a.lse_part[orow] = lse;
  return true;
}

// One CTA per (group of DV_CB_ROWS query rows, slice, sequence), one warp per
// row. The fused merge (one query per sequence): with R = 1 (SELF) each warp
// merges its own row from the registers holding its slice partial; otherwise
// the CTA whose arrival completes the row group's R slices merges them.
template <bool SELF>
__global__ void __launch_bounds__(DV_CB_ROWS * 32) decode_combine_kernel(DecodeArgs a) {
  pdl_wait();  // the records come from the decode kernel before this one
  pdl_trigger();  // the merge kernel waits for this whole grid
  const int b = blockIdx.z, r = blockIdx.y;
  const int q = blockIdx.x * DV_CB_ROWS + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  float4 res;
  float lse;
  if (q < a.qn * a.Hq && combine_slice_row(a, b, r, q, lane, res, lse)) {
    // (the loaders hand back the values just stored: the bits of qsa_merge)
    if (SELF)
      merge_row_with(1, DV_D, b * a.Hq + q, [&](int, int) { return res; },
                     [&](int) { return lse; }, a.m_out, a.m_bf16, a.m_lse);
  } else if (SELF && q < a.Hq) {
    // a selection inside one decode CTA's range, or empty: the decode kernel
    // wrote the slice's partial (one query per sequence here)
    const size_t orow = (size_t)b * a.Hq + q;
    const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.o_part + orow * DV_D) + lane);
    const float l = __ldcg(a.lse_part + orow);
    merge_row_with(1, DV_D, b * a.Hq + q, [&](int, int) { return v; }, [&](int) { return l; },
                   a.m_out, a.m_bf16, a.m_lse);
  }
  if (SELF || a.m_out == nullptr) return;
  // fused merge (one query per sequence): the CTA whose arrival completes the
  // row group's R slices merges them (its own rows, one warp per head)
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's partials before its arrival
    int *cnt = a.mcnt + (size_t)b * gridDim.x + blockIdx.x;
    s_last = atomicAdd(cnt, 1) == a.R - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();  // every other slice's partials are visible now
  if (q < a.Hq)
    merge_row(a.R, a.B * a.Hq, DV_D, a.o_part, a.lse_part, b * a.Hq + q, a.m_out, a.m_bf16,
              a.m_lse);
}

// The fused merge with 2 <= R <= DV_CG_WARPS (one query per sequence) when
// all its CTAs are resident at once: one CTA per (group of DV_CG_WARPS / R
// query heads, sequence), one warp per (slice, head). Each warp merges its
// slice's records for its head (or takes the partial the decode kernel
// wrote) and keeps the result in shared memory; after one block barrier the
// warps of slice 0 merge the R slices of their heads: no arrival counting,
// no re-read of o_part.
__global__ void __launch_bounds__(DV_CG_WARPS * 32) decode_combine_group_kernel(DecodeArgs a) {
  pdl_wait();  // the records come from the decode kernel before this one
  pdl_trigger();
  extern __shared__ float4 g_o[];  // [R][rows][32] slice partials, then the LSEs [R][rows]
  const int rows = DV_CG_WARPS / a.R;
  float *g_l = reinterpret_cast<float *>(g_o + (size_t)a.R * rows * 32);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = warp / rows, i = warp - r * rows;
  const int b = blockIdx.y, q = blockIdx.x * rows + i;
  if (r < a.R && q < a.Hq) {
    float4 res;
    float lse;
    if (!combine_slice_row(a, b, r, q, lane, res, lse)) {
      const size_t orow = ((size_t)r * a.B + b) * a.Hq + q;
      res = __ldcg(reinterpret_cast<const float4 *>(a.o_part + orow * DV_D) + lane);
      lse = __ldcg(a.lse_part + orow);
    }
    g_o[(r * rows + i) * 32 + lane] = res;
    if (lane == 0) g_l[r * rows + i] = lse;
  }
  __syncthreads();
  // (the same values as in o_part / lse_part: the bits of qsa_merge)
  if (r == 0 && q < a.Hq)
    merge_row_with(
        a.R, DV_D, b * a.Hq + q, [&](int rr, int d0) { return g_o[(rr * rows + i) * 32 + (d0 >> 2)]; },
        [&](int rr) { return g_l[rr * rows + i]; }, a.m_out, a.m_bf16, a.m_lse);
}

struct DecodePlan {
  int nhg, ncb, rb, stages, k_pad;
  size_t smem;
};

DecodePlan plan_decode(const qsa_dims &d, int B, int k, int R) {
  DecodePlan p;
  p.nhg = (d.Hkv + DV_WARPS - 1) / DV_WARPS;
  p.k_pad = (k + 3) & ~3;
  // selection row; per block slot: pool row, block index, valid tokens
  const size_t extra = (size_t)p.k_pad * 4 + (size_t)DV_TBL_BLOCKS * 9;
  const size_t static_smem = 1024;
  const size_t fit = (DV_SMEM_LIMIT - static_smem - extra) / ((size_t)DV_WARPS * DV_STAGE);
  p.stages = fit >= 4 ? 4 : (fit >= 3 ? 3 : 2);
  p.smem = (size_t)DV_WARPS * p.stages * DV_STAGE + extra;
  // CTAs per sequence: enough to keep DV_CTAS_PER_SM CTAs busy on every SM
  // of the device (the workspace size follows, so it is sized the same way
  // for the same device), at most one per tile, and enough that a CTA's tile
  // range fits its page table
  const long long slots = (long long)DV_CTAS_PER_SM * device_sm_count();
  const long long ntmax = (k + 3) / 4 + R - 1;
  long long ncb = slots / ((long long)B * p.nhg);
  if (ncb > ntmax) ncb = ntmax;
  if (ncb < 1) ncb = 1;
  const long long need = (ntmax + DV_TBL_TILES - 1) / DV_TBL_TILES;
  if (ncb < need) ncb = need;
  p.ncb = (int)ncb;
  p.rb = p.ncb + R - 1;
  return p;
}

template <int ST, int QN>
cudaError_t launch_st(const DecodeArgs &a, const DecodePlan &p, int B, cudaStream_t st) {
  cudaError_t e =
      ensure_dynamic_smem(reinterpret_cast<const void *>(sparse_decode_kernel<ST, QN>), p.smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(sparse_decode_kernel<ST, QN>, dim3(p.ncb, p.nhg, B), DV_WARPS * 32, p.smem, st,
                 a);
  if (e != cudaSuccess) return e;
  if (p.ncb == 1)  // one CTA per sequence: nothing to combine
    return a.m_out == nullptr ? e
                              : launch_merge(a.R, B, a.Hq, DV_D, a.o_part, a.lse_part, a.m_out,
                                             a.m_bf16, a.m_lse, st);
  const dim3 grid((QN * a.Hq + DV_CB_ROWS - 1) / DV_CB_ROWS, a.R, B);
  if (a.m_out != nullptr && a.R == 1)
    return launch_pdl(decode_combine_kernel<true>, grid, DV_CB_ROWS * 32, 0, st, a);
  // A CTA holding all R slices of its heads lasts as long as its slowest
  // slice: it shortens the chain while every combine CTA is resident at once,
  // but costs time when the CTAs run in several waves (then a slice's CTA
  // that finishes early makes room for the next)
  if (a.m_out != nullptr && a.R <= DV_CG_WARPS) {
    const int rows = DV_CG_WARPS / a.R;
    const long long ctas = (long long)((a.Hq + rows - 1) / rows) * B;
    if (ctas <= (long long)DV_CB_PER_SM * device_sm_count()) {
      const size_t smem = (size_t)a.R * rows * (32 * sizeof(float4) + sizeof(float));
      return launch_pdl(decode_combine_group_kernel, dim3((a.Hq + rows - 1) / rows, B),
                        a.R * rows * 32, smem, st, a);
    }
  }
  return launch_pdl(decode_combine_kernel<false>, grid, DV_CB_ROWS * 32, 0, st, a);
}

template <int QN>
cudaError_t launch_qn(const DecodeArgs &a, const DecodePlan &p, int B, cudaStream_t st) {
  switch (p.stages) {
    case 4: return launch_st<4, QN>(a, p, B, st);
    case 3: return launch_st<3, QN>(a, p, B, st);
    default: return launch_st<2, QN>(a, p, B, st);
  }
}

}  // namespace

size_t decode_ws_starts_offset(const qsa_dims &d, int B, int Qn, int k, int R) {
  const DecodePlan p = plan_decode(d, B, k, R);
  const size_t rows = (size_t)B * p.rb * (Qn < DV_QGROUP ? Qn : DV_QGROUP) * d.Hq;
  const size_t groups = (size_t)(d.Hq + DV_CB_ROWS - 1) / DV_CB_ROWS;
  const size_t used = rows * (DV_D + 1) * sizeof(float) + (size_t)B * R * sizeof(int2) +
                      (size_t)B * groups * sizeof(int);
  return (used + 15) & ~(size_t)15;
}

size_t decode_ws_bytes(const qsa_dims &d, int B, int Qn, int k, int R) {
  return decode_ws_starts_offset(d, B, Qn, k, R) + (size_t)B * (R + 1) * sizeof(int32_t);
}

cudaError_t launch_sparse_decode(const qsa_dims &d, const qsa_cache &c, int B, int Qn,
                                 const int32_t *seq_lens, const void *q, const int32_t *sel,
                                 int k, int R, float *o_part, float *lse_part, void *ws,
                                 unsigned *err, cudaStream_t st, const int32_t *row_start,
                                 int S, void *m_out, int m_bf16, float *m_lse,
                                 const int32_t *starts) {
  if (B == 0) return cudaSuccess;
  const DecodePlan p = plan_decode(d, B, k, R);
  DecodeArgs a;
  a.k_pool = static_cast<const __nv_bfloat16 *>(c.k_pool);
  a.v_pool = static_cast<const __nv_bfloat16 *>(c.v_pool);
  a.q = static_cast<const __nv_bfloat16 *>(q);
  a.block_table = c.block_table;
  a.seq_lens = seq_lens;
  a.sel = sel;
  a.starts = row_start == nullptr && Qn == 1 ? starts : nullptr;
  a.row_start = row_start;
  a.S = S;
  a.m_out = Qn == 1 ? m_out : nullptr;
  a.m_bf16 = m_bf16;
  a.m_lse = m_lse;
  a.o_part = o_part;
  a.lse_part = lse_part;
  a.B = B;
  a.Hq = d.Hq;
  a.Hkv = d.Hkv;
  a.G = d.Hq / d.Hkv;
  a.P = d.P;
  a.max_pages = c.max_pages_per_seq;
  a.num_pages = c.num_pages;
  a.k = k;
  a.k_pad = p.k_pad;
  a.R = R;
  a.ncb = p.ncb;
  a.rb = p.rb;
  a.Qn = Qn;
  a.ring_bytes = DV_WARPS * p.stages * DV_STAGE;
  a.bt_smem = (size_t)c.max_pages_per_seq * 4 <= (size_t)a.ring_bytes ? 1 : 0;
  a.scale_log2 = d.scale * LOG2E;
  a.err = err;
  // query groups of up to DV_QGROUP, each one pass over the selected K/V
  for (int q0 = 0; q0 < Qn; q0 += DV_QGROUP) {
    a.q0 = q0;
    a.qn = Qn - q0 < DV_QGROUP ? Qn - q0 : DV_QGROUP;
    const size_t rows = (size_t)B * p.rb * a.qn * d.Hq;
    a.rec_o = static_cast<float *>(ws);
    a.rec_lse = a.rec_o + rows * DV_D;
    a.span = reinterpret_cast<int2 *>(a.rec_lse + rows);
    a.mcnt = reinterpret_cast<int *>(a.span + (size_t)B * R);
    const cudaError_t e = a.qn == 2 ? launch_qn<2>(a, p, B, st) : launch_qn<1>(a, p, B, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace qsa
