// qsa_sparse_decode: exact attention over the selected micro-blocks, read as
// R context slices that each give a partial output and its log-sum-exp.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": the final softmax and value
// aggregation run on the uncompressed K and V of the kept blocks; under DCP
// each rank reads only its slice of the main KV cache while the selector
// stays replicated, and the attention results are combined afterwards. Here
// the slices are the block ranges [floor(r*nb/R), floor((r+1)*nb/R)) of one
// GPU and the one selection serves all of them.
//
// Work decomposition: the selected blocks of slice r form a contiguous run of
// the (ascending) selection list; each run is cut into chunks of DC_BLOCKS
// blocks. A CTA = (chunk slot, KV head, sequence); the slot count per
// (sequence, KV head) is ceil(k / DC_BLOCKS) + R, an upper bound on the
// chunks over all slices, so the grid is fixed on the host while the chunk
// boundaries are found on the device. Each warp gathers 8 blocks (32 tokens
// x 256 B of K and of V for its KV head) with 16-byte cp.async into swizzled
// shared memory, then runs S^T = K Q^T and O^T += V^T P^T on tensor cores
// (m16n8k16: the 16 MMA rows are tokens / head dims, the 8 columns are the
// GQA group's query heads, so no MMA row is wasted) with an online softmax
// in fp32 (exp2 domain). P^T moves from the accumulator layout to the B
// operand layout with movmatrix. The warps of a CTA merge through shared
// memory; a second small kernel merges the chunks of each slice into the
// R partials.
//
// Roofline: HBM-bound; algorithmic bytes = tokens * Hkv * D * 2 * 2 per
// sequence (each selected token's K and V rows read once).
#include "common.cuh"
#include "launch.h"

namespace qsa {
namespace {

constexpr int DC_WARPS = 4;
constexpr int DC_BPW = 8;                       // blocks per warp
constexpr int DC_BLOCKS = DC_WARPS * DC_BPW;    // blocks per CTA chunk
constexpr int DC_D = 128;                       // head dim
constexpr int DC_ROWB = DC_D * 2;               // bytes per K/V row
constexpr int DC_TOK = DC_BPW * 4;              // token rows per warp
constexpr int DC_WARP_SMEM = 2 * DC_TOK * DC_ROWB;  // K + V tiles per warp
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct DecodeArgs {
  const __nv_bfloat16 *k_pool, *v_pool, *q;
  const int32_t *block_table, *seq_lens, *sel;
  float *ws_o, *ws_lse;      // [B, Hkv, nslots, G, D], [B, Hkv, nslots, G]
  float *o_part, *lse_part;  // [R, B, Hq, D], [R, B, Hq]
  int B, Hq, Hkv, G, P, max_pages, num_pages, k, R, nslots;
  float scale_log2;
  unsigned *err;
};

// First position in the ascending list s[0..n) whose value is >= v.
__device__ __forceinline__ int lower_bound(const int32_t *s, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    int mid = (lo + hi) >> 1;
    if (s[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Chunk layout of one sequence, computed by one full warp: for slice r, its
// selection run starts at `start` and holds `count` blocks; its chunks use
// slots [slot0, slot0 + ceil(count / DC_BLOCKS)). Returns the values for the
// slice `want_r`, or locates the slice holding slot `want_slot`.
struct SliceInfo {
  int r, start, count, slot0, nchunks;
};

__device__ SliceInfo slice_info(const DecodeArgs &a, int b, int want_r, int want_slot) {
  const int lane = threadIdx.x & 31;
  const int L = a.seq_lens[b];
  const int nb = L <= 0 ? 0 : (L + 3) >> 2;
  const int kb = min(a.k, nb);
  const int32_t *s = a.sel + (size_t)b * a.k;
  int st[2], ct[2], ch[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = lane + 32 * h;
    st[h] = ct[h] = ch[h] = 0;
    if (r < a.R) {
      const int lo = (int)(((long long)r * nb) / a.R);
      const int hi = (int)(((long long)(r + 1) * nb) / a.R);
      st[h] = lower_bound(s, kb, lo);
      ct[h] = lower_bound(s, kb, hi) - st[h];
      ch[h] = (ct[h] + DC_BLOCKS - 1) / DC_BLOCKS;
    }
  }
  int inc0 = ch[0], inc1 = ch[1];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y0 = __shfl_up_sync(0xffffffffu, inc0, o), y1 = __shfl_up_sync(0xffffffffu, inc1, o);
    if (lane >= o) { inc0 += y0; inc1 += y1; }
  }
  inc1 += __shfl_sync(0xffffffffu, inc0, 31);
  const int ex0 = inc0 - ch[0], ex1 = inc1 - ch[1];
  SliceInfo out{-1, 0, 0, 0, 0};
  unsigned hit0, hit1;
  if (want_r >= 0) {
    hit0 = __ballot_sync(0xffffffffu, lane == want_r);
    hit1 = __ballot_sync(0xffffffffu, lane + 32 == want_r);
  } else {
    hit0 = __ballot_sync(0xffffffffu, lane < a.R && ch[0] > 0 && want_slot >= ex0 &&
                                          want_slot < ex0 + ch[0]);
    hit1 = __ballot_sync(0xffffffffu, lane + 32 < a.R && ch[1] > 0 && want_slot >= ex1 &&
                                          want_slot < ex1 + ch[1]);
  }
  const int h = hit0 ? 0 : (hit1 ? 1 : -1);
  if (h >= 0) {
    const int src = __ffs(h == 0 ? hit0 : hit1) - 1;
    out.r = src + 32 * h;
    out.start = __shfl_sync(0xffffffffu, h == 0 ? st[0] : st[1], src);
    out.count = __shfl_sync(0xffffffffu, h == 0 ? ct[0] : ct[1], src);
    out.slot0 = __shfl_sync(0xffffffffu, h == 0 ? ex0 : ex1, src);
    out.nchunks = __shfl_sync(0xffffffffu, h == 0 ? ch[0] : ch[1], src);
  }
  return out;
}

__global__ void __launch_bounds__(DC_WARPS * 32) sparse_decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_info[3];  // slice r, first selection index, blocks in chunk
  __shared__ float s_m[DC_WARPS][8], s_l[DC_WARPS][8];
  const int slot = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0) {
    const SliceInfo si = slice_info(a, b, -1, slot);
    if (lane == 0) {
      if (si.r < 0) {
        s_info[2] = 0;
      } else {
        const int c = slot - si.slot0;
        s_info[0] = si.r;
        s_info[1] = si.start + c * DC_BLOCKS;
        s_info[2] = min(DC_BLOCKS, si.count - c * DC_BLOCKS);
      }
    }
  }
  __syncthreads();
  const int count = s_info[2];
  if (count <= 0) return;  // slot beyond this sequence's chunks
  const int first = s_info[1];
  const int L = a.seq_lens[b];
  const int nb = (L + 3) >> 2;

  // ---- gather: this warp's blocks [warp*8, warp*8+8) of the chunk
  unsigned char *wsm = smem + warp * DC_WARP_SMEM;
  const uint32_t ks_base = smem_u32(wsm), vs_base = ks_base + DC_TOK * DC_ROWB;
  int my_row0 = 0;       // lane < 8: first pool row of block `lane`
  unsigned my_bits = 0;  // lane < 8: valid-token bits of that block
  if (lane < DC_BPW) {
    const int bi = warp * DC_BPW + lane;
    if (bi < count) {
      const int j = a.sel[(size_t)b * a.k + first + bi];
      if (j < 0 || j >= nb) {
        raise_err(a.err, ERR_SEL);
      } else {
        const int col = (4 * j) / a.P;
        if (col >= a.max_pages) {
          raise_err(a.err, ERR_BT);
        } else {
          const int page = a.block_table[(size_t)b * a.max_pages + col];
          if (page < 0 || page >= a.num_pages) {
            raise_err(a.err, ERR_PAGE);
          } else {
            my_row0 = page * a.P + (4 * j) % a.P;
            const int nv = min(4, L - 4 * j);
            my_bits = (1u << nv) - 1u;
          }
        }
      }
    }
  }
  const unsigned valid =
      __reduce_or_sync(0xffffffffu, lane < DC_BPW ? my_bits << (4 * lane) : 0u);
  // 32 rows x 16 chunks for K and for V; lane owns chunk (lane & 15) of rows
  // (lane >> 4) + 2i.
  const int chunk = lane & 15;
#pragma unroll
  for (int i = 0; i < DC_TOK / 2; ++i) {
    const int row = (lane >> 4) + 2 * i;
    const int row0 = __shfl_sync(0xffffffffu, my_row0, row >> 2);
    const bool ok = (valid >> row) & 1u;
    const size_t off = ((size_t)(row0 + (row & 3)) * a.Hkv + g) * DC_D + chunk * 8;
    const uint32_t so = swz(row, chunk, DC_ROWB);
    cp_async16(ks_base + so, ok ? (const void *)(a.k_pool + off) : (const void *)a.k_pool,
               ok ? 16 : 0);
    cp_async16(vs_base + so, ok ? (const void *)(a.v_pool + off) : (const void *)a.v_pool,
               ok ? 16 : 0);
  }
  cp_async_commit();

  // ---- query fragments (B operand of S^T = K Q^T): head g*G + lane/4
  const int gq = lane >> 2, tq = lane & 3;
  uint32_t qf[8][2];
  {
    const bool hv = gq < a.G;
    const uint32_t *qrow = reinterpret_cast<const uint32_t *>(
        a.q + ((size_t)b * a.Hq + g * a.G + (hv ? gq : 0)) * DC_D);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qf[ks][0] = hv ? qrow[ks * 8 + tq] : 0u;
      qf[ks][1] = hv ? qrow[ks * 8 + 4 + tq] : 0u;
    }
  }
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // heads 2tq, 2tq+1
  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;

  cp_async_wait<0>();
  __syncwarp();

  const int arow = (lane & 7) + ((lane >> 3) & 1) * 8;   // K: non-transposed x4
  const int akc = lane >> 4;
  const int vrow = (lane & 7) + ((lane >> 4) & 1) * 8;   // V: transposed x4
  const int vkc = (lane >> 3) & 1;
#pragma unroll
  for (int tt = 0; tt < DC_TOK / 16; ++tt) {
    if (((valid >> (16 * tt)) & 0xffffu) == 0u) continue;  // warp-uniform
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(ks_base + swz(tt * 16 + arow, 2 * ks + akc, DC_ROWB), a0, a1, a2, a3);
      mma_bf16_16816(s, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
    }
    // s[0], s[1]: token gq, heads 2tq, 2tq+1; s[2], s[3]: token gq + 8
    const bool v0 = (valid >> (16 * tt + gq)) & 1u, v1 = (valid >> (16 * tt + gq + 8)) & 1u;
    float x0 = v0 ? s[0] * a.scale_log2 : -INFINITY;
    float x1 = v0 ? s[1] * a.scale_log2 : -INFINITY;
    float x2 = v1 ? s[2] * a.scale_log2 : -INFINITY;
    float x3 = v1 ? s[3] * a.scale_log2 : -INFINITY;
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o_));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o_));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float base0 = mn0 == -INFINITY ? 0.f : mn0, base1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = exp2f(m0 - base0), c1 = exp2f(m1 - base1);
    const float p0 = exp2f(x0 - base0), p1 = exp2f(x1 - base1);
    const float p2 = exp2f(x2 - base0), p3 = exp2f(x3 - base1);
    float r0 = p0 + p2, r1 = p1 + p3;
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) {
      r0 += __shfl_xor_sync(0xffffffffu, r0, o_);
      r1 += __shfl_xor_sync(0xffffffffu, r1, o_);
    }
    l0 = l0 * c0 + r0;
    l1 = l1 * c1 + r1;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      o[mt][0] *= c0;
      o[mt][1] *= c1;
      o[mt][2] *= c0;
      o[mt][3] *= c1;
    }
    // P^T (tokens x heads) in accumulator layout -> B operand (k = tokens, n = heads)
    const uint32_t pb0 = movmatrix_t(pack_bf16x2(p0, p1));
    const uint32_t pb1 = movmatrix_t(pack_bf16x2(p2, p3));
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4_t(vs_base + swz(tt * 16 + vrow, 2 * mt + vkc, DC_ROWB), a0, a1, a2, a3);
      mma_bf16_16816(o[mt], a0, a1, a2, a3, pb0, pb1);
    }
  }

  // ---- merge the warps of the CTA through shared memory
  __syncthreads();  // every warp is done with its K/V tiles
  float *s_o = reinterpret_cast<float *>(smem);  // [DC_WARPS][8 heads][D]
  if (gq == 0) {
    s_m[warp][2 * tq] = m0;
    s_m[warp][2 * tq + 1] = m1;
    s_l[warp][2 * tq] = l0;
    s_l[warp][2 * tq + 1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    float *w0 = s_o + (warp * 8 + 2 * tq) * DC_D + mt * 16 + gq;
    float *w1 = w0 + DC_D;
    w0[0] = o[mt][0];
    w1[0] = o[mt][1];
    w0[8] = o[mt][2];
    w1[8] = o[mt][3];
  }
  __syncthreads();
  // thread -> (head h, 8 consecutive dims)
  const int h = threadIdx.x >> 4, d0 = (threadIdx.x & 15) * 8;
  if (h < a.G) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < DC_WARPS; ++w) M = fmaxf(M, s_m[w][h]);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < DC_WARPS; ++w) {
        const float f = exp2f(s_m[w][h] - M);
        lsum += f * s_l[w][h];
        const float *src = s_o + (w * 8 + h) * DC_D + d0;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += f * src[e];
      }
    }
    const size_t row = (((size_t)b * a.Hkv + g) * a.nslots + slot) * a.G + h;
    float *dst = a.ws_o + row * DC_D + d0;
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e] = acc[e] * inv;
    if (d0 == 0) a.ws_lse[row] = lsum > 0.f ? (M + log2f(lsum)) * LN2 : -INFINITY;
  }
}

// One warp per (slice r, KV head g, query head h of the group, sequence b):
// merge the chunks of slice r into o_part[r, b, g*G + h, :].
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeArgs a) {
  const int r = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const SliceInfo si = slice_info(a, b, r, -1);
  if (threadIdx.x == 0 && r == 0 && g == 0 && a.seq_lens[b] < 0) raise_err(a.err, ERR_LEN);
  if (warp >= a.G) return;
  const int hq = g * a.G + warp;
  float *dst = a.o_part + (((size_t)r * a.B + b) * a.Hq + hq) * DC_D + lane * 4;
  float *lse_dst = a.lse_part + ((size_t)r * a.B + b) * a.Hq + hq;
  const size_t row0 = (((size_t)b * a.Hkv + g) * a.nslots + si.slot0) * a.G + warp;
  float M = -INFINITY;
  for (int c = 0; c < si.nchunks; ++c) M = fmaxf(M, a.ws_lse[row0 + (size_t)c * a.G]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (M != -INFINITY) {
    for (int c = 0; c < si.nchunks; ++c) {
      const size_t row = row0 + (size_t)c * a.G;
      const float f = __expf(a.ws_lse[row] - M);
      const float4 v = *reinterpret_cast<const float4 *>(a.ws_o + row * DC_D + lane * 4);
      acc.x += f * v.x;
      acc.y += f * v.y;
      acc.z += f * v.z;
      acc.w += f * v.w;
      wsum += f;
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  *reinterpret_cast<float4 *>(dst) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lane == 0) *lse_dst = wsum > 0.f ? M + logf(wsum) : -INFINITY;
}

}  // namespace

int decode_num_slots(int k, int R) { return (k + DC_BLOCKS - 1) / DC_BLOCKS + R; }

size_t decode_ws_bytes(const qsa_dims &d, int B, int k, int R) {
  const size_t rows = (size_t)B * d.Hkv * decode_num_slots(k, R) * (d.Hq / d.Hkv);
  return rows * (DC_D + 1) * sizeof(float);
}

cudaError_t launch_sparse_decode(const qsa_dims &d, const qsa_cache &c, int B,
                                 const int32_t *seq_lens, const void *q, const int32_t *sel,
                                 int k, int R, float *o_part, float *lse_part, void *ws,
                                 unsigned *err, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  DecodeArgs a;
  a.k_pool = static_cast<const __nv_bfloat16 *>(c.k_pool);
  a.v_pool = static_cast<const __nv_bfloat16 *>(c.v_pool);
  a.q = static_cast<const __nv_bfloat16 *>(q);
  a.block_table = c.block_table;
  a.seq_lens = seq_lens;
  a.sel = sel;
  a.nslots = decode_num_slots(k, R);
  a.G = d.Hq / d.Hkv;
  const size_t rows = (size_t)B * d.Hkv * a.nslots * a.G;
  a.ws_o = static_cast<float *>(ws);
  a.ws_lse = a.ws_o + rows * DC_D;
  a.o_part = o_part;
  a.lse_part = lse_part;
  a.B = B;
  a.Hq = d.Hq;
  a.Hkv = d.Hkv;
  a.P = d.P;
  a.max_pages = c.max_pages_per_seq;
  a.num_pages = c.num_pages;
  a.k = k;
  a.R = R;
  a.scale_log2 = d.scale * LOG2E;
  a.err = err;
  const size_t smem = (size_t)DC_WARPS * DC_WARP_SMEM;
  cudaError_t e = cudaFuncSetAttribute(sparse_decode_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  sparse_decode_kernel<<<dim3(a.nslots, d.Hkv, B), DC_WARPS * 32, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<dim3(R, d.Hkv, B), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace qsa
