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
// boundaries are found on the device. Each warp gathers 4 blocks (16 tokens
// x 256 B of K and of V for its KV head) with 16-byte cp.async into swizzled
// shared memory, then runs S^T = K Q^T and O^T += V^T P^T on tensor cores
// (m16n8k16: the 16 MMA rows are tokens / head dims, the 8 columns are the
// GQA group's query heads, so no MMA row is wasted) with an online softmax
// in fp32 (exp2 domain). P^T moves from the accumulator layout to the B
// operand layout with movmatrix. The warps of a CTA merge through shared
// memory into one chunk partial (scratch, L2-resident); the CTA that
// finishes a slice last (per-slice arrival counter, zeroed by the call)
// merges that slice's chunks into its R partial. Slot 0 of each (sequence,
// KV head) writes the empty slices. One kernel launch plus a small memset.
//
// Roofline: HBM-bound; algorithmic bytes = tokens * Hkv * D * 2 * 2 per
// sequence (each selected token's K and V rows read once).
#include "common.cuh"
#include "launch.h"

namespace qsa {
namespace {

constexpr int DC_WARPS = 4;
constexpr int DC_BPW = 4;                       // blocks per warp (one 16-token MMA tile)
constexpr int DC_BLOCKS = DC_WARPS * DC_BPW;    // blocks per CTA chunk
constexpr int DC_D = 128;                       // head dim
constexpr int DC_ROWB = DC_D * 2;               // bytes per K/V row
constexpr int DC_TOK = DC_BPW * 4;              // token rows per warp
constexpr int DC_WARP_SMEM = 2 * DC_TOK * DC_ROWB;  // K + V tiles per warp
constexpr int DC_SEL_SMEM = 1024;               // selection entries staged in smem
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

struct DecodeArgs {
  const __nv_bfloat16 *k_pool, *v_pool, *q;
  const int32_t *block_table, *seq_lens, *sel;
  float *ws_o, *ws_lse;      // [B, Hkv, nslots, G, D], [B, Hkv, nslots, G]
  unsigned *ws_cnt;          // [B, Hkv, R] chunks of each slice finished so far
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

// Chunk layout of one sequence, computed by one full warp. Lane l holds
// slices l and l + 32: the run of slice r in the selection list starts at
// st and holds ct blocks; its ch = ceil(ct / DC_BLOCKS) chunks use slots
// [ex, ex + ch) (slots are numbered slice after slice).
struct SliceTable {
  int st[2], ct[2], ch[2], ex[2];
};

// `s` is the sequence's selection row (ascending, first kb = min(k, nb) valid).
__device__ SliceTable slice_table(const DecodeArgs &a, int b, const int32_t *s) {
  const int lane = threadIdx.x & 31;
  const int L = a.seq_lens[b];
  const int nb = L <= 0 ? 0 : (L + 3) >> 2;
  const int kb = min(a.k, nb);
  SliceTable t;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = lane + 32 * h;
    t.st[h] = t.ct[h] = t.ch[h] = 0;
    if (r < a.R) {
      const int lo = (int)(((long long)r * nb) / a.R);
      const int hi = (int)(((long long)(r + 1) * nb) / a.R);
      t.st[h] = lower_bound(s, kb, lo);
      t.ct[h] = lower_bound(s, kb, hi) - t.st[h];
      t.ch[h] = (t.ct[h] + DC_BLOCKS - 1) / DC_BLOCKS;
    }
  }
  int inc0 = t.ch[0], inc1 = t.ch[1];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y0 = __shfl_up_sync(0xffffffffu, inc0, o), y1 = __shfl_up_sync(0xffffffffu, inc1, o);
    if (lane >= o) { inc0 += y0; inc1 += y1; }
  }
  inc1 += __shfl_sync(0xffffffffu, inc0, 31);
  t.ex[0] = inc0 - t.ch[0];
  t.ex[1] = inc1 - t.ch[1];
  return t;
}

struct SliceInfo {
  int r, start, count, slot0, nchunks;
};

// The slice holding chunk slot `slot` (r = -1 if the slot is unused).
__device__ SliceInfo slice_of_slot(const SliceTable &t, int R, int slot) {
  const int lane = threadIdx.x & 31;
  SliceInfo out{-1, 0, 0, 0, 0};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const unsigned hit = __ballot_sync(0xffffffffu, lane + 32 * h < R && t.ch[h] > 0 &&
                                                        slot >= t.ex[h] &&
                                                        slot < t.ex[h] + t.ch[h]);
    if (hit && out.r < 0) {
      const int src = __ffs(hit) - 1;
      out.r = src + 32 * h;
      out.start = __shfl_sync(0xffffffffu, t.st[h], src);
      out.count = __shfl_sync(0xffffffffu, t.ct[h], src);
      out.slot0 = __shfl_sync(0xffffffffu, t.ex[h], src);
      out.nchunks = __shfl_sync(0xffffffffu, t.ch[h], src);
    }
  }
  return out;
}

__global__ void __launch_bounds__(DC_WARPS * 32) sparse_decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_info[5];  // slice r, first selection index, blocks, slot0, chunks
  __shared__ float s_m[DC_WARPS][8], s_l[DC_WARPS][8];
  __shared__ int s_last;
  __shared__ int32_t s_sel[DC_SEL_SMEM];
  const int slot = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the selection row, staged once so that the slice searches run in shared memory
  const int32_t *sel_row = a.sel + (size_t)b * a.k;
  if (a.k <= DC_SEL_SMEM) {
    for (int i = threadIdx.x; i < a.k; i += blockDim.x) s_sel[i] = sel_row[i];
    sel_row = s_sel;
  }
  __syncthreads();
  if (warp == 0) {
    const SliceTable tab = slice_table(a, b, sel_row);
    const SliceInfo si = slice_of_slot(tab, a.R, slot);
    if (lane == 0) {
      if (si.r < 0) {
        s_info[2] = 0;
      } else {
        const int c = slot - si.slot0;
        s_info[0] = si.r;
        s_info[1] = si.start + c * DC_BLOCKS;
        s_info[2] = min(DC_BLOCKS, si.count - c * DC_BLOCKS);
        s_info[3] = si.slot0;
        s_info[4] = si.nchunks;
      }
    }
    if (slot == 0) {
      // slices that own no selected block: O_r = 0, LSE_r = -inf
      if (lane == 0 && g == 0 && a.seq_lens[b] < 0) raise_err(a.err, ERR_LEN);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        unsigned empty = __ballot_sync(0xffffffffu, lane + 32 * hh < a.R && tab.ch[hh] == 0);
        while (empty) {
          const int r = __ffs(empty) - 1 + 32 * hh;
          empty &= empty - 1;
          for (int h = 0; h < a.G; ++h) {
            const size_t row = ((size_t)r * a.B + b) * a.Hq + g * a.G + h;
            *reinterpret_cast<float4 *>(a.o_part + row * DC_D + lane * 4) =
                make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane == 0) a.lse_part[row] = -INFINITY;
          }
        }
      }
    }
  }
  __syncthreads();
  const int count = s_info[2];
  if (count <= 0) return;  // slot beyond this sequence's chunks
  const int first = s_info[1];
  const int L = a.seq_lens[b];
  const int nb = (L + 3) >> 2;

  // ---- gather: this warp's blocks [warp*DC_BPW, (warp+1)*DC_BPW) of the chunk
  unsigned char *wsm = smem + warp * DC_WARP_SMEM;
  const uint32_t ks_base = smem_u32(wsm), vs_base = ks_base + DC_TOK * DC_ROWB;
  int my_row0 = 0;       // lane < DC_BPW: first pool row of block `lane`
  unsigned my_bits = 0;  // lane < DC_BPW: valid-token bits of that block
  if (lane < DC_BPW) {
    const int bi = warp * DC_BPW + lane;
    if (bi < count) {
      const int j = sel_row[first + bi];
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
  // DC_TOK rows x 16 chunks for K and for V; lane owns chunk (lane & 15) of
  // rows (lane >> 4) + 2i.
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
    *reinterpret_cast<float4 *>(dst) =
        make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<float4 *>(dst + 4) =
        make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    if (d0 == 0) a.ws_lse[row] = lsum > 0.f ? (M + log2f(lsum)) * LN2 : -INFINITY;
  }

  // ---- the CTA that finishes slice r last merges its chunks into o_part[r]
  // (barrier, then one gpu-scope fence and the arrival by thread 0: the fence
  // is cumulative over the CTA's partial writes the barrier ordered before it)
  const int r = s_info[0], slot0 = s_info[3], nchunks = s_info[4];
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned done = atomicAdd(a.ws_cnt + ((size_t)b * a.Hkv + g) * a.R + r, 1u);
    __threadfence();
    s_last = (done + 1u == (unsigned)nchunks);
  }
  __syncthreads();
  if (!s_last) return;
  if (h < a.G) {
    const size_t row0 = (((size_t)b * a.Hkv + g) * a.nslots + slot0) * a.G + h;
    float M = -INFINITY;
    for (int c = 0; c < nchunks; ++c) M = fmaxf(M, __ldcg(a.ws_lse + row0 + (size_t)c * a.G));
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, wsum = 0.f;
    if (M != -INFINITY) {
      for (int c = 0; c < nchunks; ++c) {
        const size_t rc = row0 + (size_t)c * a.G;
        const float f = __expf(__ldcg(a.ws_lse + rc) - M);
        const float4 v0 = __ldcg(reinterpret_cast<const float4 *>(a.ws_o + rc * DC_D + d0));
        const float4 v1 = __ldcg(reinterpret_cast<const float4 *>(a.ws_o + rc * DC_D + d0 + 4));
        acc[0] += f * v0.x; acc[1] += f * v0.y; acc[2] += f * v0.z; acc[3] += f * v0.w;
        acc[4] += f * v1.x; acc[5] += f * v1.y; acc[6] += f * v1.z; acc[7] += f * v1.w;
        wsum += f;
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    const size_t orow = ((size_t)r * a.B + b) * a.Hq + g * a.G + h;
    float *o = a.o_part + orow * DC_D + d0;
    *reinterpret_cast<float4 *>(o) =
        make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<float4 *>(o + 4) =
        make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
    if (d0 == 0) a.lse_part[orow] = wsum > 0.f ? M + logf(wsum) : -INFINITY;
  }
}

}  // namespace

int decode_num_slots(int k, int R) { return (k + DC_BLOCKS - 1) / DC_BLOCKS + R; }

size_t decode_ws_bytes(const qsa_dims &d, int B, int k, int R) {
  const size_t rows = (size_t)B * d.Hkv * decode_num_slots(k, R) * (d.Hq / d.Hkv);
  return rows * (DC_D + 1) * sizeof(float) + (size_t)B * d.Hkv * R * sizeof(unsigned);
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
  a.ws_cnt = reinterpret_cast<unsigned *>(a.ws_lse + rows);
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
  e = cudaMemsetAsync(a.ws_cnt, 0, (size_t)B * d.Hkv * R * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  sparse_decode_kernel<<<dim3(a.nslots, d.Hkv, B), DC_WARPS * 32, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace qsa
