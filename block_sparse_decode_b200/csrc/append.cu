// qsa_append: scatter new tokens into the paged pools, then store the
// compressed key of every micro-block those tokens close.
//
// Page "Qwen 4 QSA gets decode context parallelism" (orcarouter.ai), section
// "What the pull request actually changes": QSA keeps the main KV cache plus
// the indexer's selector/side caches; keys are compressed into micro-blocks
// at ratio 4; synthetic batches must not write the side caches (padding
// entries here write nothing at all).
//
// Two phases: the first writes K, V and the per-token indexer key of every
// token (one warp per token, 16-byte loads and stores); the second, for every
// token with pos % 4 == 3, reads the block's 4 indexer keys back from the pool
// and writes their mean. Ordering the phases makes a bulk prefill (tokens of a
// block written by the same call, in any order) give the same side cache as
// one token per call. Up to 128 tokens (decode: one per sequence) both phases
// run in one CTA separated by a barrier, one launch; larger calls use two
// launches on the stream. Traffic is a few KiB per token; decode appends are
// latency-bound.
#include "common.cuh"
#include "launch.h"

namespace qsa {
namespace {

struct AppendArgs {
  const int32_t *tok_seq, *tok_pos;
  const uint4 *k_new, *v_new, *x_new;
  uint4 *k_pool, *v_pool, *x_pool;
  __nv_bfloat16 *side_pool;
  const int32_t *block_table;
  int N, P, num_seqs, max_pages, num_pages;
  int kv_vec;  // 16-byte vectors per token row of K (= of V): Hkv*D/8
  int x_vec;   // 16-byte vectors per indexer key: di/8
  int di;
  unsigned *err;
};

// Physical page of (seq, pos), or -1 after flagging a bounds error.
__device__ __forceinline__ int locate(const AppendArgs &a, int s, int p, int lane) {
  if (s >= a.num_seqs) {
    if (lane == 0) raise_err(a.err, ERR_SEQ);
    return -1;
  }
  int j = p / a.P;
  if (j >= a.max_pages) {
    if (lane == 0) raise_err(a.err, ERR_BT);
    return -1;
  }
  int page = a.block_table[(size_t)s * a.max_pages + j];
  if (page < 0 || page >= a.num_pages) {
    if (lane == 0) raise_err(a.err, ERR_PAGE);
    return -1;
  }
  return page;
}

// Phase 1 for one token (one warp): K, V and indexer key into the pools.
// Returns (page, position) of the token; page -1 if it writes nothing.
// The token's input rows are loaded together with its sequence and position,
// before the page lookup that depends on them.
__device__ __forceinline__ int2 write_token(const AppendArgs &a, int tok, int lane) {
  const int s = a.tok_seq[tok], p = a.tok_pos[tok];
  const uint4 *ks = a.k_new + (size_t)tok * a.kv_vec;
  const uint4 *vs = a.v_new + (size_t)tok * a.kv_vec;
  const uint4 *xs = a.x_new + (size_t)tok * a.x_vec;
  constexpr int U = 2;  // 16-byte vectors of K (and of V) held per lane: Hkv*D <= 512
  uint4 kr[U], vr[U], xr = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int i = lane + 32 * u;
    if (i < a.kv_vec) {
      kr[u] = ks[i];
      vr[u] = vs[i];
    }
  }
  if (lane < a.x_vec) xr = xs[lane];
  if (s < 0 || p < 0) return make_int2(-1, p);  // padding / synthetic entry: no write
  const int page = locate(a, s, p, lane);
  if (page < 0) return make_int2(-1, p);
  const size_t row = (size_t)page * a.P + (p % a.P);
  uint4 *kd = a.k_pool + row * a.kv_vec;
  uint4 *vd = a.v_pool + row * a.kv_vec;
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int i = lane + 32 * u;
    if (i < a.kv_vec) {
      kd[i] = kr[u];
      vd[i] = vr[u];
    }
  }
  for (int i = lane + 32 * U; i < a.kv_vec; i += 32) {  // wider rows than U vectors per lane
    kd[i] = ks[i];
    vd[i] = vs[i];
  }
  if (lane < a.x_vec) a.x_pool[row * a.x_vec + lane] = xr;
  return make_int2(page, p);
}

// Phase 2 for one token (one warp) that closes a micro-block (position p, on
// page `page`): store the block's compressed key in the side pool. The four
// indexer keys are read through L2 (phase 1 of this launch may have written
// them from other SMs).
__device__ __forceinline__ void compress_at(const AppendArgs &a, int p, int page, int lane) {
  const int slot = p % a.P;
  const uint32_t *x = reinterpret_cast<const uint32_t *>(a.x_pool) +
                      ((size_t)page * a.P + slot - 3) * (a.di / 2);
  uint32_t *out = reinterpret_cast<uint32_t *>(a.side_pool) +
                  ((size_t)page * (a.P / 4) + slot / 4) * (a.di / 2);
  const int half = a.di / 2;  // bf16 pairs per key
  for (int e = lane; e < half; e += 32) {
    const uint32_t v0 = __ldcg(x + e), v1 = __ldcg(x + half + e);
    const uint32_t v2 = __ldcg(x + 2 * half + e), v3 = __ldcg(x + 3 * half + e);
    // fp32 sum in token order, then IEEE division by 4, then RNE to bf16.
    float lo = __fadd_rn(__fadd_rn(__fadd_rn(bf16lo(v0), bf16lo(v1)), bf16lo(v2)), bf16lo(v3));
    float hi = __fadd_rn(__fadd_rn(__fadd_rn(bf16hi(v0), bf16hi(v1)), bf16hi(v2)), bf16hi(v3));
    out[e] = pack_bf16x2(__fdiv_rn(lo, 4.0f), __fdiv_rn(hi, 4.0f));
  }
}

// Phase 2 when the page has to be looked up again (separate launch).
__device__ __forceinline__ void compress_block(const AppendArgs &a, int tok, int lane) {
  const int s = a.tok_seq[tok], p = a.tok_pos[tok];
  if (s < 0 || p < 0 || (p & 3) != 3) return;
  const int page = locate(a, s, p, 32);  // errors were flagged by the first launch
  if (page < 0) return;
  compress_at(a, p, page, lane);
}

__global__ void __launch_bounds__(256) append_tokens_kernel(AppendArgs a) {
  pdl_wait();
  const int tok = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (tok < a.N) write_token(a, tok, threadIdx.x & 31);
}

__global__ void __launch_bounds__(256) append_compress_kernel(AppendArgs a) {
  pdl_wait();
  const int tok = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (tok < a.N) compress_block(a, tok, threadIdx.x & 31);
}

// Both phases in one CTA (small N, e.g. one token per sequence in decode):
// the barrier orders every phase-1 write before any phase-2 read; a warp keeps
// the position and page of its (at most SMALL_PER_WARP) tokens across it.
constexpr int SMALL_WARPS = 16;
constexpr int SMALL_PER_WARP = 8;
constexpr int SMALL_MAX_N = SMALL_PER_WARP * SMALL_WARPS;
__global__ void __launch_bounds__(SMALL_WARPS * 32, 1) append_small_kernel(AppendArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait();
  int2 pp[SMALL_PER_WARP];  // (page, position) of this warp's tokens
#pragma unroll
  for (int u = 0; u < SMALL_PER_WARP; ++u) {
    const int tok = warp + SMALL_WARPS * u;
    pp[u] = tok < a.N ? write_token(a, tok, lane) : make_int2(-1, 0);
  }
  __syncthreads();
  pdl_trigger();
#pragma unroll
  for (int u = 0; u < SMALL_PER_WARP; ++u)
    if (pp[u].x >= 0 && (pp[u].y & 3) == 3) compress_at(a, pp[u].y, pp[u].x, lane);
}

}  // namespace

cudaError_t launch_append(const qsa_dims &d, const qsa_cache &c, int N, const int32_t *tok_seq,
                          const int32_t *tok_pos, const void *k_new, const void *v_new,
                          const void *kidx_new, unsigned *err, cudaStream_t st) {
  if (N == 0) return cudaSuccess;
  AppendArgs a;
  a.tok_seq = tok_seq;
  a.tok_pos = tok_pos;
  a.k_new = static_cast<const uint4 *>(k_new);
  a.v_new = static_cast<const uint4 *>(v_new);
  a.x_new = static_cast<const uint4 *>(kidx_new);
  a.k_pool = static_cast<uint4 *>(c.k_pool);
  a.v_pool = static_cast<uint4 *>(c.v_pool);
  a.x_pool = static_cast<uint4 *>(c.kidx_pool);
  a.side_pool = static_cast<__nv_bfloat16 *>(c.side_pool);
  a.block_table = c.block_table;
  a.N = N;
  a.P = d.P;
  a.num_seqs = c.num_seqs;
  a.max_pages = c.max_pages_per_seq;
  a.num_pages = c.num_pages;
  a.kv_vec = d.Hkv * d.D / 8;
  a.x_vec = d.di / 8;
  a.di = d.di;
  a.err = err;
  if (N <= SMALL_MAX_N) return launch_pdl(append_small_kernel, 1, SMALL_WARPS * 32, 0, st, a);
  const int threads = 256, per_block = threads / 32;
  const int blocks = (N + per_block - 1) / per_block;
  cudaError_t e = launch_pdl(append_tokens_kernel, blocks, threads, 0, st, a);
  if (e != cudaSuccess) return e;
  return launch_pdl(append_compress_kernel, blocks, threads, 0, st, a);
}

}  // namespace qsa
