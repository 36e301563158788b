// Device helpers shared by the tensor-core scoring kernels (decode and
// prefill): mbarriers with bounded waits, TMA tile loads, tcgen05 MMA issue,
// commit and TMEM loads, the partial-block score on CUDA cores, and the host
// lookup of cuTensorMapEncodeTiled.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace qsa {

constexpr uint32_t TC_SPIN_LIMIT = 1u << 22;  // try_wait rounds before giving up
constexpr uint32_t TC_DRAIN_LIMIT = 1u << 20;

// Failure injection for the decode scoring kernel, read at each launch from
// the environment variable QSA_DEBUG_STALL_SCORE: when it is "1", the
// producer warps issue no copy (a barrier that nothing completes) and the
// roles' waits give up after TC_STALL_LIMIT rounds. This exercises the
// timeout path (the TIMEOUT bit, the drain, the release of TMEM) on a real
// GPU without faulting or hanging anything; unset, it costs one getenv.
constexpr uint32_t TC_STALL_LIMIT = 1024;
bool debug_stall_score();

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.b32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; on timeout (or once another role gave up) returns false. The
// drain after an abort passes honor_abort = false: it must still wait for its
// own copies and MMAs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned *err, uint32_t limit = TC_SPIN_LIMIT,
                                          bool honor_abort = true) {
  for (uint32_t i = 0; i < limit; ++i) {
    if (mbar_try(bar, parity)) return true;
    if (honor_abort && (i & 255u) == 255u && *abort_flag) return false;
  }
  *abort_flag = 1;
  raise_err(err, ERR_TIMEOUT);
  return false;
}
__device__ __forceinline__ void mbar_arrive_expect(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival counts toward the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 columns of TMEM without waiting; tc_wait_ld() makes them usable.
__device__ __forceinline__ void tc_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Score of the trailing partial block of a query whose context is the first
// L tokens of the sequence with block-table row bt_row (whole warp; every
// lane returns it). The key is the bf16-rounded mean of its L mod 4 indexer
// keys, built exactly as the side cache builds complete blocks; q_rows holds
// the query's Hi <= HMAX indexer rows of DI elements, w_row its Hi head
// weights. It runs while the memory system streams at full load, where each
// dependent round trip costs microseconds, so it makes two: the query rows
// and weights are asked into L1 first (one 128-byte line per lane), the up to
// 3 key rows are loaded together once the page id is known, and the per-head
// loop then reads the query from L1. Same operations in the same order as
// before, so the score is the same bits.
template <int DI, int HMAX = 32>
__device__ float partial_block_score_row(const __nv_bfloat16 *kidx_pool, int P,
                                         const int32_t *bt_row, int max_pages, int num_pages,
                                         int L, const __nv_bfloat16 *q_rows, const float *w_row,
                                         int Hi, unsigned *err, bool *ok_out) {
  const int lane = threadIdx.x & 31;
  const int nfull = L >> 2, n = L - 4 * nfull, pos = 4 * nfull;
  const int col = pos / P;
  constexpr int QLINES = HMAX * DI * 2 / 128;  // 128-byte lines of HMAX query rows
#pragma unroll
  for (int l = lane; l < QLINES; l += 32)
    if (l * 128 < Hi * DI * 2)
      asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const char *>(q_rows) + l * 128));
  if (lane == 0) asm volatile("prefetch.global.L1 [%0];" ::"l"(w_row));
  int page = -1;
  if (col < max_pages) page = bt_row[col];
  const bool ok = page >= 0 && page < num_pages;
  *ok_out = ok;
  if (!ok) {
    if (lane == 0) raise_err(err, col < max_pages ? ERR_PAGE : ERR_BT);
    return 0.f;
  }
  const uint32_t *x = reinterpret_cast<const uint32_t *>(kidx_pool) +
                      ((size_t)page * P + pos % P) * (DI / 2);
  uint32_t xv[3][DI / 64];
#pragma unroll
  for (int u = 0; u < 3; ++u)
#pragma unroll
    for (int i = 0; i < DI / 64; ++i) xv[u][i] = u < n ? x[u * (DI / 2) + lane + 32 * i] : 0u;
  float klo[DI / 64], khi[DI / 64];
#pragma unroll
  for (int i = 0; i < DI / 64; ++i) {
    float lo = bf16lo(xv[0][i]), hi = bf16hi(xv[0][i]);
#pragma unroll
    for (int u = 1; u < 3; ++u) {
      if (u < n) {
        lo = __fadd_rn(lo, bf16lo(xv[u][i]));
        hi = __fadd_rn(hi, bf16hi(xv[u][i]));
      }
    }
    const uint32_t kc = pack_bf16x2(__fdiv_rn(lo, (float)n), __fdiv_rn(hi, (float)n));
    klo[i] = bf16lo(kc);
    khi[i] = bf16hi(kc);
  }
  float score = 0.f;
#pragma unroll 4
  for (int h = 0; h < Hi; ++h) {
    const uint32_t *qrow = reinterpret_cast<const uint32_t *>(q_rows + (size_t)h * DI);
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < DI / 64; ++i) {
      const uint32_t q = qrow[lane + 32 * i];
      part = fmaf(klo[i], bf16lo(q), part);
      part = fmaf(khi[i], bf16hi(q), part);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    score = fmaf(w_row[h], fmaxf(part, 0.f), score);
  }
  return score;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver (no link-time libcuda dependency).
EncodeTiledFn encode_tiled_fn(cudaError_t *status);

}  // namespace qsa
