// Internal host-side launchers of the QSA kernels (not part of the C ABI).
// Each returns the cudaError_t of its launch(es); argument checks happen in
// abi.cu before any of these is called.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/qsa.h"

namespace qsa {

// Launch `kern` as a programmatic dependent of the previous kernel on the
// stream (see pdl_wait / pdl_trigger in common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// Raise a kernel's dynamic shared memory limit to at least `bytes` on the
// current device; the driver is called only when the limit has to grow.
cudaError_t ensure_dynamic_smem(const void *kernel, size_t bytes);

// Device address of this device's error word (set up once per device).
unsigned *device_error_word(cudaError_t *status);
int device_sm_count();
void set_last_error(const char *msg);  // message returned by qsa_last_error()

cudaError_t launch_append(const qsa_dims &d, const qsa_cache &c, int N, const int32_t *tok_seq,
                          const int32_t *tok_pos, const void *k_new, const void *v_new,
                          const void *kidx_new, unsigned *err, cudaStream_t st);

bool index_score_supported(const qsa_dims &d);  // page sizes the TMA gather can address
// Scores through warp-level MMAs for any page size P (a multiple of 4).
cudaError_t launch_index_score_warp(const qsa_dims &d, const qsa_cache &c, int B,
                                    const int32_t *seq_lens, const void *q_idx, const float *w,
                                    float *scores, int ld, unsigned *err, cudaStream_t st);
cudaError_t launch_index_score(const qsa_dims &d, const qsa_cache &c, int B,
                               const int32_t *seq_lens, const void *q_idx, const float *w,
                               float *scores, int ld, unsigned *err, cudaStream_t st);

constexpr int TOPK_CLUSTER = 8;
constexpr int TOPK_MAX_KEYS_PER_CTA = 49152;  // 192 KiB of keys per CTA
// Top-k runs one cluster of 8 or 4 CTAs per sequence, the larger size whose
// clusters all stay resident; when neither is (e.g. 128 sequences, 256
// prefill rows), one CTA per sequence from this many sequences on, for score
// rows of at most TOPK_ROW_MAX_KEYS blocks (2 bytes each in shared memory).
// Measured: 8 rows take 13.9 us in clusters of 8 and 44.8 us one CTA each;
// 64 rows of up to 65,536 blocks 28.9 us in clusters of 4 and 30.7 us one
// CTA each; 256 rows 140 us in clusters of 8 and 57 us one CTA each.
constexpr int TOPK_ROW_MIN_B = 64;
constexpr int TOPK_ROW_MAX_KEYS = 65536;
// starts (may be nullptr): [B, R + 1] slice starts of each selection for the
// decode step (st[r] = selected blocks below floor(r nb / R)); *wrote_starts
// tells whether the chosen kernel wrote them (the one-CTA-per-row kernel does
// not).
cudaError_t launch_topk(int B, const int32_t *seq_lens, const float *scores, int ld, int k,
                        int32_t *sel, unsigned *err, cudaStream_t st, int32_t *starts = nullptr,
                        int R = 0, bool *wrote_starts = nullptr);

size_t decode_ws_bytes(const qsa_dims &d, int B, int Qn, int k, int R);
// Offset of the [B, R + 1] int slice starts at the end of that workspace,
// which the decode step's top-k kernel writes for its decode kernel.
size_t decode_ws_starts_offset(const qsa_dims &d, int B, int Qn, int k, int R);
// row_start != nullptr: B prefill rows of S chunks (sequence s holds rows
// [row_start[s], row_start[s+1]), seq_lens[s] counts its chunk), Qn = 1.
// m_out != nullptr (Qn = 1): the R partials are also merged into m_out
// [B, Hq, D] (bf16 if m_bf16) and m_lse [B, Hq], by the combine kernel's last
// CTA per row group (or the merge kernel when no sequence is split).
cudaError_t launch_sparse_decode(const qsa_dims &d, const qsa_cache &c, int B, int Qn,
                                 const int32_t *seq_lens, const void *q, const int32_t *sel,
                                 int k, int R, float *o_part, float *lse_part, void *ws,
                                 unsigned *err, cudaStream_t st,
                                 const int32_t *row_start = nullptr, int S = 0,
                                 void *m_out = nullptr, int m_bf16 = 0, float *m_lse = nullptr,
                                 const int32_t *starts = nullptr);

cudaError_t launch_select_owned(const int32_t *sel, int B, int k, int P, int W, int r,
                                int32_t *out, cudaStream_t st);

// Sparse prefill scoring (prefill.cu): query rows of appended chunks, groups
// of prefill_group_rows(d) rows of one sequence sharing each side-cache tile.
bool prefill_supported(const qsa_dims &d);
int prefill_group_rows(const qsa_dims &d);
size_t prefill_plan_ws_bytes(const qsa_dims &d, int S, int Nq);
cudaError_t launch_prefill_index_score(const qsa_dims &d, const qsa_cache &c, int S,
                                       const int32_t *seq_lens, const int32_t *row_start, int Nq,
                                       const void *q_idx, const float *w, float *scores, int ld,
                                       int32_t *row_len, void *ws, unsigned *err,
                                       cudaStream_t st);

cudaError_t launch_merge(int R, int B, int Hq, int D, const float *o_part, const float *lse_part,
                         void *out, int out_is_bf16, float *lse_out, cudaStream_t st);

}  // namespace qsa
