// C ABI of libqsa.so: argument checks, the device error word and dispatch to
// the kernel launchers. See include/qsa.h for the contract of every call.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "launch.h"

#define QSA_VERSION_NUM 100  // 0.1.0

// Tracing: built with -DQSA_NVTX (python -m block_sparse_decode_b200.build
// --nvtx), every C-ABI call is an NVTX range named after it, so a profiler
// timeline shows which launches each call enqueued. NVTX v3 is header-only:
// without a tool attached a range costs a branch.
#ifdef QSA_NVTX
#include <nvtx3/nvToolsExt.h>
namespace {
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace
#define QSA_RANGE(name) NvtxRange qsa_nvtx_range_(name)
#else
#define QSA_RANGE(name) ((void)0)
#endif

namespace qsa {

// One error word per device (module-scope device variable, no allocation).
__device__ unsigned g_err_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned *g_err_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

thread_local std::string t_last_error;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

}  // namespace

unsigned *device_error_word(cudaError_t *status) {
  *status = cudaSuccess;
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) {
    *status = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_err_ptr[dev] == nullptr) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_err_word);
    if (e != cudaSuccess) {
      *status = e;
      return nullptr;
    }
    g_err_ptr[dev] = static_cast<unsigned *>(p);
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    g_sm_count[dev] = sms > 0 ? sms : 148;
  }
  return g_err_ptr[dev];
}

void set_last_error(const char *msg) { t_last_error = msg ? msg : ""; }

cudaError_t ensure_dynamic_smem(const void *kernel, size_t bytes) {
  struct Entry {
    const void *fn;
    int dev;
    size_t bytes;
  };
  static std::mutex mu;
  static Entry set[256];
  static int nset = 0;
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(mu);
  int slot = -1;
  for (int i = 0; i < nset; ++i)
    if (set[i].fn == kernel && set[i].dev == dev) slot = i;
  if (slot >= 0 && set[slot].bytes >= bytes) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  if (slot >= 0) {
    set[slot].bytes = bytes;
  } else if (nset < 256) {
    set[nset++] = Entry{kernel, dev, bytes};
  }
  return cudaSuccess;
}

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;  // no device: a B200's count
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm_count[dev] <= 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      (void)cudaGetLastError();
      sms = 0;
    }
    if (sms <= 0) return 148;
    g_sm_count[dev] = sms;
  }
  return g_sm_count[dev];
}

}  // namespace qsa

using namespace qsa;

namespace {

qsa_status fail(qsa_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

qsa_status ok() {
  t_last_error.clear();
  return QSA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qsa_status check_dims(const qsa_dims *d) {
  if (d == nullptr) return fail(QSA_ERR_INVALID_ARG, "dims is NULL");
  if (d->Hq <= 0 || d->Hkv <= 0 || d->D <= 0 || d->Hi <= 0 || d->di <= 0 || d->P <= 0)
    return fail(QSA_ERR_INVALID_ARG, "dims must be positive");
  if (d->Hq % d->Hkv != 0)
    return fail(QSA_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", d->Hq, d->Hkv);
  if (d->D != 128) return fail(QSA_ERR_UNSUPPORTED, "head dim D=%d unsupported (128)", d->D);
  if (d->di != 64 && d->di != 128)
    return fail(QSA_ERR_UNSUPPORTED, "indexer dim di=%d unsupported (64, 128)", d->di);
  if (d->Hi > 32) return fail(QSA_ERR_UNSUPPORTED, "indexer heads Hi=%d > 32", d->Hi);
  if (d->Hq / d->Hkv > 8)
    return fail(QSA_ERR_UNSUPPORTED, "GQA group %d > 8", d->Hq / d->Hkv);
  if (d->P % 4 != 0 || d->P > 1024)
    return fail(QSA_ERR_UNSUPPORTED, "page size P=%d must be a multiple of 4, <= 1024", d->P);
  if (!(d->scale == d->scale)) return fail(QSA_ERR_INVALID_ARG, "scale is NaN");
  return QSA_OK;
}

qsa_status check_cache(const qsa_cache *c, bool need_kv, bool need_side) {
  if (c == nullptr) return fail(QSA_ERR_INVALID_ARG, "cache is NULL");
  if (c->block_table == nullptr) return fail(QSA_ERR_INVALID_ARG, "block_table is NULL");
  if (c->num_seqs < 0 || c->max_pages_per_seq <= 0 || c->num_pages <= 0)
    return fail(QSA_ERR_INVALID_ARG, "cache sizes must be positive");
  if (need_kv && (c->k_pool == nullptr || c->v_pool == nullptr || !aligned16(c->k_pool) ||
                  !aligned16(c->v_pool)))
    return fail(QSA_ERR_INVALID_ARG, "k_pool / v_pool NULL or not 16-byte aligned");
  if (need_side && (c->kidx_pool == nullptr || c->side_pool == nullptr ||
                    !aligned16(c->kidx_pool) || !aligned16(c->side_pool)))
    return fail(QSA_ERR_INVALID_ARG, "kidx_pool / side_pool NULL or not 16-byte aligned");
  return QSA_OK;
}

qsa_status cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return ok();
  return fail(QSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define QSA_TRY(x)                      \
  do {                                  \
    qsa_status _s = (x);                \
    if (_s != QSA_OK) return _s;        \
  } while (0)

#define QSA_ERRWORD(var)                                        \
  cudaError_t _ee;                                              \
  unsigned *var = device_error_word(&_ee);                      \
  if (var == nullptr) return cuda_status(_ee, "device error word")

}  // namespace

extern "C" {

int32_t qsa_version(void) { return QSA_VERSION_NUM; }

const char *qsa_last_error(void) { return t_last_error.c_str(); }

qsa_status qsa_append(const qsa_dims *dims, const qsa_cache *cache, int32_t N,
                      const int32_t *tok_seq, const int32_t *tok_pos, const void *k_new,
                      const void *v_new, const void *kidx_new, qsa_stream_t stream) {
  QSA_RANGE("qsa_append");
  try {
    QSA_TRY(check_dims(dims));
    QSA_TRY(check_cache(cache, true, true));
    if (N < 0) return fail(QSA_ERR_INVALID_ARG, "N < 0");
    if (N > 0 && (tok_seq == nullptr || tok_pos == nullptr || k_new == nullptr ||
                  v_new == nullptr || kidx_new == nullptr))
      return fail(QSA_ERR_INVALID_ARG, "a token array is NULL");
    if (N > 0 && (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kidx_new)))
      return fail(QSA_ERR_INVALID_ARG, "k_new / v_new / kidx_new not 16-byte aligned");
    QSA_ERRWORD(err);
    return cuda_status(launch_append(*dims, *cache, N, tok_seq, tok_pos, k_new, v_new, kidx_new,
                                     err, reinterpret_cast<cudaStream_t>(stream)),
                       "qsa_append launch");
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_append: internal exception");
  }
}

qsa_status qsa_index_score(const qsa_dims *dims, const qsa_cache *cache, int32_t B,
                           const int32_t *seq_lens, const void *q_idx, const float *w,
                           float *scores, int32_t ld_scores, qsa_stream_t stream) {
  QSA_RANGE("qsa_index_score");
  try {
    QSA_TRY(check_dims(dims));
    QSA_TRY(check_cache(cache, false, true));
    if (B < 0 || B > 16384) return fail(QSA_ERR_INVALID_ARG, "B=%d outside [0, 16384]", B);
    if (B > cache->num_seqs)
      return fail(QSA_ERR_INVALID_ARG, "B=%d exceeds block_table rows %d", B, cache->num_seqs);
    if (ld_scores <= 0) return fail(QSA_ERR_INVALID_ARG, "ld_scores must be positive");
    if (B > 0 && (seq_lens == nullptr || q_idx == nullptr || w == nullptr || scores == nullptr))
      return fail(QSA_ERR_INVALID_ARG, "an argument array is NULL");
    if (B > 0 && !aligned16(q_idx)) return fail(QSA_ERR_INVALID_ARG, "q_idx not 16-byte aligned");
    QSA_ERRWORD(err);
    return cuda_status(launch_index_score(*dims, *cache, B, seq_lens, q_idx, w, scores, ld_scores,
                                          err, reinterpret_cast<cudaStream_t>(stream)),
                       "qsa_index_score launch");
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_index_score: internal exception");
  }
}

size_t qsa_topk_workspace_size(int32_t B, int32_t ld_scores, int32_t k) {
  (void)B;
  (void)ld_scores;
  (void)k;
  return 0;
}

namespace {

// qsa_topk_select's checks and launch; starts / R / wrote_starts as in
// launch_topk (the decode step's slice starts).
qsa_status topk_checked(int32_t B, const int32_t *seq_lens, const float *scores,
                        int32_t ld_scores, int32_t k, int32_t *sel, qsa_stream_t stream,
                        int32_t *starts, int R, bool *wrote_starts) {
  try {
    if (B < 0 || B > 65535) return fail(QSA_ERR_INVALID_ARG, "B=%d outside [0, 65535]", B);
    if (k < 1 || k > 4096) return fail(QSA_ERR_UNSUPPORTED, "k=%d outside [1, 4096]", k);
    if (ld_scores <= 0 || ld_scores > TOPK_CLUSTER * TOPK_MAX_KEYS_PER_CTA)
      return fail(QSA_ERR_UNSUPPORTED, "ld_scores=%d outside [1, %d]", ld_scores,
                  TOPK_CLUSTER * TOPK_MAX_KEYS_PER_CTA);
    if (B > 0 && (seq_lens == nullptr || scores == nullptr || sel == nullptr))
      return fail(QSA_ERR_INVALID_ARG, "an argument array is NULL");
    QSA_ERRWORD(err);
    return cuda_status(launch_topk(B, seq_lens, scores, ld_scores, k, sel, err,
                                   reinterpret_cast<cudaStream_t>(stream), starts, R,
                                   wrote_starts),
                       "qsa_topk_select launch");
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_topk_select: internal exception");
  }
}

}  // namespace

qsa_status qsa_topk_select(int32_t B, const int32_t *seq_lens, const float *scores,
                           int32_t ld_scores, int32_t k, int32_t *sel, void *ws, size_t ws_bytes,
                           qsa_stream_t stream) {
  QSA_RANGE("qsa_topk_select");
  (void)ws;
  (void)ws_bytes;
  return topk_checked(B, seq_lens, scores, ld_scores, k, sel, stream, nullptr, 0, nullptr);
}

size_t qsa_sparse_decode_workspace_size(const qsa_dims *dims, int32_t B, int32_t k, int32_t R) {
  return qsa_sparse_decode_mq_workspace_size(dims, B, 1, k, R);
}

size_t qsa_sparse_decode_mq_workspace_size(const qsa_dims *dims, int32_t B, int32_t Qn, int32_t k,
                                           int32_t R) {
  if (dims == nullptr || B <= 0 || Qn <= 0 || k <= 0 || R <= 0 || dims->Hkv <= 0 || dims->Hq <= 0)
    return 0;
  return decode_ws_bytes(*dims, B, Qn, k, R);
}

qsa_status qsa_sparse_decode(const qsa_dims *dims, const qsa_cache *cache, int32_t B,
                             const int32_t *seq_lens, const void *q, const int32_t *sel,
                             int32_t k, int32_t R, float *o_part, float *lse_part, void *ws,
                             size_t ws_bytes, qsa_stream_t stream) {
  QSA_RANGE("qsa_sparse_decode");
  return qsa_sparse_decode_mq(dims, cache, B, 1, seq_lens, q, sel, k, R, o_part, lse_part, ws,
                              ws_bytes, stream);
}

qsa_status qsa_sparse_decode_mq(const qsa_dims *dims, const qsa_cache *cache, int32_t B,
                                int32_t Qn, const int32_t *seq_lens, const void *q,
                                const int32_t *sel, int32_t k, int32_t R, float *o_part,
                                float *lse_part, void *ws, size_t ws_bytes,
                                qsa_stream_t stream) {
  QSA_RANGE("qsa_sparse_decode_mq");
  try {
    QSA_TRY(check_dims(dims));
    QSA_TRY(check_cache(cache, true, false));
    if (B < 0 || B > 65535) return fail(QSA_ERR_INVALID_ARG, "B=%d outside [0, 65535]", B);
    if (B > cache->num_seqs)
      return fail(QSA_ERR_INVALID_ARG, "B=%d exceeds block_table rows %d", B, cache->num_seqs);
    if (Qn < 1 || Qn > 8) return fail(QSA_ERR_UNSUPPORTED, "Qn=%d outside [1, 8]", Qn);
    if (k < 1 || k > 4096) return fail(QSA_ERR_UNSUPPORTED, "k=%d outside [1, 4096]", k);
    if (R < 1 || R > 64) return fail(QSA_ERR_UNSUPPORTED, "R=%d outside [1, 64]", R);
    if (B == 0) return ok();
    if (seq_lens == nullptr || q == nullptr || sel == nullptr || o_part == nullptr ||
        lse_part == nullptr)
      return fail(QSA_ERR_INVALID_ARG, "an argument array is NULL");
    if (!aligned16(q) || !aligned16(o_part) || !aligned16(ws))
      return fail(QSA_ERR_INVALID_ARG, "q / o_part / ws not 16-byte aligned");
    const size_t need = decode_ws_bytes(*dims, B, Qn, k, R);
    if (need > 0 && (ws == nullptr || ws_bytes < need))
      return fail(QSA_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, need);
    QSA_ERRWORD(err);
    return cuda_status(launch_sparse_decode(*dims, *cache, B, Qn, seq_lens, q, sel, k, R, o_part,
                                            lse_part, ws, err,
                                            reinterpret_cast<cudaStream_t>(stream)),
                       "qsa_sparse_decode launch");
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_sparse_decode: internal exception");
  }
}

qsa_status qsa_select_owned(int32_t B, const int32_t *sel, int32_t k, int32_t P, int32_t W,
                            int32_t r, int32_t *sel_out, qsa_stream_t stream) {
  QSA_RANGE("qsa_select_owned");
  try {
    if (B < 0 || B > 65535) return fail(QSA_ERR_INVALID_ARG, "B=%d outside [0, 65535]", B);
    if (k < 1 || k > 4096) return fail(QSA_ERR_UNSUPPORTED, "k=%d outside [1, 4096]", k);
    if (P <= 0 || P % 4 != 0) return fail(QSA_ERR_INVALID_ARG, "P=%d not a positive multiple of 4", P);
    if (W < 1 || W > 1024 || r < 0 || r >= W)
      return fail(QSA_ERR_INVALID_ARG, "rank %d of %d outside the supported range", r, W);
    if (B > 0 && (sel == nullptr || sel_out == nullptr))
      return fail(QSA_ERR_INVALID_ARG, "an argument array is NULL");
    if (B > 0 && sel == sel_out) return fail(QSA_ERR_INVALID_ARG, "sel_out must not alias sel");
    return cuda_status(launch_select_owned(sel, B, k, P, W, r, sel_out,
                                           reinterpret_cast<cudaStream_t>(stream)),
                       "qsa_select_owned launch");
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_select_owned: internal exception");
  }
}

qsa_status qsa_merge(int32_t R, int32_t B, int32_t Hq, int32_t D, const float *o_part,
                     const float *lse_part, void *out, int32_t out_is_bf16, float *lse_out,
                     qsa_stream_t stream) {
  QSA_RANGE("qsa_merge");
  try {
    if (R < 1 || R > 64) return fail(QSA_ERR_UNSUPPORTED, "R=%d outside [1, 64]", R);
    if (B < 0 || Hq <= 0 || D <= 0 || D % 4 != 0)
      return fail(QSA_ERR_INVALID_ARG, "bad B / Hq / D (D must be a positive multiple of 4)");
    if ((long long)B * Hq > (1LL << 30)) return fail(QSA_ERR_INVALID_ARG, "B*Hq too large");
    if (B == 0) return ok();
    if (o_part == nullptr || lse_part == nullptr || out == nullptr)
      return fail(QSA_ERR_INVALID_ARG, "an argument array is NULL");
    if (!aligned16(o_part) || (reinterpret_cast<uintptr_t>(out) & 7u) != 0)
      return fail(QSA_ERR_INVALID_ARG, "o_part not 16-byte / out not 8-byte aligned");
    return cuda_status(launch_merge(R, B, Hq, D, o_part, lse_part, out, out_is_bf16, lse_out,
                                    reinterpret_cast<cudaStream_t>(stream)),
                       "qsa_merge launch");
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_merge: internal exception");
  }
}

qsa_status qsa_decode_step(const qsa_dims *dims, const qsa_cache *cache, int32_t N,
                           const int32_t *tok_seq, const int32_t *tok_pos, const void *k_new,
                           const void *v_new, const void *kidx_new, int32_t B,
                           const int32_t *seq_lens, const void *q, const void *q_idx,
                           const float *w, int32_t k, int32_t R, float *scores, int32_t ld_scores,
                           int32_t *sel, float *o_part, float *lse_part, void *ws,
                           size_t ws_bytes, void *out, int32_t out_is_bf16, float *lse_out,
                           qsa_stream_t stream) {
  QSA_RANGE("qsa_decode_step");
  qsa_status st = QSA_OK;
  if (N != 0)
    st = qsa_append(dims, cache, N, tok_seq, tok_pos, k_new, v_new, kidx_new, stream);
  if (st == QSA_OK)
    st = qsa_index_score(dims, cache, B, seq_lens, q_idx, w, scores, ld_scores, stream);
  // the top-k kernel also hands the decode kernel each selection's slice
  // starts, through the end of the workspace (when it is large enough)
  int32_t *starts = nullptr;
  bool have_starts = false;
  if (st == QSA_OK && dims != nullptr && check_dims(dims) == QSA_OK && ws != nullptr &&
      aligned16(ws) && B > 0 && k >= 1 && k <= 4096 && R >= 1 && R <= 64 &&
      ws_bytes >= decode_ws_bytes(*dims, B, 1, k, R))
    starts = reinterpret_cast<int32_t *>(static_cast<char *>(ws) +
                                         decode_ws_starts_offset(*dims, B, 1, k, R));
  if (st == QSA_OK)
    st = topk_checked(B, seq_lens, scores, ld_scores, k, sel, stream, starts, R, &have_starts);
  if (st == QSA_OK) {
    // qsa_sparse_decode and qsa_merge with the merge fused into the decode's
    // combine kernel (same arithmetic as qsa_merge); both calls' checks apply
    try {
      QSA_TRY(check_dims(dims));
      QSA_TRY(check_cache(cache, true, false));
      if (B < 0 || B > 65535) return fail(QSA_ERR_INVALID_ARG, "B=%d outside [0, 65535]", B);
      if (B > cache->num_seqs)
        return fail(QSA_ERR_INVALID_ARG, "B=%d exceeds block_table rows %d", B, cache->num_seqs);
      if (k < 1 || k > 4096) return fail(QSA_ERR_UNSUPPORTED, "k=%d outside [1, 4096]", k);
      if (R < 1 || R > 64) return fail(QSA_ERR_UNSUPPORTED, "R=%d outside [1, 64]", R);
      if (B == 0) return ok();
      if (seq_lens == nullptr || q == nullptr || sel == nullptr || o_part == nullptr ||
          lse_part == nullptr || out == nullptr)
        return fail(QSA_ERR_INVALID_ARG, "an argument array is NULL");
      if (!aligned16(q) || !aligned16(o_part) || !aligned16(ws) ||
          (reinterpret_cast<uintptr_t>(out) & 7u) != 0)
        return fail(QSA_ERR_INVALID_ARG, "q / o_part / ws not 16-byte or out not 8-byte aligned");
      const size_t need = decode_ws_bytes(*dims, B, 1, k, R);
      if (need > 0 && (ws == nullptr || ws_bytes < need))
        return fail(QSA_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, need);
      QSA_ERRWORD(err);
      st = cuda_status(launch_sparse_decode(*dims, *cache, B, 1, seq_lens, q, sel, k, R, o_part,
                                            lse_part, ws, err,
                                            reinterpret_cast<cudaStream_t>(stream), nullptr, 0,
                                            out, out_is_bf16, lse_out,
                                            have_starts ? starts : nullptr),
                       "qsa_decode_step decode + merge launch");
    } catch (...) {
      return fail(QSA_ERR_CUDA, "qsa_decode_step: internal exception");
    }
  }
  return st;
}

size_t qsa_prefill_index_score_workspace_size(const qsa_dims *dims, int32_t S, int32_t Nq) {
  if (dims == nullptr || S < 0 || Nq < 0 || !prefill_supported(*dims)) return 0;
  return prefill_plan_ws_bytes(*dims, S, Nq);
}

qsa_status qsa_prefill_index_score(const qsa_dims *dims, const qsa_cache *cache, int32_t S,
                                   const int32_t *seq_lens, const int32_t *row_start, int32_t Nq,
                                   const void *q_idx, const float *w, float *scores,
                                   int32_t ld_scores, int32_t *row_len, void *ws,
                                   size_t ws_bytes, qsa_stream_t stream) {
  QSA_RANGE("qsa_prefill_index_score");
  try {
    QSA_TRY(check_dims(dims));
    QSA_TRY(check_cache(cache, false, true));
    if (S < 0 || S > cache->num_seqs)
      return fail(QSA_ERR_INVALID_ARG, "S=%d outside [0, block_table rows %d]", S,
                  cache->num_seqs);
    if (Nq < 0 || Nq > 65535) return fail(QSA_ERR_INVALID_ARG, "Nq=%d outside [0, 65535]", Nq);
    if (ld_scores <= 0) return fail(QSA_ERR_INVALID_ARG, "ld_scores must be positive");
    if (!prefill_supported(*dims))
      return fail(QSA_ERR_UNSUPPORTED,
                  "qsa_prefill_index_score needs Hi in {4, 8, 16, 32} and the page size P a "
                  "multiple of 32");
    if (S == 0 || Nq == 0) return ok();
    if (seq_lens == nullptr || row_start == nullptr || q_idx == nullptr || w == nullptr ||
        scores == nullptr || row_len == nullptr || ws == nullptr)
      return fail(QSA_ERR_INVALID_ARG, "an argument array is NULL");
    if (!aligned16(q_idx) || !aligned16(ws))
      return fail(QSA_ERR_INVALID_ARG, "q_idx / ws not 16-byte aligned");
    const size_t need = prefill_plan_ws_bytes(*dims, S, Nq);
    if (ws_bytes < need)
      return fail(QSA_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, need);
    QSA_ERRWORD(err);
    return cuda_status(launch_prefill_index_score(*dims, *cache, S, seq_lens, row_start, Nq,
                                                  q_idx, w, scores, ld_scores, row_len, ws, err,
                                                  reinterpret_cast<cudaStream_t>(stream)),
                       "qsa_prefill_index_score launch");
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_prefill_index_score: internal exception");
  }
}

qsa_status qsa_prefill_sparse_decode(const qsa_dims *dims, const qsa_cache *cache, int32_t S,
                                     const int32_t *seq_lens, const int32_t *row_start,
                                     int32_t Nq, const void *q, const int32_t *sel, int32_t k,
                                     int32_t R, float *o_part, float *lse_part, void *ws,
                                     size_t ws_bytes, qsa_stream_t stream) {
  QSA_RANGE("qsa_prefill_sparse_decode");
  try {
    QSA_TRY(check_dims(dims));
    QSA_TRY(check_cache(cache, true, false));
    if (S < 0 || S > cache->num_seqs)
      return fail(QSA_ERR_INVALID_ARG, "S=%d outside [0, block_table rows %d]", S,
                  cache->num_seqs);
    if (Nq < 0 || Nq > 65535) return fail(QSA_ERR_INVALID_ARG, "Nq=%d outside [0, 65535]", Nq);
    if (k < 1 || k > 4096) return fail(QSA_ERR_UNSUPPORTED, "k=%d outside [1, 4096]", k);
    if (R < 1 || R > 64) return fail(QSA_ERR_UNSUPPORTED, "R=%d outside [1, 64]", R);
    if (S == 0 || Nq == 0) return ok();
    if (seq_lens == nullptr || row_start == nullptr || q == nullptr || sel == nullptr ||
        o_part == nullptr || lse_part == nullptr)
      return fail(QSA_ERR_INVALID_ARG, "an argument array is NULL");
    if (!aligned16(q) || !aligned16(o_part) || !aligned16(ws))
      return fail(QSA_ERR_INVALID_ARG, "q / o_part / ws not 16-byte aligned");
    const size_t need = decode_ws_bytes(*dims, Nq, 1, k, R);
    if (need > 0 && (ws == nullptr || ws_bytes < need))
      return fail(QSA_ERR_INVALID_ARG, "workspace %zu bytes < %zu needed", ws_bytes, need);
    QSA_ERRWORD(err);
    return cuda_status(launch_sparse_decode(*dims, *cache, Nq, 1, seq_lens, q, sel, k, R, o_part,
                                            lse_part, ws, err,
                                            reinterpret_cast<cudaStream_t>(stream), row_start, S),
                       "qsa_prefill_sparse_decode launch");
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_prefill_sparse_decode: internal exception");
  }
}

namespace {
size_t align256(size_t x) { return (x + 255) / 256 * 256; }
}  // namespace

size_t qsa_sparse_prefill_workspace_size(const qsa_dims *dims, int32_t S, int32_t Nq, int32_t k,
                                         int32_t R) {
  if (dims == nullptr || S < 0 || Nq <= 0 || k <= 0 || R <= 0 || dims->Hkv <= 0 ||
      dims->Hq <= 0 || !prefill_supported(*dims))
    return 0;
  return align256(prefill_plan_ws_bytes(*dims, S, Nq)) + decode_ws_bytes(*dims, Nq, 1, k, R);
}

qsa_status qsa_sparse_prefill(const qsa_dims *dims, const qsa_cache *cache, int32_t S,
                              const int32_t *seq_lens, const int32_t *row_start, int32_t Nq,
                              const void *q, const void *q_idx, const float *w, int32_t k,
                              int32_t R, float *scores, int32_t ld_scores, int32_t *row_len,
                              int32_t *sel, float *o_part, float *lse_part, void *ws,
                              size_t ws_bytes, void *out, int32_t out_is_bf16, float *lse_out,
                              qsa_stream_t stream) {
  QSA_RANGE("qsa_sparse_prefill");
  if (dims == nullptr) return fail(QSA_ERR_INVALID_ARG, "dims is NULL");
  if (S < 0 || Nq < 0) return fail(QSA_ERR_INVALID_ARG, "S or Nq negative");
  if (S == 0 || Nq == 0) return ok();
  if (!prefill_supported(*dims))
    return fail(QSA_ERR_UNSUPPORTED, "qsa_sparse_prefill needs Hi in {4, 8, 16, 32}");
  const size_t plan = align256(prefill_plan_ws_bytes(*dims, S, Nq));
  if (ws == nullptr || ws_bytes < plan)
    return fail(QSA_ERR_INVALID_ARG, "workspace of %zu bytes is too small", ws_bytes);
  unsigned char *wd = static_cast<unsigned char *>(ws) + plan;
  qsa_status st = qsa_prefill_index_score(dims, cache, S, seq_lens, row_start, Nq, q_idx, w,
                                          scores, ld_scores, row_len, ws, plan, stream);
  if (st == QSA_OK)
    st = qsa_topk_select(Nq, row_len, scores, ld_scores, k, sel, nullptr, 0, stream);
  if (st == QSA_OK)
    st = qsa_prefill_sparse_decode(dims, cache, S, seq_lens, row_start, Nq, q, sel, k, R, o_part,
                                   lse_part, wd, ws_bytes - plan, stream);
  if (st == QSA_OK)
    st = qsa_merge(R, Nq, dims->Hq, dims->D, o_part, lse_part, out, out_is_bf16, lse_out, stream);
  return st;
}

qsa_status qsa_check_device_errors(qsa_stream_t stream, int32_t *flags) {
  QSA_RANGE("qsa_check_device_errors");
  try {
    if (flags) *flags = 0;
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_status(e, "stream synchronize");
    QSA_ERRWORD(err);
    (void)err;
    unsigned v = 0;
    e = cudaMemcpyFromSymbol(&v, g_err_word, sizeof v);
    if (e != cudaSuccess) return cuda_status(e, "read error word");
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_err_word, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_status(e, "clear error word");
    if (flags) *flags = (int32_t)v;
    if (v & ~ERR_TIMEOUT) return fail(QSA_ERR_BOUNDS, "device index check failed (flags 0x%x)", v);
    if (v & ERR_TIMEOUT) return fail(QSA_ERR_TIMEOUT, "device wait timed out (flags 0x%x)", v);
    return ok();
  } catch (...) {
    return fail(QSA_ERR_CUDA, "qsa_check_device_errors: internal exception");
  }
}

}  // extern "C"
