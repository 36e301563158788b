// qsa_sparse_decode_static: qsa_sparse_decode for callers that cannot
// allocate device memory. Its scratch is a file-scope device array of fixed
// size that lives in the library's module image, so the call needs no
// workspace argument and makes no allocation of any kind.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace qsa {
namespace {

constexpr size_t kStaticScratchBytes = (size_t)QSA_STATIC_SCRATCH_BYTES;

// Every device that loads the library holds this array until the process
// exits. All calls share it.
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of this device's array. Host code cannot pass the symbol
// itself (on the host it names a stand-in, not device memory), so the address
// is looked up once per device, with that device current.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace qsa

extern "C" qsa_status qsa_sparse_decode_static(const qsa_dims *dims, const qsa_cache *cache,
                                               int32_t B, const int32_t *seq_lens,
                                               const void *q, const int32_t *sel, int32_t k,
                                               int32_t R, float *o_part, float *lse_part,
                                               qsa_stream_t stream) {
  try {
    const size_t need = qsa_sparse_decode_workspace_size(dims, B, k, R);
    if (need > qsa::kStaticScratchBytes) {
      char msg[256];
      snprintf(msg, sizeof msg,
               "qsa_sparse_decode_static: this call needs %zu scratch bytes, more than the "
               "%zu-byte static scratch (use qsa_sparse_decode with a caller workspace)",
               need, qsa::kStaticScratchBytes);
      qsa::set_last_error(msg);
      return QSA_ERR_UNSUPPORTED;
    }
    void *scratch = nullptr;
    const cudaError_t e = qsa::scratch_address(&scratch);
    if (e != cudaSuccess) {
      char msg[256];
      snprintf(msg, sizeof msg, "qsa_sparse_decode_static: static scratch address: %s",
               cudaGetErrorString(e));
      qsa::set_last_error(msg);
      return QSA_ERR_CUDA;
    }
    // the regular entry point does every argument check
    return qsa_sparse_decode(dims, cache, B, seq_lens, q, sel, k, R, o_part, lse_part, scratch,
                             qsa::kStaticScratchBytes, stream);
  } catch (...) {
    qsa::set_last_error("qsa_sparse_decode_static: internal exception");
    return QSA_ERR_CUDA;
  }
}
