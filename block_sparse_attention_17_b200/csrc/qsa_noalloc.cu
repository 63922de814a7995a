// qsa_decode_noalloc: the decode step with its scratch in a file-scope device
// array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory for scratch: a host program whose
// own allocator owns all of the GPU's memory and hands none out to libraries,
// or a latency-critical loop that must never call cudaMalloc (which can
// synchronise the device). For them this entry point runs the same kernels as
// qsa_decode with the scratch taken from kScratchBytes of device memory that
// the library declares statically; every GPU that loads the library holds this
// array until the process exits.
#include <stdio.h>

#include <mutex>

#include "qsa_common.cuh"
#include "qsa_kernels.h"

namespace {

constexpr size_t kScratchBytes = 4u << 20;   // 4 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" qsa_status qsa_decode_noalloc(const qsa_config* cfg, int batch, int n_q, int cap,
                                         const int32_t* kv_len, const void* q,
                                         const void* k_cache, const void* v_cache,
                                         const void* iq, const void* ik_cache, const float* iw,
                                         const void* gate, float* pooled_cache, void* out,
                                         float* lse, int32_t* sel, int32_t* nsel,
                                         int32_t* dev_err, void* stream) {
  char msg[256];
  const size_t need = qsa_decode_workspace_size(cfg, batch, n_q, cap);
  if (need == 0) {
    // an empty batch, or a geometry qsa_decode rejects and explains
    return qsa_decode(cfg, batch, n_q, cap, kv_len, q, k_cache, v_cache, iq, ik_cache, iw,
                      gate, pooled_cache, out, lse, sel, nsel, dev_err, nullptr, 0, stream);
  }
  if (need > kScratchBytes) {
    snprintf(msg, sizeof(msg),
             "qsa_decode_noalloc: this geometry needs %zu bytes of scratch, more than the "
             "%zu-byte static scratch; use qsa_decode with a workspace",
             need, kScratchBytes);
    qsa::set_last_error(msg);
    return QSA_ERR_WORKSPACE;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "qsa_decode_noalloc: no usable current device (%s)",
             cudaGetErrorString(e));
    qsa::set_last_error(msg);
    return QSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof(msg),
             "qsa_decode_noalloc: device ordinal %d is beyond the %d devices it serves", dev,
             kMaxDevices);
    qsa::set_last_error(msg);
    return QSA_ERR_UNSUPPORTED;
  }
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
      // host code only sees a stand-in for the array: its device address is
      // looked up once per device, with that device current
      e = cudaGetSymbolAddress(&g_scratch_ptr[dev], g_decode_scratch);
      if (e != cudaSuccess) {
        g_scratch_ptr[dev] = nullptr;
        snprintf(msg, sizeof(msg), "qsa_decode_noalloc: cudaGetSymbolAddress: %s",
                 cudaGetErrorString(e));
        qsa::set_last_error(msg);
        return QSA_ERR_CUDA;
      }
    }
    ptr = g_scratch_ptr[dev];
  }
  return qsa_decode(cfg, batch, n_q, cap, kv_len, q, k_cache, v_cache, iq, ik_cache, iw, gate,
                    pooled_cache, out, lse, sel, nsel, dev_err, ptr, kScratchBytes, stream);
}
