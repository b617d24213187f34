// qsa_noalloc.cu -- qsa_sparse_prefill_noalloc: the sparse-prefill entry point for
// callers that cannot allocate device memory (declared in include/qsa.h).
//
// Who needs it: a serving runtime that gives every free byte of HBM to its KV-cache
// pool at start-up and bans cudaMalloc afterwards, a plugin whose host framework owns
// the allocator and offers no hook into it, or code that must not allocate while a
// stream is being captured.  Such a caller can still pass its inputs and outputs, but
// not the workspace that splitting the selection width (nsplit > 1) needs.  Here that
// scratch is a file-scope device array of fixed size that lives as long as the
// process, on every GPU that loads the library.  Nothing in this file allocates.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "qsa.h"
#include "qsa_internal.h"

namespace {

// The shared scratch: fp32 split partials and base-2 log-sum-exp values.  Host code
// must never pass `g_static_scratch` itself to a kernel: on the host that name is only
// a stand-in for the symbol, not a device address.  The address comes from
// cudaGetSymbolAddress, once per device (and again after the device's context changes).
static __device__ __align__(256) unsigned char g_static_scratch[QSA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Per device: the context the address was looked up in (its process-unique ID) and the
// address.  A device reset or any new context on the device changes the ID, and the next
// call looks the address up again instead of reusing one that is no longer mapped.
struct ScratchSlot {
  uint64_t ctx_id = 0;
  void* addr = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array in the context current on the calling thread:
// looked up with cudaGetSymbolAddress on the first call per device (with that device
// current) and again whenever the device's context has changed since; cached otherwise.
qsa_status_t scratch_address(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    qsa::set_error_detail("cudaGetDevice: %s", cudaGetErrorString(e));
    return QSA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    qsa::set_error_detail("device ordinal %d is beyond the %d devices this entry point serves",
                          dev, kMaxDevices);
    return QSA_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchSlot& slot = g_scratch[dev];
  const uint64_t ctx = qsa::current_context_id();
  if (ctx == 0 || slot.addr == nullptr || slot.ctx_id != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr) {
      qsa::set_error_detail("cudaGetSymbolAddress of the static scratch on device %d: %s", dev,
                            cudaGetErrorString(e));
      return QSA_ERR_CUDA;
    }
    // (the lookup makes the device's context current if nothing had before)
    slot.ctx_id = qsa::current_context_id();
    slot.addr = p;
  }
  *addr = slot.addr;
  return QSA_OK;
}

}  // namespace

extern "C" qsa_status_t qsa_sparse_prefill_noalloc(
    const void* q, int64_t q_stride_t, int64_t q_stride_h, const void* k_cache,
    int64_t k_stride_s, int64_t k_stride_h, const void* v_cache, int64_t v_stride_s,
    int64_t v_stride_h, const int32_t* slot_idx, int64_t idx_stride_t, const int32_t* width,
    int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int64_t S, int32_t W, float scale, void* out,
    int64_t out_stride_t, int64_t out_stride_h, int32_t nsplit, uint32_t* err_word,
    void* stream) {
  if (nsplit < 0) {
    qsa::set_error_detail("negative nsplit");
    return QSA_ERR_INVALID_ARG;
  }
  // The split count this call will use: the automatic plan needs the SM count of the
  // current device (a host-side attribute query, no allocation).
  int32_t num_sms = 0;
  if (nsplit == 0 && Tq > 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) {
      qsa::set_error_detail("multiprocessor count query: %s", cudaGetErrorString(e));
      return QSA_ERR_CUDA;
    }
  }
  size_t need = 0;
  const int32_t planned = qsa_sparse_prefill_plan(Tq, Hq, Hkv, D, W, num_sms, nsplit, &need);
  if (planned < 0) return static_cast<qsa_status_t>(-planned);  // detail already set
  if (need > QSA_STATIC_SCRATCH_BYTES) {
    qsa::set_error_detail(
        "this shape needs %zu bytes of split scratch (nsplit=%d) but the static scratch holds "
        "%zu; request fewer splits or use qsa_sparse_prefill with a workspace",
        need, planned, static_cast<size_t>(QSA_STATIC_SCRATCH_BYTES));
    return QSA_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0) {
    const qsa_status_t st = scratch_address(&scratch);
    if (st != QSA_OK) return st;
  }
  return qsa_sparse_prefill(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache,
                            v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D,
                            S, W, scale, out, out_stride_t, out_stride_h, planned, scratch,
                            need > 0 ? static_cast<size_t>(QSA_STATIC_SCRATCH_BYTES) : 0,
                            err_word, stream);
}
