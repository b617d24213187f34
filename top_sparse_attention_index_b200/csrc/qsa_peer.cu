// qsa_peer.cu -- the context-parallel combine over records addressed one pointer each
// (this device's memory or peer memory mapped with CUDA IPC), and the IPC helpers.
// Entry points: include/qsa_peer.h.
#include <cuda.h>  // driver types of the address-range query (resolved at run time)
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "qsa_internal.h"
#include "qsa_peer.h"
#include "qsa_ptx.cuh"

namespace {

using qsa::bf16hi_to_f32;
using qsa::bf16lo_to_f32;
using qsa::fast_exp2;
using qsa::pack_bf16x2;

constexpr float kNegInfP = -__builtin_huge_valf();
constexpr int kPeerUnroll = 8;  // records whose rows a warp has in flight at once

struct PeerParams {
  const void* rec_o[QSA_MAX_PEERS];
  const float* rec_lse[QSA_MAX_PEERS];
  uint16_t* out[QSA_MAX_PEERS];
  int64_t out_stride_t, out_stride_h;
  int32_t R, n_out, Hq, t0, t1;
};

// One warp per (t, h) of the rows [t0, t1): lane r < R reads record r's lse, the warp
// reduces their maximum, then every lane adds its eight elements of D over the records in
// order (weight 2^(lse_r - max)), the rows of up to kPeerUnroll records in flight at once
// (each read regardless of its weight; a record with lse = -inf is left out by a select),
// and stores the normalised row as bf16 to every output.  The arithmetic is the same, in
// the same order, as the combine of stacked records.
template <bool IN_BF16>
__global__ void __launch_bounds__(128)
    qsa_peer_combine_kernel(const __grid_constant__ PeerParams p) {
  const int64_t rows = int64_t(p.t1 - p.t0) * p.Hq;
  const int64_t i = int64_t(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (i >= rows) return;
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(p.t0) * p.Hq + i;  // (t, h) row of the records
  const int64_t t = row / p.Hq, h = row % p.Hq;
  const float lse_l = lane < p.R ? p.rec_lse[lane][row] : kNegInfP;
  // lane r holds record r's row address; the loop takes it with a shuffle
  const unsigned long long o_l =
      lane < p.R ? reinterpret_cast<unsigned long long>(p.rec_o[lane]) +
                       static_cast<unsigned long long>(row) * qsa::kHeadDim * (IN_BF16 ? 2 : 4)
                 : 0ull;
  float mstar = lse_l;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, off));
  float res[8];
  if (mstar == kNegInfP) {  // no valid slot in any record
#pragma unroll
    for (int e = 0; e < 8; ++e) res[e] = 0.f;
  } else {
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    float wsum = 0.f;
#pragma unroll kPeerUnroll
    for (int r = 0; r < p.R; ++r) {
      const float lse = __shfl_sync(0xffffffffu, lse_l, r);
      const unsigned long long rowp = __shfl_sync(0xffffffffu, o_l, r);
      float x[8];
      if constexpr (IN_BF16) {
        const uint4 v = *(reinterpret_cast<const uint4*>(rowp) + lane);
        x[0] = bf16lo_to_f32(v.x); x[1] = bf16hi_to_f32(v.x);
        x[2] = bf16lo_to_f32(v.y); x[3] = bf16hi_to_f32(v.y);
        x[4] = bf16lo_to_f32(v.z); x[5] = bf16hi_to_f32(v.z);
        x[6] = bf16lo_to_f32(v.w); x[7] = bf16hi_to_f32(v.w);
      } else {
        const float4* src = reinterpret_cast<const float4*>(rowp) + 2 * lane;
        const float4 a = src[0], b = src[1];
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
      }
      if (lse != kNegInfP) {  // warp-uniform
        const float w = fast_exp2(lse - mstar);
        wsum += w;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += w * x[e];
      }
    }
    const float inv = 1.f / wsum;
#pragma unroll
    for (int e = 0; e < 8; ++e) res[e] = acc[e] * inv;
  }
  uint4 v;
  v.x = pack_bf16x2(res[0], res[1]);
  v.y = pack_bf16x2(res[2], res[3]);
  v.z = pack_bf16x2(res[4], res[5]);
  v.w = pack_bf16x2(res[6], res[7]);
  for (int k = 0; k < p.n_out; ++k)
    *reinterpret_cast<uint4*>(p.out[k] + t * p.out_stride_t + h * p.out_stride_h + lane * 8) = v;
}

bool aligned(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; }

qsa_status_t bad(qsa_status_t st, const char* what) {
  qsa::set_error_detail("%s", what);
  return st;
}

// (also clears the runtime's last-error state, so that a refused IPC call is not reported
// again by the next launch's error check)
qsa_status_t cuda_fail(const char* where, cudaError_t e) {
  qsa::set_error_detail("%s: %s", where, cudaGetErrorString(e));
  (void)cudaGetLastError();
  return QSA_ERR_CUDA;
}

// cuMemGetAddressRange through the runtime's driver entry-point query (no link-time
// dependency on libcuda), looked up once per process.
using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
AddressRangeFn address_range_fn() {
  static const AddressRangeFn fn = []() -> AddressRangeFn {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult r{};
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault,
                                         &r) != cudaSuccess ||
        r != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<AddressRangeFn>(f);
  }();
  return fn;
}

}  // namespace

extern "C" {

qsa_status_t qsa_combine_peer_records(const void* const* rec_o, const float* const* rec_lse,
                                      int32_t R, int32_t record_bf16, int32_t Tq, int32_t Hq,
                                      int32_t D, int32_t t0, int32_t t1, void* const* out,
                                      int32_t n_out, int64_t out_stride_t, int64_t out_stride_h,
                                      void* stream) {
  qsa::set_error_detail("");
  if (record_bf16 != 0 && record_bf16 != 1)
    return bad(QSA_ERR_INVALID_ARG, "record_bf16 must be 0 or 1");
  if (R < 1 || R > QSA_MAX_PEERS || n_out < 1 || n_out > QSA_MAX_PEERS)
    return bad(QSA_ERR_INVALID_ARG, "R and n_out must lie in [1, QSA_MAX_PEERS]");
  if (Tq < 0 || Hq < 1 || t0 < 0 || t0 > t1 || t1 > Tq)
    return bad(QSA_ERR_INVALID_ARG, "bad sizes: need Tq >= 0, Hq >= 1, 0 <= t0 <= t1 <= Tq");
  if (D != qsa::kHeadDim) return bad(QSA_ERR_UNSUPPORTED, "head dimension (only 256)");
  if (out_stride_t < 0 || out_stride_h < 0 || out_stride_t % 8 != 0 || out_stride_h % 8 != 0)
    return bad(QSA_ERR_INVALID_ARG, "out strides must be non-negative multiples of 8 elements");
  if (rec_o == nullptr || rec_lse == nullptr || out == nullptr)
    return bad(QSA_ERR_INVALID_ARG, "NULL pointer array");
  PeerParams p{};
  for (int r = 0; r < R; ++r) {
    if (rec_o[r] == nullptr || rec_lse[r] == nullptr || !aligned(rec_o[r], 16) ||
        !aligned(rec_lse[r], 4))
      return bad(QSA_ERR_INVALID_ARG, "record pointers must be non-NULL, O 16-byte and lse 4-byte aligned");
    p.rec_o[r] = rec_o[r];
    p.rec_lse[r] = rec_lse[r];
  }
  for (int k = 0; k < n_out; ++k) {
    if (out[k] == nullptr || !aligned(out[k], 16))
      return bad(QSA_ERR_INVALID_ARG, "output pointers must be non-NULL and 16-byte aligned");
    p.out[k] = static_cast<uint16_t*>(out[k]);
  }
  const int64_t rows = int64_t(t1 - t0) * Hq;
  if (rows == 0) return QSA_OK;
  if (rows > int64_t(INT32_MAX) * 4) return bad(QSA_ERR_INVALID_ARG, "too many rows for one launch");
  p.R = R;
  p.n_out = n_out;
  p.Hq = Hq;
  p.t0 = t0;
  p.t1 = t1;
  p.out_stride_t = out_stride_t;
  p.out_stride_h = out_stride_h;
  const unsigned grid = static_cast<unsigned>((rows + 3) / 4);
  auto st = static_cast<cudaStream_t>(stream);
  if (record_bf16)
    qsa_peer_combine_kernel<true><<<grid, 128, 0, st>>>(p);
  else
    qsa_peer_combine_kernel<false><<<grid, 128, 0, st>>>(p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? QSA_OK : cuda_fail("qsa_combine_peer_records: launch", e);
}

qsa_status_t qsa_ipc_export(const void* ptr, void* handle, uint64_t* offset) {
  qsa::set_error_detail("");
  if (ptr == nullptr || handle == nullptr || offset == nullptr)
    return bad(QSA_ERR_INVALID_ARG, "qsa_ipc_export: NULL argument");
  static_assert(sizeof(cudaIpcMemHandle_t) == QSA_IPC_HANDLE_BYTES, "IPC handle size");
  const AddressRangeFn range = address_range_fn();
  if (range == nullptr) return bad(QSA_ERR_CUDA, "qsa_ipc_export: cuMemGetAddressRange unavailable");
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS)
    return bad(QSA_ERR_CUDA, "qsa_ipc_export: not device memory of the current context");
  cudaIpcMemHandle_t h{};
  const cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return cuda_fail("qsa_ipc_export", e);
  std::memcpy(handle, &h, sizeof h);
  *offset = static_cast<uint64_t>(reinterpret_cast<CUdeviceptr>(ptr) - base);
  return QSA_OK;
}

qsa_status_t qsa_ipc_import(const void* handle, void** base) {
  qsa::set_error_detail("");
  if (handle == nullptr || base == nullptr)
    return bad(QSA_ERR_INVALID_ARG, "qsa_ipc_import: NULL argument");
  cudaIpcMemHandle_t h{};
  std::memcpy(&h, handle, sizeof h);
  const cudaError_t e = cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess);
  return e == cudaSuccess ? QSA_OK : cuda_fail("qsa_ipc_import", e);
}

qsa_status_t qsa_ipc_close(void* base) {
  qsa::set_error_detail("");
  if (base == nullptr) return bad(QSA_ERR_INVALID_ARG, "qsa_ipc_close: NULL base");
  const cudaError_t e = cudaIpcCloseMemHandle(base);
  return e == cudaSuccess ? QSA_OK : cuda_fail("qsa_ipc_close", e);
}

}  // extern "C"
