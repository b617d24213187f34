// qsa_internal.h -- launch-side interface between the C ABI (qsa_api.cu) and the
// kernels (qsa_attn.cu).  Not installed; not part of the public ABI.
#pragma once

#include <cuda.h>  // CUtensorMap
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace qsa {

constexpr int kHeadDim = 256;           // D: the only head dimension implemented
constexpr int kMaxGroup = 16;           // largest G = Hq / Hkv
#ifndef QSA_MAX_SLOTS
#define QSA_MAX_SLOTS 2240
#endif
constexpr int kMaxSlotsPerSplit = QSA_MAX_SLOTS;  // per-split slot list staged in smem
constexpr int kMinSlotsPerSplit = 128;  // the planner never makes splits narrower
constexpr int kMaxBlock = 16;           // largest block size of block selection

// Everything one launch of the fused kernel needs (passed by value).
struct FwdParams {
  const uint16_t* q;        // bf16 bits [Tq, Hq, D]
  const void* k_cache;      // [S, Hkv, D]: bf16 bits, or E4M3 codes when kv_fp8
  const void* v_cache;
  const int32_t* slot_idx;  // [Tq, W] row stride idx_stride_t
  const int32_t* width;     // [Tq] or nullptr
  uint16_t* out;            // bf16 bits [Tq, Hq, D]
  float* ws_o;              // fp32 [nsplit, Tq, Hq, D] (nsplit > 1)
  float* ws_lse;            // fp32 [nsplit, Tq, Hq] base-2 log-sum-exp (nsplit > 1)
  uint32_t* err_word;       // optional
  int64_t q_stride_t, q_stride_h;
  int64_t k_stride_s, k_stride_h;
  int64_t v_stride_s, v_stride_h;
  int64_t idx_stride_t;
  int64_t out_stride_t, out_stride_h;
  int64_t S;
  int32_t Tq, Hq, Hkv, G, W;
  int32_t nsplit;
  int32_t split_len;        // positions of the W axis per split
  uint32_t k_row_bytes;     // k_stride_s * element bytes: one slot step of K in bytes
  uint32_t v_row_bytes;     // v_stride_s * element bytes
  float scale_log2;         // scale * log2(e) (times k_scale for an E4M3 cache)
  int32_t block;            // slots named by one selected entry (1 = slot selection)
  int32_t kv_fp8;           // 1: k_cache / v_cache hold E4M3 codes
  float v_scale;            // E4M3 cache: multiplier of the normalised output
  int32_t head_major;       // 1: work units ordered KV head slowest (see kernel_order)
  int32_t num_sms;          // multiprocessors of the device (chooses the kernel shape)
  // Selected entries (slot numbers, or block numbers with block selection): an entry v is
  // valid when 0 <= v < ent_total and local when ent_lo <= v < ent_hi; the cache holds the
  // rows of the local entries, row (v - ent_lo) * block + e.  Unsharded: ent_lo = 0,
  // ent_hi = ent_total = floor(S / block); a slot-range shard [slot_lo, slot_lo + S) of a
  // cache of S_total slots: slot_lo / block, floor((slot_lo + S) / block), S_total / block.
  int32_t ent_lo;
  int32_t ent_hi;
  int32_t ent_total;
  // 1: write the normalised fp32 O and the base-2 LSE (ws_o / ws_lse layout, the call's
  // own split plan combined into one record per (t, h)) instead of bf16 out
  int32_t partial_out;
  void* part_o;             // partial_out: [Tq, Hq, D], fp32 or bf16 (rec_bf16)
  float* part_lse;          // partial_out: fp32 [Tq, Hq]
  int32_t rec_bf16;         // partial_out: the record's O is bf16 (else fp32)
  int32_t in_bf16;          // combine of gathered records: ws_o holds bf16 O (else fp32)
};

// Kernel configuration chosen for a group size G (shared by planner and launcher).
struct KernelShape {
  int ntile;        // n8 tiles covering G (1 or 2)
  int slot_lanes;   // warps along the slot axis
  int threads;
  int stage_rows;   // selected slots per pipeline stage
  int stages;
  size_t smem_bytes;
  int ctas_per_sm;  // expected residency (for the planner)
};

KernelShape kernel_shape(int G);

// Work-unit order of K1: KV head slowest when the whole K/V cache is larger than
// kHeadMajorBytes (about three quarters of B200's 126 MB L2) and one head's slice is
// smaller, so the resident CTAs keep one L2-sized slice hot; otherwise the heads of a
// query row run side by side and share its index row.
constexpr double kHeadMajorBytes = 96.0 * 1024 * 1024;
inline int32_t kernel_order_head_major(int64_t S, int32_t Hkv, int32_t kv_elem_bytes) {
  const double slice = double(S) * kHeadDim * kv_elem_bytes * 2;  // one head's K and V
  return (Hkv > 1 && slice * Hkv > kHeadMajorBytes && slice <= kHeadMajorBytes) ? 1 : 0;
}

// Enqueue the fused kernel (and the combine when nsplit > 1) on `stream`.
cudaError_t launch_sparse_prefill(const FwdParams& p, cudaStream_t stream);

// Enqueue the LSE combine of p.nsplit partial records (p.ws_o / p.ws_lse) into bf16 out,
// or into one partial record (p.part_o / p.part_lse) when p.partial_out.
cudaError_t launch_combine(const FwdParams& p, cudaStream_t stream);

size_t workspace_bytes_for(int32_t Tq, int32_t Hq, int32_t nsplit);

// Context-parallel shards: a pass that copies every row's local entries (in order, after
// the width and validity checks) to idx [Tq, W] (row stride W) and their number to
// count [Tq], so that K1 then reads only those.  Scratch: the two arrays, 256-aligned.
size_t shard_compact_bytes(int32_t Tq, int32_t W);
cudaError_t launch_shard_compact(const FwdParams& p, int32_t* idx, int32_t* count,
                                 cudaStream_t stream);

// printf-style detail for qsa_last_error_detail() on the calling host thread.
void set_error_detail(const char* fmt, ...);

// Process-unique identifier of the CUDA context current on the calling thread (the
// driver's context ID), or 0 when none is current or the driver cannot say.  Per-device
// state that lives in a context (a symbol's device address, a kernel's function
// attributes) is cached under this ID, so a device reset or a new primary context
// invalidates the cache instead of leaving stale addresses behind.
uint64_t current_context_id();

// 2-D tensor map over `rows` rows of `row_bytes` bytes (512: bf16, 256: E4M3 codes),
// `pitch` bytes apart, for tile::gather4 row gathers: a box of one 128-byte column block
// of one row, 128-byte swizzle.  Host only (the driver's encoder, looked up once).
cudaError_t encode_row_gather_map(CUtensorMap* map, const void* base, uint64_t rows,
                                  uint32_t row_bytes, uint64_t pitch);
size_t workspace_lse_offset(int32_t Tq, int32_t Hq, int32_t nsplit);

}  // namespace qsa
