// qsa_api.cu -- the C ABI of libqsa.so: argument validation, the split planner and the
// launch.  Declarations and the full contract are in include/qsa.h.
//
// The host side never synchronises and never allocates: every check below uses only
// the scalar arguments and pointer values, so a call is a pure enqueue on `stream`
// (unlike the Ascend adapter described in "What the pull request actually adds",
// whose extent check copies two scalars to the host).
#include <cuda.h>  // driver types of the context-ID query (resolved at run time)
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>

#include "qsa.h"
#include "qsa_internal.h"

namespace {

thread_local char g_detail[512] = "";

qsa_status_t fail(qsa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_detail, sizeof g_detail, fmt, ap);
  va_end(ap);
  return st;
}

struct Plan {
  int32_t nsplit;
  int32_t split_len;
  size_t workspace;
};

// Shape validation shared by the planner and the launch; returns QSA_OK or an error.
qsa_status_t check_block(int32_t block) {
  if (block < 1 || block > qsa::kMaxBlock)
    return fail(QSA_ERR_INVALID_ARG, "block size %d outside 1..%d", block, qsa::kMaxBlock);
  return QSA_OK;
}

qsa_status_t check_shape(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int32_t W) {
  if (Tq < 0 || W < 0) return fail(QSA_ERR_INVALID_ARG, "negative size: Tq=%d W=%d", Tq, W);
  if (Hq <= 0 || Hkv <= 0 || D <= 0)
    return fail(QSA_ERR_INVALID_ARG, "non-positive size: Hq=%d Hkv=%d D=%d", Hq, Hkv, D);
  if (Hq % Hkv != 0) return fail(QSA_ERR_INVALID_ARG, "Hq=%d is not a multiple of Hkv=%d", Hq, Hkv);
  if (D != qsa::kHeadDim) return fail(QSA_ERR_UNSUPPORTED, "head dimension %d (only 256)", D);
  const int32_t G = Hq / Hkv;
  if (G > qsa::kMaxGroup) return fail(QSA_ERR_UNSUPPORTED, "group size G=%d (1..16)", G);
  return QSA_OK;
}

// Splits of the W axis.  One split's slots (entries x block) must fit the shared-memory
// offset list; with fewer work units than one wave of CTAs, more splits fill that wave
// but none is narrower than kMinSlotsPerSplit slots.
Plan make_plan(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t W, int32_t block, int32_t num_sms,
               int32_t request) {
  const int32_t G = Hq / Hkv;
  const int32_t per_split_max = qsa::kMaxSlotsPerSplit / block;  // entries
  const int32_t min_split = W > 0 ? (W + per_split_max - 1) / per_split_max : 1;
  const int32_t max_split = W > 0 ? W : 1;
  int32_t n;
  if (request > 0) {
    n = request < min_split ? min_split : (request > max_split ? max_split : request);
  } else {
    // Fewer work units than one wave of CTAs: split W until the CTAs fill (at most) one
    // wave -- more splits cost more than the extra parallelism gives (measured on
    // decode-shape batches); never splits narrower than kMinSlotsPerSplit.
    const qsa::KernelShape ks = qsa::kernel_shape(G);
    const int64_t wave = int64_t(num_sms > 0 ? num_sms : 1) * ks.ctas_per_sm;
    const int64_t units = int64_t(Tq) * Hkv;
    n = min_split;
    if (units > 0 && units < wave) {
      const int64_t want = wave / units;
      const int64_t min_entries = (qsa::kMinSlotsPerSplit + block - 1) / block;
      const int64_t cap = W >= min_entries ? W / min_entries : 1;
      const int64_t pick = want < cap ? want : cap;
      if (pick > n) n = int32_t(pick);
    }
  }
  int32_t split_len = W > 0 ? (W + n - 1) / n : 0;
  if (W > 0) n = (W + split_len - 1) / split_len;  // no split lies wholly past W
  return {n, split_len, qsa::workspace_bytes_for(Tq, Hq, n)};
}

int32_t device_sm_count(int dev) {
  static std::atomic<int32_t> cache[64];
  if (dev >= 0 && dev < 64) {
    const int32_t c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64) cache[dev].store(sms, std::memory_order_relaxed);
  return sms;
}

// A context-parallel shard (a slot range smaller than the whole cache) with an unsplit
// plan first compacts every row's local entries, so the fused kernel does not scan the
// whole global selection for the few entries it holds (measured at the long-prefill shape:
// one of 8 shards 360 vs 447 us, one of 4 597 vs 660 us, the compaction pass aside).
constexpr int32_t kCompactMinW = 32;
bool shard_compaction(int32_t nsplit, int64_t S, int64_t S_total, int32_t W) {
  return nsplit == 1 && S < S_total && W >= kCompactMinW;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool stride_ok(int64_t s) { return s >= 0 && (s % 8) == 0; }

}  // namespace

namespace qsa {
// Lets other translation units of the library report a detail for their own errors.
void set_error_detail(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(g_detail, sizeof g_detail, fmt, ap);
  va_end(ap);
}

// The two driver entry points are looked up through the runtime once per process, so the
// library needs no link-time dependency on libcuda.
uint64_t current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  struct Fns {
    GetCurrentFn get_current = nullptr;
    GetIdFn get_id = nullptr;
  };
  static const Fns fns = [] {
    Fns f;
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult ra{}, rb{};
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &a, 12000, cudaEnableDefault, &ra) ==
            cudaSuccess &&
        ra == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &b, 12000, cudaEnableDefault, &rb) ==
            cudaSuccess &&
        rb == cudaDriverEntryPointSuccess) {
      f.get_current = reinterpret_cast<GetCurrentFn>(a);
      f.get_id = reinterpret_cast<GetIdFn>(b);
    }
    return f;
  }();
  if (fns.get_current == nullptr || fns.get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (fns.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (fns.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(id);
}
}  // namespace qsa

extern "C" {

int32_t qsa_abi_version(void) { return 2; }

const char* qsa_status_string(qsa_status_t status) {
  switch (status) {
    case QSA_OK: return "QSA_OK";
    case QSA_ERR_INVALID_ARG: return "QSA_ERR_INVALID_ARG";
    case QSA_ERR_UNSUPPORTED: return "QSA_ERR_UNSUPPORTED";
    case QSA_ERR_WORKSPACE: return "QSA_ERR_WORKSPACE";
    case QSA_ERR_CUDA: return "QSA_ERR_CUDA";
  }
  return "QSA_ERR_UNKNOWN";
}

const char* qsa_last_error_detail(void) { return g_detail; }

int32_t qsa_sparse_prefill_block_plan(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int32_t W,
                                      int32_t block, int32_t num_sms, int32_t nsplit_request,
                                      size_t* workspace_bytes) {
  qsa_status_t st = check_shape(Tq, Hq, Hkv, D, W);
  if (st == QSA_OK) st = check_block(block);
  if (st != QSA_OK) return -int32_t(st);
  if (nsplit_request < 0) return -int32_t(fail(QSA_ERR_INVALID_ARG, "negative nsplit request"));
  const Plan pl = make_plan(Tq, Hq, Hkv, W, block, num_sms, nsplit_request);
  if (workspace_bytes != nullptr) *workspace_bytes = pl.workspace;
  return pl.nsplit;
}

int32_t qsa_sparse_prefill_plan(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int32_t W,
                                int32_t num_sms, int32_t nsplit_request,
                                size_t* workspace_bytes) {
  return qsa_sparse_prefill_block_plan(Tq, Hq, Hkv, D, W, 1, num_sms, nsplit_request,
                                       workspace_bytes);
}

int32_t qsa_sparse_prefill_partial_plan(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int32_t W,
                                        int32_t block, int64_t S, int64_t S_total,
                                        int32_t num_sms, int32_t nsplit_request,
                                        size_t* workspace_bytes) {
  size_t ws = 0;
  const int32_t n =
      qsa_sparse_prefill_block_plan(Tq, Hq, Hkv, D, W, block, num_sms, nsplit_request, &ws);
  if (n < 0) return n;
  if (S < 0 || S_total < S)
    return -int32_t(fail(QSA_ERR_INVALID_ARG, "S %lld and S_total %lld: need 0 <= S <= S_total",
                         (long long)S, (long long)S_total));
  if (shard_compaction(n, S, S_total, W)) ws = qsa::shard_compact_bytes(Tq, W);
  if (workspace_bytes != nullptr) *workspace_bytes = ws;
  return n;
}

size_t qsa_sparse_prefill_workspace_bytes(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t W,
                                          int32_t D, int32_t num_sms) {
  size_t bytes = 0;
  if (qsa_sparse_prefill_plan(Tq, Hq, Hkv, D, W, num_sms, 0, &bytes) < 0) return SIZE_MAX;
  return bytes;
}

}  // extern "C"

namespace {

// Slot-range shard and partial output of prefill_impl (context parallel).
struct PartialArgs {
  int64_t slot_lo = 0;
  int64_t S_total = -1;  // -1: S (unsharded)
  void* part_o = nullptr;
  float* part_lse = nullptr;  // both set: write one normalised record + base-2 LSE
  bool rec_bf16 = false;      // the record's O in bf16 (else fp32)
};

// The body shared by every launching entry point.  kv_fp8: k_cache / v_cache hold E4M3
// codes (one byte per element, strides multiples of 16) dequantised with k_scale and
// v_scale; otherwise bf16 (strides multiples of 8 elements) and the scales are 1.
qsa_status_t prefill_impl(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                          const void* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                          const void* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                          const int32_t* slot_idx, int64_t idx_stride_t, const int32_t* width,
                          int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int64_t S, int32_t W,
                          int32_t block, float scale, bool kv_fp8, float k_scale, float v_scale,
                          void* out, int64_t out_stride_t, int64_t out_stride_h, int32_t nsplit,
                          void* workspace, size_t workspace_bytes, uint32_t* err_word,
                          void* stream, const PartialArgs& part = PartialArgs()) {
  g_detail[0] = '\0';
  qsa_status_t st = check_shape(Tq, Hq, Hkv, D, W);
  if (st == QSA_OK) st = check_block(block);
  if (st != QSA_OK) return st;
  if (S < 0) return fail(QSA_ERR_INVALID_ARG, "negative S");
  if (nsplit < 0) return fail(QSA_ERR_INVALID_ARG, "negative nsplit");
  if (!std::isfinite(scale)) return fail(QSA_ERR_INVALID_ARG, "scale is not finite");
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale))
    return fail(QSA_ERR_INVALID_ARG, "k_scale or v_scale is not finite");
  const bool partial = part.part_o != nullptr || part.part_lse != nullptr;
  const int64_t S_total = part.S_total < 0 ? S : part.S_total;
  if (part.slot_lo < 0 || (S > 0 && part.slot_lo % block != 0))
    return fail(QSA_ERR_INVALID_ARG, "slot_lo %lld must be a non-negative multiple of block %d",
                (long long)part.slot_lo, block);
  if (S_total < part.slot_lo + S)
    return fail(QSA_ERR_INVALID_ARG, "S_total %lld below slot_lo + S = %lld", (long long)S_total,
                (long long)(part.slot_lo + S));
  if (S_total > int64_t(INT32_MAX) * block)
    return fail(QSA_ERR_UNSUPPORTED, "S_total beyond the int32 selection range");
  if (Tq == 0) return QSA_OK;

  // (an empty shard, S == 0, reads no cache row and may pass NULL caches)
  if (q == nullptr || (S > 0 && (k_cache == nullptr || v_cache == nullptr)) ||
      (!partial && out == nullptr))
    return fail(QSA_ERR_INVALID_ARG, "NULL q, k_cache, v_cache or out");
  if (partial && (part.part_o == nullptr || part.part_lse == nullptr))
    return fail(QSA_ERR_INVALID_ARG, "NULL part_o or part_lse");
  if (partial && (!aligned16(part.part_o) || !aligned4(part.part_lse)))
    return fail(QSA_ERR_INVALID_ARG, "part_o must be 16-byte and part_lse 4-byte aligned");
  if (W > 0 && slot_idx == nullptr) return fail(QSA_ERR_INVALID_ARG, "NULL slot_idx with W > 0");
  // (in partial mode `out` is not used: the record buffers take its place)
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || (!partial && !aligned16(out)))
    return fail(QSA_ERR_INVALID_ARG, "q, k_cache, v_cache and out must be 16-byte aligned");
  if ((slot_idx != nullptr && !aligned4(slot_idx)) || (width != nullptr && !aligned4(width)) ||
      (err_word != nullptr && !aligned4(err_word)))
    return fail(QSA_ERR_INVALID_ARG, "slot_idx, width and err_word must be 4-byte aligned");
  if (!stride_ok(q_stride_t) || !stride_ok(q_stride_h) || !stride_ok(out_stride_t) ||
      !stride_ok(out_stride_h))
    return fail(QSA_ERR_INVALID_ARG, "q and out strides must be non-negative multiples of 8 elements");
  // K / V strides: 16 bytes = 8 bf16 elements or 16 E4M3 codes.
  const int64_t kv_elem = kv_fp8 ? 1 : 2;
  const auto kv_stride_ok = [&](int64_t x) { return x >= 0 && (x * kv_elem) % 16 == 0; };
  if (!kv_stride_ok(k_stride_s) || !kv_stride_ok(k_stride_h) || !kv_stride_ok(v_stride_s) ||
      !kv_stride_ok(v_stride_h))
    return fail(QSA_ERR_INVALID_ARG, "k_cache / v_cache strides must be non-negative multiples of %d elements",
                int(16 / kv_elem));
  if (idx_stride_t < 0) return fail(QSA_ERR_INVALID_ARG, "negative idx_stride_t");
  // The kernels step from slot to slot by a 32-bit byte stride.
  if (uint64_t(k_stride_s) * kv_elem > UINT32_MAX || uint64_t(v_stride_s) * kv_elem > UINT32_MAX)
    return fail(QSA_ERR_UNSUPPORTED, "slot stride of 4 GiB or more");

  // the multiprocessor count sizes the automatic split plan (and, below, the kernel shape)
  auto query_sms = [](int32_t& sms) -> qsa_status_t {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    sms = device_sm_count(dev);
    if (sms <= 0) return fail(QSA_ERR_CUDA, "cannot query the multiprocessor count");
    return QSA_OK;
  };
  int32_t num_sms = 0;
  if (nsplit == 0) {
    const qsa_status_t st = query_sms(num_sms);
    if (st != QSA_OK) return st;
  }
  const Plan pl = make_plan(Tq, Hq, Hkv, W, block, num_sms, nsplit);
  if (int64_t(Tq) * Hkv * pl.nsplit > int64_t(INT32_MAX))
    return fail(QSA_ERR_INVALID_ARG, "too many work units for one launch");
  if (pl.workspace > 0) {
    if (workspace == nullptr || workspace_bytes < pl.workspace)
      return fail(QSA_ERR_WORKSPACE, "workspace of %zu bytes needed for nsplit=%d, got %zu",
                  pl.workspace, pl.nsplit, workspace == nullptr ? size_t(0) : workspace_bytes);
    if (!aligned16(workspace)) return fail(QSA_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  }

  if (num_sms == 0) {  // every argument is valid: only now touch the device
    const qsa_status_t st = query_sms(num_sms);
    if (st != QSA_OK) return st;
  }
  qsa::FwdParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.slot_idx = slot_idx;
  p.width = width;
  p.out = static_cast<uint16_t*>(out);
  p.ws_o = static_cast<float*>(workspace);
  p.ws_lse = pl.workspace > 0
                 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                            qsa::workspace_lse_offset(Tq, Hq, pl.nsplit))
                 : nullptr;
  p.err_word = err_word;
  p.q_stride_t = q_stride_t;
  p.q_stride_h = q_stride_h;
  p.k_stride_s = k_stride_s;
  p.k_stride_h = k_stride_h;
  p.v_stride_s = v_stride_s;
  p.v_stride_h = v_stride_h;
  p.idx_stride_t = idx_stride_t;
  p.out_stride_t = out_stride_t;
  p.out_stride_h = out_stride_h;
  p.S = S;
  p.Tq = Tq;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.W = W;
  p.nsplit = pl.nsplit;
  p.split_len = pl.split_len;
  p.k_row_bytes = uint32_t(k_stride_s * kv_elem);
  p.v_row_bytes = uint32_t(v_stride_s * kv_elem);
  // log2(e): the kernels use 2^x; an E4M3 cache's k_scale multiplies every score
  p.scale_log2 = kv_fp8 ? scale * k_scale * 1.4426950408889634f : scale * 1.4426950408889634f;
  p.block = block;
  p.kv_fp8 = kv_fp8 ? 1 : 0;
  p.v_scale = kv_fp8 ? v_scale : 1.0f;
  p.head_major = qsa::kernel_order_head_major(S, Hkv, int32_t(kv_elem));
  p.num_sms = num_sms;
  p.ent_lo = int32_t(part.slot_lo / block);
  p.ent_hi = int32_t((part.slot_lo + S) / block);
  p.ent_total = int32_t(S_total / block);
  if (partial) {
    p.partial_out = 1;
    p.part_o = part.part_o;
    p.part_lse = part.part_lse;
    p.rec_bf16 = part.rec_bf16 ? 1 : 0;
    if (pl.nsplit == 1) {  // the single split's record is the partial record itself
      p.ws_o = part.rec_bf16 ? nullptr : static_cast<float*>(part.part_o);
      p.ws_lse = part.part_lse;
    }
  }

  // a shard with room for the compaction in its workspace: compact each row's local
  // entries first and run the fused kernel on them (the same entries in the same order,
  // so the same result bit for bit)
  if (partial && shard_compaction(pl.nsplit, S, S_total, W) && workspace != nullptr &&
      aligned16(workspace) && workspace_bytes >= qsa::shard_compact_bytes(Tq, W)) {
    int32_t* cidx = static_cast<int32_t*>(workspace);
    int32_t* ccount = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) +
                                                 (size_t(Tq) * size_t(W) * 4 + 255) / 256 * 256);
    cudaError_t e = qsa::launch_shard_compact(p, cidx, ccount, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
    p.slot_idx = cidx;
    p.idx_stride_t = W;
    p.width = ccount;
  }

  const cudaError_t e = qsa::launch_sparse_prefill(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  return QSA_OK;
}

}  // namespace

extern "C" {

qsa_status_t qsa_sparse_prefill_block(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                                      const void* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                                      const void* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                                      const int32_t* slot_idx, int64_t idx_stride_t,
                                      const int32_t* width, int32_t Tq, int32_t Hq, int32_t Hkv,
                                      int32_t D, int64_t S, int32_t W, int32_t block, float scale,
                                      void* out, int64_t out_stride_t, int64_t out_stride_h,
                                      int32_t nsplit, void* workspace, size_t workspace_bytes,
                                      uint32_t* err_word, void* stream) {
  return prefill_impl(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache,
                      v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S, W,
                      block, scale, false, 1.0f, 1.0f, out, out_stride_t, out_stride_h, nsplit,
                      workspace, workspace_bytes, err_word, stream);
}

qsa_status_t qsa_sparse_prefill_partial(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                                        const void* k_cache, int64_t k_stride_s,
                                        int64_t k_stride_h, const void* v_cache,
                                        int64_t v_stride_s, int64_t v_stride_h,
                                        const int32_t* slot_idx, int64_t idx_stride_t,
                                        const int32_t* width, int32_t Tq, int32_t Hq, int32_t Hkv,
                                        int32_t D, int64_t S, int32_t W, int32_t block,
                                        int64_t slot_lo, int64_t S_total, int32_t kv_fp8,
                                        float scale, float k_scale, float v_scale, void* part_o,
                                        float* part_lse, int32_t record_bf16, int32_t nsplit,
                                        void* workspace, size_t workspace_bytes,
                                        uint32_t* err_word, void* stream) {
  if (kv_fp8 != 0 && kv_fp8 != 1) return fail(QSA_ERR_INVALID_ARG, "kv_fp8 must be 0 or 1");
  if (record_bf16 != 0 && record_bf16 != 1)
    return fail(QSA_ERR_INVALID_ARG, "record_bf16 must be 0 or 1");
  PartialArgs part;
  part.slot_lo = slot_lo;
  part.S_total = S_total;
  part.part_o = part_o;
  part.part_lse = part_lse;
  part.rec_bf16 = record_bf16 != 0;
  if (Tq > 0 && (part_o == nullptr || part_lse == nullptr)) {
    g_detail[0] = '\0';
    return fail(QSA_ERR_INVALID_ARG, "NULL part_o or part_lse");
  }
  if (S_total < 0) return fail(QSA_ERR_INVALID_ARG, "negative S_total");
  return prefill_impl(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache,
                      v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S, W,
                      block, scale, kv_fp8 != 0, kv_fp8 ? k_scale : 1.0f, kv_fp8 ? v_scale : 1.0f,
                      nullptr, 0, 0, nsplit, workspace, workspace_bytes, err_word, stream, part);
}

qsa_status_t qsa_combine_partials(const void* part_o, const float* part_lse, int32_t record_bf16,
                                  int32_t R, int32_t Tq, int32_t Hq, int32_t D, void* out,
                                  int64_t out_stride_t, int64_t out_stride_h, void* stream) {
  g_detail[0] = '\0';
  if (record_bf16 != 0 && record_bf16 != 1)
    return fail(QSA_ERR_INVALID_ARG, "record_bf16 must be 0 or 1");
  if (R < 1 || Tq < 0 || Hq < 1)
    return fail(QSA_ERR_INVALID_ARG, "bad sizes: R=%d Tq=%d Hq=%d", R, Tq, Hq);
  if (D != qsa::kHeadDim) return fail(QSA_ERR_UNSUPPORTED, "head dimension %d (only 256)", D);
  if (Tq == 0) return QSA_OK;
  if (part_o == nullptr || part_lse == nullptr || out == nullptr)
    return fail(QSA_ERR_INVALID_ARG, "NULL part_o, part_lse or out");
  if (!aligned16(part_o) || !aligned4(part_lse) || !aligned16(out))
    return fail(QSA_ERR_INVALID_ARG, "part_o and out must be 16-byte, part_lse 4-byte aligned");
  if (!stride_ok(out_stride_t) || !stride_ok(out_stride_h))
    return fail(QSA_ERR_INVALID_ARG, "out strides must be non-negative multiples of 8 elements");
  if (int64_t(Tq) * Hq > int64_t(INT32_MAX) * 4)
    return fail(QSA_ERR_INVALID_ARG, "too many rows for one launch");
  qsa::FwdParams p{};
  p.ws_o = static_cast<float*>(const_cast<void*>(part_o));
  p.ws_lse = const_cast<float*>(part_lse);
  p.in_bf16 = record_bf16;
  p.out = static_cast<uint16_t*>(out);
  p.out_stride_t = out_stride_t;
  p.out_stride_h = out_stride_h;
  p.Tq = Tq;
  p.Hq = Hq;
  p.nsplit = R;
  const cudaError_t e = qsa::launch_combine(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QSA_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  return QSA_OK;
}

qsa_status_t qsa_sparse_prefill_fp8kv(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                                      const void* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                                      const void* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                                      const int32_t* slot_idx, int64_t idx_stride_t,
                                      const int32_t* width, int32_t Tq, int32_t Hq, int32_t Hkv,
                                      int32_t D, int64_t S, int32_t W, int32_t block, float scale,
                                      float k_scale, float v_scale, void* out,
                                      int64_t out_stride_t, int64_t out_stride_h, int32_t nsplit,
                                      void* workspace, size_t workspace_bytes,
                                      uint32_t* err_word, void* stream) {
  return prefill_impl(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache,
                      v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S, W,
                      block, scale, true, k_scale, v_scale, out, out_stride_t, out_stride_h, nsplit,
                      workspace, workspace_bytes, err_word, stream);
}

qsa_status_t qsa_sparse_prefill(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                                const void* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                                const void* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                                const int32_t* slot_idx, int64_t idx_stride_t,
                                const int32_t* width, int32_t Tq, int32_t Hq, int32_t Hkv,
                                int32_t D, int64_t S, int32_t W, float scale, void* out,
                                int64_t out_stride_t, int64_t out_stride_h, int32_t nsplit,
                                void* workspace, size_t workspace_bytes, uint32_t* err_word,
                                void* stream) {
  return qsa_sparse_prefill_block(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h,
                                  v_cache, v_stride_s, v_stride_h, slot_idx, idx_stride_t, width,
                                  Tq, Hq, Hkv, D, S, W, 1, scale, out, out_stride_t, out_stride_h,
                                  nsplit, workspace, workspace_bytes, err_word, stream);
}

}  // extern "C"
