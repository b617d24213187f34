/*
 * qsa.h -- C ABI of the B200 (sm_100a) Top-K-selected sparse attention library
 * used for QSA prefill (libqsa.so).
 *
 * Source of the operation: the article "Qwen4-Exp QSA comes to Huawei's Ascend:
 * inside SGLang's opt-in CANN prefill PR" (orcarouter.ai blog).
 *   - section "What the pull request actually adds": attention over already-rotated
 *     Q and K, scale * Q K^T, softmax, times V (the packed-embedding paragraph); the
 *     original head-dim-256 scale is kept; unordered physical slots with -1 padding;
 *     fully masked rows keep the zero-output convention; supported local head shapes
 *     (16,2), (24,2), (12,1), (6,1), (3,1); BF16 with head dimension 256.
 *   - section "Nine tests that passed, and a speed number that did not come from this
 *     branch": unordered physical slots at widths 1/63/64/65/2051, default and explicit
 *     scales, fully masked rows, zero selection width, non-contiguous tensors, an FP32
 *     CPU reference from the same BF16 inputs, and the long-prefill case
 *     (7,810 queries x 2,051 selected slots over a 65,536-slot cache).
 *   - section "Why QSA is the awkward part, in numbers": sparse block size 1 (one
 *     selected slot is one token) and the untouched selected-token interface.
 *
 * What one call computes.  Let G = Hq / Hkv.  For every query row t in [0, Tq) and
 * every query head h in [0, Hq), with KV head j = floor(h / G):
 *
 *   V_t   = { slot_idx[t, w] : 0 <= w < width[t], slot_idx[t, w] != -1 }   (a multiset)
 *   s_i   = scale * sum_d q[t, h, d] * k_cache[V_t[i], j, d]
 *   p_i   = exp(s_i - max_i s_i),  l = sum_i p_i
 *   out[t, h, :] = sum_i p_i * v_cache[V_t[i], j, :] / l,      or exactly +0 if V_t is empty.
 *
 * The order of the slots in a row does not matter; -1 may appear anywhere inside the
 * first width[t] entries and is skipped; entries at w >= width[t] are never read.
 *
 * Conventions shared by every entry point:
 *   - All tensors are bf16 (q, k_cache, v_cache, out) or int32 (slot_idx, width) in
 *     DEVICE memory, owned by the caller.  The library allocates nothing, never
 *     synchronises the stream or the device, and only enqueues work on `stream`.
 *   - Strides are in ELEMENTS of the tensor's own type.  The innermost (d) stride is 1.
 *     q is [Tq, Hq, D], k_cache / v_cache are [S, Hkv, D], out is [Tq, Hq, D],
 *     slot_idx is [Tq, W] (row stride idx_stride_t, column stride 1), width is [Tq]
 *     contiguous.
 *   - Only D == 256 and 1 <= G <= 16 are implemented (QSA_ERR_UNSUPPORTED otherwise).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).
 */
#ifndef QSA_H_
#define QSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point. */
typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = 1, /* a NULL required pointer, a negative size, Hq % Hkv != 0,
                              a misaligned base or stride, a NaN/Inf scale, too small a
                              workspace for the requested split count                */
  QSA_ERR_UNSUPPORTED = 2, /* D != 256, or G = Hq / Hkv outside 1..16                    */
  QSA_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than the plan requires          */
  QSA_ERR_CUDA = 4         /* a CUDA runtime call or a kernel launch failed             */
} qsa_status_t;

/* Bits that the kernels OR into *err_word (device memory, optional). */
#define QSA_ERRBIT_SLOT_RANGE 0x1u /* a slot index outside [-1, S) was seen; it was masked */
#define QSA_ERRBIT_WIDTH_RANGE 0x2u /* a width[t] outside [0, W] was seen; it was clamped   */
#define QSA_ERRBIT_Q_RANGE 0x4u     /* fp8-KV entry point only: a query element with
                                       |q| >= 65536 (beyond the f16 range the fp8-KV
                                       products run in); that row's output is not valid  */

/* Largest number of selected positions one split processes (the per-split index list
 * is staged whole in shared memory).  Wider selections are split automatically. */
#define QSA_MAX_SLOTS_PER_SPLIT 2240

/* Version of this ABI; bumped on any signature change. */
int32_t qsa_abi_version(void);

/*
 * qsa_sparse_prefill_plan -- host-only planner (no CUDA call, no device access).
 *
 * Returns the number of W-splits `nsplit` that qsa_sparse_prefill will use for this
 * shape and writes the matching workspace size in bytes to *workspace_bytes (may be
 * NULL).  nsplit_request == 0 asks for the automatic choice for a device with
 * `num_sms` multiprocessors; nsplit_request > 0 forces that count (it is raised to
 * the minimum that keeps every split within QSA_MAX_SLOTS_PER_SPLIT positions and
 * lowered to at most W).  With nsplit == 1 no workspace is needed (0 bytes).
 * With nsplit > 1 the workspace holds fp32 partial outputs [nsplit, Tq, Hq, D] and
 * base-2 log-sum-exp values [nsplit, Tq, Hq], each region 256-byte aligned.
 * Returns a negative qsa_status_t value (e.g. -QSA_ERR_INVALID_ARG) when the shape
 * itself is invalid or unsupported.
 */
int32_t qsa_sparse_prefill_plan(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int32_t W,
                                int32_t num_sms, int32_t nsplit_request,
                                size_t* workspace_bytes);

/*
 * qsa_sparse_prefill_workspace_bytes -- workspace size of the automatic plan.
 *
 * Host only, like qsa_sparse_prefill_plan, of which it is the nsplit_request == 0 case
 * with the arguments in the order (Tq, Hq, Hkv, W, D, num_sms): the bytes of device
 * scratch that qsa_sparse_prefill with nsplit == 0 needs on a device of `num_sms`
 * multiprocessors (0 when the plan does not split W).  Returns SIZE_MAX when the shape
 * is invalid or unsupported (qsa_last_error_detail() says why).
 */
size_t qsa_sparse_prefill_workspace_bytes(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t W,
                                          int32_t D, int32_t num_sms);

/*
 * qsa_sparse_prefill -- selected-slot sparse attention for one prefill batch.
 *
 * Arguments (all device pointers unless stated):
 *   q            bf16 [Tq, Hq, D], strides (q_stride_t, q_stride_h, 1).  Already rotated.
 *   k_cache      bf16 [S, Hkv, D], strides (k_stride_s, k_stride_h, 1).  Already rotated.
 *   v_cache      bf16 [S, Hkv, D], strides (v_stride_s, v_stride_h, 1).
 *   slot_idx     int32 [Tq, W], row stride idx_stride_t.  Unordered physical slots;
 *                -1 = masked.  Any other value outside [0, S) is masked as well and sets
 *                QSA_ERRBIT_SLOT_RANGE in *err_word.
 *   width        int32 [Tq] selection width per row, or NULL meaning W for every row.
 *                Values outside [0, W] are clamped and set QSA_ERRBIT_WIDTH_RANGE
 *                (the host cannot see device values without a synchronisation).
 *   Tq, Hq, Hkv, D, S, W   sizes; Tq == 0 is a no-op returning QSA_OK; W == 0 writes
 *                exact zeros.
 *   scale        multiplier of Q K^T (1/sqrt(256) = 1/16 keeps the original scale).
 *   out          bf16 [Tq, Hq, D], strides (out_stride_t, out_stride_h, 1).  Written in
 *                full (rows with no valid slot get +0.0).  Must not alias the inputs.
 *   nsplit       0 = automatic (the planner's choice for the current device), else the
 *                requested split count (adjusted exactly as qsa_sparse_prefill_plan does).
 *   workspace    device scratch of at least the planned size (may be NULL when the plan
 *                needs 0 bytes).  Contents on entry are irrelevant.
 *   err_word     device uint32 that receives QSA_ERRBIT_* bits via atomic OR, or NULL.
 *                The caller clears it; it is read back whenever the caller chooses.
 *   stream       cudaStream_t on which all work is enqueued.
 *
 * Alignment: q, k_cache, v_cache and out must be 16-byte aligned and their t/h/s
 * strides multiples of 8 elements (16 bytes); slot_idx and width 4-byte aligned.
 * Errors are reported before any launch and leave `out` untouched.  The call is
 * deterministic: the same inputs give bitwise the same `out` (inputs are read-only).
 */
qsa_status_t qsa_sparse_prefill(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                                const void* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                                const void* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                                const int32_t* slot_idx, int64_t idx_stride_t,
                                const int32_t* width, int32_t Tq, int32_t Hq, int32_t Hkv,
                                int32_t D, int64_t S, int32_t W, float scale, void* out,
                                int64_t out_stride_t, int64_t out_stride_h, int32_t nsplit,
                                void* workspace, size_t workspace_bytes, uint32_t* err_word,
                                void* stream);

/* Largest block size of block selection. */
#define QSA_MAX_BLOCK 16

/*
 * qsa_sparse_prefill_block_plan / qsa_sparse_prefill_block -- block selection.
 *
 * Source: the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in
 * CANN prefill PR", section "Why QSA is the awkward part, in numbers": the indexer
 * selects micro-blocks (compression ratio 4, a budget of 2,048 micro-blocks per query);
 * the article's path keeps sparse block size 1 and names "block4" as later work.
 * Reading taken here: every selected entry b of slot_idx names the `block` consecutive
 * physical slots b*block .. b*block + block - 1 (block 4 = micro-blocks of four tokens
 * laid out contiguously in the cache).  An entry is valid when it is not -1 and its
 * whole block lies in [0, S); any other value is masked and sets QSA_ERRBIT_SLOT_RANGE.
 * W counts entries (blocks).  1 <= block <= QSA_MAX_BLOCK (QSA_ERR_INVALID_ARG
 * otherwise).  Everything else is exactly qsa_sparse_prefill_plan / qsa_sparse_prefill,
 * which are these functions with block = 1.
 */
int32_t qsa_sparse_prefill_block_plan(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int32_t W,
                                      int32_t block, int32_t num_sms, int32_t nsplit_request,
                                      size_t* workspace_bytes);

qsa_status_t qsa_sparse_prefill_block(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                                      const void* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                                      const void* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                                      const int32_t* slot_idx, int64_t idx_stride_t,
                                      const int32_t* width, int32_t Tq, int32_t Hq, int32_t Hkv,
                                      int32_t D, int64_t S, int32_t W, int32_t block, float scale,
                                      void* out, int64_t out_stride_t, int64_t out_stride_h,
                                      int32_t nsplit, void* workspace, size_t workspace_bytes,
                                      uint32_t* err_word, void* stream);

/*
 * qsa_sparse_prefill_fp8kv -- the same attention over an fp8_e4m3 K/V cache.
 *
 * Source: the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in
 * CANN prefill PR", section "Where this sits in the Qwen4Exp serving build-out", which
 * reports fp8_e4m3 as the KV-cache format that performed better for this attention's
 * decode.  Reading taken here: k_cache and v_cache hold one OCP FP8 E4M3 code per
 * element (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals, NaN =
 * S.1111.111, no infinities) and each tensor carries one float scale, so the
 * dequantised element is value(code) * k_scale (resp. v_scale).  What one call
 * computes is the definition at the top of this file with
 *   k_cache[s, j, d] := value(k_code[s, j, d]) * k_scale,
 *   v_cache[s, j, d] := value(v_code[s, j, d]) * v_scale.
 * Dequantisation happens on the gathered rows inside the kernel; the cache is read-only.
 *
 * Arguments are those of qsa_sparse_prefill_block, except:
 *   k_cache, v_cache   E4M3 codes (one byte each) [S, Hkv, D]; strides
 *                      (k_stride_s, k_stride_h, 1) in elements = bytes, each a
 *                      non-negative multiple of 16; base 16-byte aligned.
 *   k_scale, v_scale   finite floats (QSA_ERR_INVALID_ARG otherwise).
 * q and out stay bf16 with the alignment rules of qsa_sparse_prefill.  The split plan
 * and workspace are those of qsa_sparse_prefill_block_plan for the same shape and
 * block.  Numerics: the products run on f16 tensor-core inputs with fp32 accumulation;
 * every E4M3 value is exact in f16 and a bf16 query element is exact in f16 for
 * 2^-17 <= |q| < 65536 (smaller magnitudes lose low bits, at most 2^-25 absolute);
 * a query element with |q| >= 65536 sets QSA_ERRBIT_Q_RANGE and its row's output is
 * not valid.  Code NaN in the cache propagates as NaN.
 */
qsa_status_t qsa_sparse_prefill_fp8kv(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                                      const void* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                                      const void* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                                      const int32_t* slot_idx, int64_t idx_stride_t,
                                      const int32_t* width, int32_t Tq, int32_t Hq, int32_t Hkv,
                                      int32_t D, int64_t S, int32_t W, int32_t block, float scale,
                                      float k_scale, float v_scale, void* out,
                                      int64_t out_stride_t, int64_t out_stride_h, int32_t nsplit,
                                      void* workspace, size_t workspace_bytes,
                                      uint32_t* err_word, void* stream);

/*
 * qsa_sparse_prefill_partial / qsa_combine_partials -- context parallelism: the K/V cache
 * split by slot range across devices.
 *
 * Source: the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in
 * CANN prefill PR", section "Where this sits in the Qwen4Exp serving build-out", which
 * names decode context parallelism (DCP) for this attention path.  Reading taken here:
 * device r holds the global slots [slot_lo_r, slot_lo_r + S_r) of the cache; every device
 * sees the same (global) selection; each computes, over its own slots only, the
 * softmax-normalised output and the log-sum-exp of its scores; the records of all devices
 * are exchanged (an all-gather) and combined with log-sum-exp weights, which gives exactly
 * the attention over the union of the slots (the same combine as the split-W path).
 *
 * qsa_sparse_prefill_partial: arguments as qsa_sparse_prefill_block (kv_fp8 = 0, bf16
 * caches) or qsa_sparse_prefill_fp8kv (kv_fp8 = 1, E4M3 caches with k_scale / v_scale),
 * except:
 *   k_cache, v_cache   this device's slots only: row s of the tensors is global slot
 *                      slot_lo + s, 0 <= s < S.
 *   slot_lo            first global slot held here, a non-negative multiple of block
 *                      (any value <= S_total for an empty shard, S == 0).
 *   S_total            global slot extent (>= slot_lo + S).  Selected entries in
 *                      [0, S_total) outside this device's range are skipped silently;
 *                      entries outside [-1, S_total) set QSA_ERRBIT_SLOT_RANGE.
 *   part_o             [Tq, Hq, D] contiguous (16-byte aligned), fp32 or, with
 *                      record_bf16 = 1, bf16 (round to nearest even; half the bytes to
 *                      exchange): the output normalised over this device's valid slots
 *                      (zeros where it has none).
 *   part_lse           fp32 [Tq, Hq] contiguous: log2 of the sum over this device's valid
 *                      slots of 2^(scale * log2(e) * s_i) (k_scale included for E4M3), i.e.
 *                      the base-2 log-sum-exp of the scaled scores; -inf where none.
 *                      Always fp32.
 *   record_bf16        0: part_o fp32; 1: part_o bf16.  Any other value: QSA_ERR_INVALID_ARG.
 * The split plan is that of qsa_sparse_prefill_block_plan, and so is the workspace the
 * call requires; the device's own splits are combined into the one record before the
 * call's work ends.  With an unsplit plan on a shard smaller than the whole cache
 * (S < S_total), a workspace of the size qsa_sparse_prefill_partial_plan returns lets
 * the call first copy every row's local entries (in order) to the workspace, so that the
 * fused kernel reads only those instead of the whole global selection; with less (or
 * none) the fused kernel scans the global selection itself.  Both give the same result,
 * bit for bit.
 *
 * qsa_sparse_prefill_partial_plan: host only, like qsa_sparse_prefill_block_plan, whose
 * split count it returns; *workspace_bytes (may be NULL) receives the workspace for the
 * fastest form of the call: the split workspace when the plan splits W, else the
 * compaction buffer ([Tq, W] and [Tq] int32, each 256-byte aligned) when the shard is
 * smaller than the cache (S < S_total) and W >= 32, else 0.  Returns a negative
 * qsa_status_t value for an invalid shape or 0 <= S <= S_total violated.
 *
 * qsa_combine_partials: out[t, h, :] = sum_r 2^(lse_r - m) O_r / sum_r 2^(lse_r - m),
 * m = max_r lse_r, over R records stacked as part_o [R, Tq, Hq, D] (fp32, or bf16 with
 * record_bf16 = 1) and part_lse fp32 [R, Tq, Hq] (the layout an all-gather of the
 * records produces); the sums run in fp32 in record order; records with
 * lse = -inf weigh 0; a row with no record above -inf is written as exact zeros.  out is
 * bf16 [Tq, Hq, D] with strides (out_stride_t, out_stride_h, 1), multiples of 8.
 * Both entry points enqueue on `stream` only and allocate nothing.
 */
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
                                        uint32_t* err_word, void* stream);

int32_t qsa_sparse_prefill_partial_plan(int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int32_t W,
                                        int32_t block, int64_t S, int64_t S_total,
                                        int32_t num_sms, int32_t nsplit_request,
                                        size_t* workspace_bytes);

qsa_status_t qsa_combine_partials(const void* part_o, const float* part_lse, int32_t record_bf16,
                                  int32_t R, int32_t Tq, int32_t Hq, int32_t D, void* out,
                                  int64_t out_stride_t, int64_t out_stride_h, void* stream);

/* Size of the device scratch array that qsa_sparse_prefill_noalloc uses (16 MiB). */
#define QSA_STATIC_SCRATCH_BYTES ((size_t)16 << 20)

/*
 * qsa_sparse_prefill_noalloc -- qsa_sparse_prefill for callers that cannot allocate.
 *
 * The article has no counterpart to this entry point; it exists for users of the
 * library.  Some callers have no way to hand over a workspace: a serving runtime that
 * reserved all free HBM for its KV-cache pool at start-up and forbids cudaMalloc
 * afterwards, a host framework that owns the allocator and gives a plugin no hook into
 * it, or code that must not allocate while a stream is being captured.  Only the
 * split-W path (nsplit > 1) needs scratch; this entry point takes it from a
 * file-scope device array of QSA_STATIC_SCRATCH_BYTES in libqsa.so, which every GPU
 * that loads the library holds until the process exits.
 *
 * Arguments, layouts, ownership and errors are those of qsa_sparse_prefill without
 * `workspace` / `workspace_bytes`.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.  Additional behaviour:
 *   - the first call on a device (the current device) that needs scratch looks up that
 *     device's address of the array (cudaGetSymbolAddress) and caches it under the
 *     current CUDA context's unique ID; make that first call before any stream capture
 *     on the device.  After a device reset (or with another context current) the
 *     address is looked up again on the next call, so no stale address is used;
 *   - a shape whose plan needs more scratch than QSA_STATIC_SCRATCH_BYTES returns
 *     QSA_ERR_WORKSPACE before any launch (qsa_sparse_prefill_plan gives the need;
 *     a smaller nsplit request, or the workspace entry point, are the ways out);
 *   - all calls on a device share the one array and it keeps whatever the last call
 *     left in it; nothing in it has to start at zero: every log-sum-exp value a call
 *     reads was written earlier in the same call, and a split's partial output row is
 *     read but ignored when that split's log-sum-exp is -inf (an empty split, whose row
 *     the call does not write), so stale contents never reach `out`.  Calls whose
 *     kernels overlap on the GPU (e.g. on two streams) race on the array: serialise them.
 */
qsa_status_t qsa_sparse_prefill_noalloc(const void* q, int64_t q_stride_t, int64_t q_stride_h,
                                        const void* k_cache, int64_t k_stride_s,
                                        int64_t k_stride_h, const void* v_cache,
                                        int64_t v_stride_s, int64_t v_stride_h,
                                        const int32_t* slot_idx, int64_t idx_stride_t,
                                        const int32_t* width, int32_t Tq, int32_t Hq,
                                        int32_t Hkv, int32_t D, int64_t S, int32_t W,
                                        float scale, void* out, int64_t out_stride_t,
                                        int64_t out_stride_h, int32_t nsplit,
                                        uint32_t* err_word, void* stream);

/* Human-readable name of a status code (static storage). */
const char* qsa_status_string(qsa_status_t status);

/* Detail of the most recent non-OK status returned on the calling host thread
 * (static thread-local storage; "" if none). */
const char* qsa_last_error_detail(void);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H_ */
