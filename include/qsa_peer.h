/*
 * qsa_peer.h -- context parallelism with the record exchange fused into the combine.
 *
 * Source: the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in
 * CANN prefill PR", section "Where this sits in the Qwen4Exp serving build-out", which
 * names decode context parallelism for this attention path.  The reading (qsa.h,
 * qsa_sparse_prefill_partial): every device holds a slot range of the cache, computes over
 * its own slots the softmax-normalised output O_r and the base-2 log-sum-exp lse_r of its
 * scores, and the records of all devices are combined with log-sum-exp weights.
 *
 * qsa.h's qsa_combine_partials reads the records stacked in one local buffer, which an
 * all-gather fills first.  qsa_combine_peer_records reads every record where it lies,
 * through one device pointer per record: memory of this device, or another device's
 * memory mapped into this process (CUDA IPC; on one node the loads cross NVLink /
 * NVSwitch as plain peer loads, no multicast).  The exchange is then the combine kernel's
 * own loads, overlapped with its arithmetic row by row, and no gathered copy of the
 * records exists.  The kernel can also store each combined row to several output buffers
 * (this device's and peers'), so that each device combining only its own share of the
 * query rows and storing it to every device's output replaces both the record all-gather
 * and an all-gather of the outputs.
 *
 * The IPC helpers below export and map the device allocations that hold the records and
 * outputs; they are plain wrappers of the CUDA runtime's IPC calls, with the byte offset of
 * a pointer inside its allocation carried alongside the handle (allocators hand out
 * pieces of larger allocations, and a handle names a whole allocation).
 *
 * Ordering is the caller's: every record a combine reads must be complete, and no record
 * or output buffer may be rewritten while another device's combine still reads or writes
 * it.  On devices of one process group a collective issued on the same stream before and
 * after the combine (every rank's stream reaches it only after its own earlier kernels)
 * gives that order; no kernel of this library waits on another device.
 */
#ifndef QSA_PEER_H_
#define QSA_PEER_H_

#include "qsa.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Records (and output buffers) one combine can address. */
#define QSA_MAX_PEERS 16

/* Bytes of a CUDA IPC memory handle. */
#define QSA_IPC_HANDLE_BYTES 64

/*
 * qsa_combine_peer_records -- out_k[t, h, :] = sum_r 2^(lse_r - m) O_r / sum_r 2^(lse_r - m),
 * m = max_r lse_r, for t0 <= t < t1 and every head h, stored to each of the n_out outputs.
 *
 *   rec_o       HOST array of R device pointers: record r's O, [Tq, Hq, D] contiguous,
 *               fp32 or (record_bf16 = 1) bf16, 16-byte aligned, as
 *               qsa_sparse_prefill_partial writes it.
 *   rec_lse     HOST array of R device pointers: record r's lse, fp32 [Tq, Hq] contiguous,
 *               4-byte aligned.
 *   R           1 <= R <= QSA_MAX_PEERS; the sums run in fp32 in the order r = 0 .. R-1,
 *               the same arithmetic as qsa_combine_partials (the results are bitwise
 *               equal for the same records); records with lse = -inf weigh 0, and a row
 *               with no record above -inf is written as exact zeros.
 *   record_bf16 0 or 1 (otherwise QSA_ERR_INVALID_ARG).
 *   Tq, Hq, D   the records' shape; D must be 256 (QSA_ERR_UNSUPPORTED otherwise).
 *   t0, t1      the query rows combined, 0 <= t0 <= t1 <= Tq (t0 == t1: nothing to do).
 *   out         HOST array of n_out device pointers (1 <= n_out <= QSA_MAX_PEERS), each a
 *               bf16 [Tq, Hq, D] output (16-byte aligned) with strides (out_stride_t,
 *               out_stride_h, 1), non-negative multiples of 8; row t of each is written,
 *               rows outside [t0, t1) are not touched.
 * Every pointer must be addressable from the device current on the calling thread (its
 * own memory, or peer memory mapped into this process); the library cannot check that and
 * a wrong pointer faults the kernel.  Host arrays are read during the call only.
 * Enqueues one kernel on `stream`; allocates nothing, never synchronises.
 */
qsa_status_t qsa_combine_peer_records(const void* const* rec_o, const float* const* rec_lse,
                                      int32_t R, int32_t record_bf16, int32_t Tq, int32_t Hq,
                                      int32_t D, int32_t t0, int32_t t1, void* const* out,
                                      int32_t n_out, int64_t out_stride_t, int64_t out_stride_h,
                                      void* stream);

/*
 * qsa_ipc_export -- the CUDA IPC handle (QSA_IPC_HANDLE_BYTES bytes written to `handle`)
 * of the device allocation that contains `ptr`, and ptr's byte offset in it (*offset).
 * QSA_ERR_INVALID_ARG for NULL arguments; QSA_ERR_CUDA when the runtime refuses (e.g.
 * memory from an allocator whose allocations cannot be exported this way), with the
 * runtime's message in qsa_last_error_detail().
 */
qsa_status_t qsa_ipc_export(const void* ptr, void* handle, uint64_t* offset);

/*
 * qsa_ipc_import -- maps into this process, on the current device, the allocation whose
 * handle another process exported (*base: the mapping's first byte; add the exporter's
 * offset).  Peer access is enabled as the mapping needs it.  A handle from this same
 * process cannot be imported (the runtime refuses it: use the pointer itself).
 */
qsa_status_t qsa_ipc_import(const void* handle, void** base);

/* qsa_ipc_close -- unmaps a base returned by qsa_ipc_import (after the work using it). */
qsa_status_t qsa_ipc_close(void* base);

#ifdef __cplusplus
}
#endif

#endif /* QSA_PEER_H_ */
