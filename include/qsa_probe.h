/*
 * qsa_probe.h -- measurement entry point of libqsa.so: the gather-rate probe.
 *
 * Not part of the attention computation.  It measures, on the device at hand, the
 * SM-side roofline of the sparse-attention gather: how fast the SMs pull rows chosen at
 * random from an L2-resident buffer into shared memory (512-byte rows: one bf16 (slot,
 * head) row of K or V with head dimension 256; 256-byte rows: the same in E4M3 codes),
 * and read each landed row back once with ldmatrix, as the fused kernel of qsa.h does
 * before its tensor-core products.  The long-prefill case of the article "Qwen4-Exp QSA
 * comes to Huawei's Ascend: inside SGLang's opt-in CANN prefill PR" (section "Nine tests
 * that passed, and a speed number that did not come from this branch": 7,810 queries x
 * 2,051 selected slots over a 65,536-slot cache) gathers from a cache about the size of
 * B200's L2, so most of its gathered rows are L2 hits and this rate, not HBM bandwidth,
 * is the bound it runs against.
 */
#ifndef QSA_PROBE_H_
#define QSA_PROBE_H_

#include "qsa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * qsa_probe_gather -- enqueue one launch of the gather probe on `stream`.
 *
 *   method         0: cp.async.cg 16-byte copies, every lane of a warp copying one chunk
 *                     of each row (the fused kernel's loader);
 *                  1: TMA tile::gather4 (four rows x 128 bytes per instruction, 128-byte
 *                     swizzle) issued by one lane of each warp, mbarrier completion;
 *                  2: the same TMA gathers issued by one producer warp for all warps of
 *                     the CTA (full / empty mbarrier rings);
 *                  3: the TMA gathers of a sub-tile issued by several lanes of each warp
 *                     in one warp instruction (one gather4 per lane).
 *   read_back      0: the rows are only landed; 1: every landed 16-row sub-tile is read
 *                  back once (ldmatrix.x4); 2: read back and every fragment compared with
 *                  the source bytes of its row (a check of the shared-memory layout; slow),
 *                  the number of mismatches added to sink[1].
 *   src            device buffer of `rows` rows of `row_bytes` (512 or 256) bytes each,
 *                  `pitch_bytes` apart (a multiple of 16, >= row_bytes); 16-byte aligned.
 *                  Read only.  rows <= 2^31.
 *   warps_per_cta  consumer warps per CTA (1..15); method 2 adds one producer warp.
 *   stages         sub-tiles in flight per warp (2..4); shared memory per CTA is
 *                  warps x stages x 16 x row_bytes (at most 227 KiB).
 *   ctas, iters    grid size, and 16-row sub-tiles each warp gathers.
 *   seed           seed of the rows' random sequence (a linear congruential generator
 *                  per warp, mapped onto [0, rows)).
 *   sink           device uint32[258]: bit 0 of sink[0] is set if a wait timed out and
 *                  bit 1 if the shared-memory window was not 1024-byte aligned (either
 *                  way the launch is not a valid measurement); sink[1] counts layout
 *                  mismatches (read_back 2); the rest is a sink for the values read back.
 *                  The caller clears sink[0] and sink[1].
 * Bytes moved by one launch: ctas x warps_per_cta x iters x 16 x row_bytes.  The caller
 * times the launch (CUDA events on `stream`).  Returns QSA_ERR_INVALID_ARG for
 * arguments outside the ranges above, QSA_ERR_CUDA if the tensor map cannot be encoded
 * or the launch fails.  Allocates nothing.
 */
qsa_status_t qsa_probe_gather(int32_t method, int32_t read_back, const void* src, int64_t rows,
                              int64_t pitch_bytes, int32_t row_bytes, int32_t warps_per_cta,
                              int32_t stages, int32_t ctas, int32_t iters, uint32_t seed,
                              uint32_t* sink, void* stream);

/*
 * qsa_probe_mma_operands -- enqueue one launch of the MMA operand-rate probe on `stream`.
 *
 * The fused kernel reads every gathered K and V row from shared memory once, into its
 * matrix products.  On sm_100a that read can be done by the warps (ldmatrix into
 * registers for the warp-level mma, the form the fused kernel uses) or by the tensor core
 * itself (tcgen05.mma reads both operands through shared-memory matrix descriptors and
 * accumulates in tensor memory).  This probe measures how many operand bytes per clock
 * each form reads from one SM's shared memory, so the two can be compared at the skinny
 * shapes of this path (many slots x a group of 8 to 16 heads).
 *
 *   method  0: ldmatrix.x4 by 16 warps over a 64 KiB window (n must be 0); bytes read per
 *              CTA: rounds x 16 warps x 128 x 512.
 *           1: tcgen05.mma.cta_group::1.kind::f16, M = 128, N = n, K = 16 per
 *              instruction, bf16 K-major operands without swizzle, fp32 accumulator in
 *              tensor memory, issued by one thread back to back, completion through
 *              tcgen05.commit on an mbarrier (a bounded wait); bytes read per CTA:
 *              rounds x 16 x (128 + n) x 32.  The operands are bf16 ones, so every
 *              accumulator element must end at rounds x 256; each of the 128 lanes of column
 *              0 is checked.
 *   n       method 1: 16, 32, 64, 128 or 256.
 *   rounds  1 .. 65,536 passes.
 *   ctas    grid size (one CTA per SM is what the probe is sized for: the tcgen05 variant
 *           takes 200 KiB of shared memory).
 *   out     device int64 [2 + ctas], 8-byte aligned; the caller clears out[0] and out[1].
 *           out[0] bit 0: a completion wait timed out (the launch is not a measurement);
 *           out[1]: accumulator elements that are not rounds x 256 (method 1); out[2 + b]:
 *           the SM clock cycles CTA b spent in its timed loop (clock64).
 * Operand bytes per clock per SM = bytes read per CTA / max_b out[2 + b].  Returns
 * QSA_ERR_INVALID_ARG for arguments outside the ranges above, QSA_ERR_CUDA if the launch
 * fails.  Allocates nothing (the tensor memory the tcgen05 variant allocates is freed by
 * the same CTA before it exits).
 */
qsa_status_t qsa_probe_mma_operands(int32_t method, int32_t n, int32_t rounds, int32_t ctas,
                                    int64_t* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QSA_PROBE_H_ */
