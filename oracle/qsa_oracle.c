/*
 * qsa_oracle.c -- plain CPU oracle for selected-slot sparse attention (QSA prefill).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark may load this library.  The CUDA library shares no code, header,
 * table or helper with it, and neither one calls the other.
 *
 * What it follows: the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's
 * opt-in CANN prefill PR" (orcarouter.ai blog):
 *   - "What the pull request actually adds", packed-embedding paragraph: the output is
 *     softmax(scale * Q K^T) V over the selected slots (the packing C = [K, V],
 *     Q' = [Q, 0] is an exact identity and is NOT used here: this is the plain
 *     definition); the original head-dim-256 scale is kept.
 *   - same section, sizing bullet: -1 entries are padding (masked) and fully masked
 *     rows output zero ("zero-output convention").
 *   - "Nine tests that passed, ...": an FP32 CPU reference computed from the same BF16
 *     inputs; unordered physical slots; zero selection width.
 *   - "Why QSA is the awkward part, in numbers": block selection ("block4"), see
 *     qsa_oracle_forward_block.
 *   - "Where this sits in the Qwen4Exp serving build-out": the fp8_e4m3 KV cache, see
 *     qsa_oracle_forward_fp8kv (E4M3 decoded field by field from the format's definition).
 * Precision: the article fixes FP32 for the reference, so every accumulation below is
 * a float in plain sequential order.  exp is the C library's expf.
 *
 * Readings where the article is silent (each is listed in the design notes):
 *   - query head h reads KV head floor(h / G), G = Hq / Hkv (contiguous GQA groups);
 *   - entries at w >= width[t] are ignored; -1 anywhere inside the width is masked;
 *   - an index outside [-1, S) is masked and raises bit 0 of *err_word;
 *     a width outside [0, W] is clamped and raises bit 1;
 *   - duplicate slots count once per occurrence (softmax over the multiset).
 *
 * bf16 inputs arrive as raw uint16 bit patterns; a bf16 value is the top half of the
 * float with the same bits, so widening is exact.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static float bf16_to_float(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* One (t, h) output row: the plain definition, written out.  Returns the number of
 * valid slots it used.  `scratch_s` holds up to W scores, `scratch_i` up to W slots. */
static int32_t oracle_row(const uint16_t* q_row, const uint16_t* k_cache,
                          const uint16_t* v_cache, int64_t k_stride_s, int64_t k_stride_h,
                          int64_t v_stride_s, int64_t v_stride_h, const int32_t* idx_row,
                          int32_t width_t, int32_t j, int32_t D, int64_t S, float scale,
                          float* out_row, float* scratch_s, int64_t* scratch_i,
                          uint32_t* err_bits) {
  /* 1. The valid selected slots of this query row (unordered, -1 skipped). */
  int32_t n = 0;
  for (int32_t w = 0; w < width_t; ++w) {
    int32_t slot = idx_row[w];
    if (slot == -1) continue;
    if (slot < -1 || (int64_t)slot >= S) {
      *err_bits |= 1u;
      continue;
    }
    scratch_i[n++] = (int64_t)slot;
  }

  /* 2. Fully masked row or zero width: exactly zero. */
  if (n == 0) {
    for (int32_t d = 0; d < D; ++d) out_row[d] = 0.0f;
    return 0;
  }

  /* 3. Scores s_i = scale * <q, k_i>. */
  for (int32_t i = 0; i < n; ++i) {
    const uint16_t* k_row = k_cache + scratch_i[i] * k_stride_s + (int64_t)j * k_stride_h;
    float acc = 0.0f;
    for (int32_t d = 0; d < D; ++d) acc += bf16_to_float(q_row[d]) * bf16_to_float(k_row[d]);
    scratch_s[i] = scale * acc;
  }

  /* 4. Softmax over the selected slots only. */
  float m = scratch_s[0];
  for (int32_t i = 1; i < n; ++i)
    if (scratch_s[i] > m) m = scratch_s[i];
  float l = 0.0f;
  for (int32_t i = 0; i < n; ++i) {
    scratch_s[i] = expf(scratch_s[i] - m);
    l += scratch_s[i];
  }

  /* 5. out = (sum_i p_i v_i) / l. */
  for (int32_t d = 0; d < D; ++d) out_row[d] = 0.0f;
  for (int32_t i = 0; i < n; ++i) {
    const uint16_t* v_row = v_cache + scratch_i[i] * v_stride_s + (int64_t)j * v_stride_h;
    for (int32_t d = 0; d < D; ++d) out_row[d] += scratch_s[i] * bf16_to_float(v_row[d]);
  }
  for (int32_t d = 0; d < D; ++d) out_row[d] = out_row[d] / l;
  return n;
}

/*
 * qsa_oracle_forward -- fp32 reference for the rows listed in `rows` (or all Tq rows
 * when rows == NULL).  Host pointers throughout.
 *   q        bf16 bits, element (t, h, d) at q[t*q_stride_t + h*q_stride_h + d]
 *   k_cache  bf16 bits, element (s, j, d) at k_cache[s*k_stride_s + j*k_stride_h + d]
 *   v_cache  likewise with the v strides
 *   slot_idx int32, element (t, w) at slot_idx[t*idx_stride_t + w]
 *   width    int32 [Tq] or NULL (= W)
 *   out      float [nrows or Tq, Hq, D] contiguous; row r of the output is rows[r]
 *   err_bits receives the OR of the flags described above (may be NULL)
 * Returns 0 on success, -1 on invalid sizes (Hq % Hkv != 0 and the like).
 * Parallel over query rows with OpenMP when compiled with -fopenmp.
 */
int qsa_oracle_forward(const uint16_t* q, int64_t q_stride_t, int64_t q_stride_h,
                       const uint16_t* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                       const uint16_t* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                       const int32_t* slot_idx, int64_t idx_stride_t, const int32_t* width,
                       int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int64_t S, int32_t W,
                       float scale, const int64_t* rows, int64_t nrows, float* out,
                       uint32_t* err_bits) {
  if (Tq < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || S < 0 || W < 0) return -1;
  if (Hq % Hkv != 0) return -1;
  const int32_t G = Hq / Hkv;
  const int64_t n_out = rows ? nrows : (int64_t)Tq;
  uint32_t all_bits = 0;

#pragma omp parallel reduction(| : all_bits)
  {
    float* scratch_s = (float*)malloc(sizeof(float) * (size_t)(W > 0 ? W : 1));
    int64_t* scratch_i = (int64_t*)malloc(sizeof(int64_t) * (size_t)(W > 0 ? W : 1));
    uint32_t bits = 0;
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_out; ++r) {
      const int64_t t = rows ? rows[r] : r;
      int32_t width_t = width ? width[t] : W;
      if (width_t < 0 || width_t > W) {
        bits |= 2u;
        width_t = width_t < 0 ? 0 : W;
      }
      const int32_t* idx_row = slot_idx + t * idx_stride_t;
      for (int32_t h = 0; h < Hq; ++h) {
        const int32_t j = h / G;
        const uint16_t* q_row = q + t * q_stride_t + (int64_t)h * q_stride_h;
        float* out_row = out + (r * Hq + h) * (int64_t)D;
        oracle_row(q_row, k_cache, v_cache, k_stride_s, k_stride_h, v_stride_s, v_stride_h,
                   idx_row, width_t, j, D, S, scale, out_row, scratch_s, scratch_i, &bits);
      }
    }
    free(scratch_s);
    free(scratch_i);
    all_bits |= bits;
  }
  if (err_bits) *err_bits |= all_bits;
  return 0;
}

/*
 * qsa_oracle_forward_block -- block selection: every selected entry b of slot_idx names
 * the `block` consecutive physical slots b*block .. b*block + block - 1 (sparse block
 * size `block`; the article's path keeps block size 1 and names "block4" as later work,
 * section "Why QSA is the awkward part, in numbers").  The definition: expand each
 * valid entry into its slots, in order, then apply the slot-level definition above.
 * An entry is valid when it is not -1 and its whole block lies in [0, S); any other
 * value raises bit 0 of *err_bits and is skipped.  Arguments as qsa_oracle_forward,
 * W counting entries (blocks), plus `block` >= 1.
 */
int qsa_oracle_forward_block(const uint16_t* q, int64_t q_stride_t, int64_t q_stride_h,
                             const uint16_t* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                             const uint16_t* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                             const int32_t* slot_idx, int64_t idx_stride_t, const int32_t* width,
                             int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int64_t S, int32_t W,
                             int32_t block, float scale, const int64_t* rows, int64_t nrows,
                             float* out, uint32_t* err_bits) {
  if (Tq < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || S < 0 || W < 0 || block < 1) return -1;
  if (Hq % Hkv != 0) return -1;
  const int32_t G = Hq / Hkv;
  const int64_t n_out = rows ? nrows : (int64_t)Tq;
  const int64_t cap = (int64_t)W * block;
  uint32_t all_bits = 0;

#pragma omp parallel reduction(| : all_bits)
  {
    int32_t* expanded = (int32_t*)malloc(sizeof(int32_t) * (size_t)(cap > 0 ? cap : 1));
    float* scratch_s = (float*)malloc(sizeof(float) * (size_t)(cap > 0 ? cap : 1));
    int64_t* scratch_i = (int64_t*)malloc(sizeof(int64_t) * (size_t)(cap > 0 ? cap : 1));
    uint32_t bits = 0;
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_out; ++r) {
      const int64_t t = rows ? rows[r] : r;
      int32_t width_t = width ? width[t] : W;
      if (width_t < 0 || width_t > W) {
        bits |= 2u;
        width_t = width_t < 0 ? 0 : W;
      }
      /* expand the valid blocks into their slots */
      const int32_t* idx_row = slot_idx + t * idx_stride_t;
      int32_t n = 0;
      for (int32_t w = 0; w < width_t; ++w) {
        const int32_t b = idx_row[w];
        if (b == -1) continue;
        if (b < -1 || ((int64_t)b + 1) * block > S) {
          bits |= 1u;
          continue;
        }
        for (int32_t e = 0; e < block; ++e) expanded[n++] = b * block + e;
      }
      for (int32_t h = 0; h < Hq; ++h) {
        const int32_t j = h / G;
        const uint16_t* q_row = q + t * q_stride_t + (int64_t)h * q_stride_h;
        float* out_row = out + (r * Hq + h) * (int64_t)D;
        oracle_row(q_row, k_cache, v_cache, k_stride_s, k_stride_h, v_stride_s, v_stride_h,
                   expanded, n, j, D, S, scale, out_row, scratch_s, scratch_i, &bits);
      }
    }
    free(expanded);
    free(scratch_s);
    free(scratch_i);
    all_bits |= bits;
  }
  if (err_bits) *err_bits |= all_bits;
  return 0;
}

/*
 * fp8_e4m3 KV cache.  The article's section "Where this sits in the Qwen4Exp serving
 * build-out" reports fp8_e4m3 as the better-performing KV-cache format for this
 * attention's decode.  Reading used here: the cache holds one OCP FP8 E4M3 code per
 * element, and each of K and V carries one float scale (a dequantised element is
 * code value x scale); the attention is then the definition above applied to the
 * dequantised rows.
 *
 * e4m3_value -- the value of one E4M3 code, decoded field by field: 1 sign bit, 4
 * exponent bits with bias 7, 3 mantissa bits; an exponent field of 0 encodes the
 * subnormals (m / 8) * 2^(1 - 7); the pattern S.1111.111 is NaN and there are no
 * infinities (the "FN" variant, largest finite magnitude 448).
 */
static float e4m3_value(uint8_t code) {
  const int sign = code >> 7;
  const int e = (code >> 3) & 15;
  const int m = code & 7;
  float mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    mag = ldexpf((float)m / 8.0f, 1 - 7);
  else
    mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return sign ? -mag : mag;
}

/* Decode n E4M3 codes (exported for the tests). */
void qsa_oracle_decode_e4m3(const uint8_t* codes, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(codes[i]);
}

/*
 * qsa_oracle_forward_fp8kv -- fp32 reference with an fp8_e4m3 K/V cache.
 *   k_cache, v_cache  E4M3 codes, element (s, j, d) at k_cache[s*k_stride_s +
 *                     j*k_stride_h + d] (strides in elements = bytes)
 *   k_scale, v_scale  dequantisation scales: K = e4m3_value(code) * k_scale, likewise V
 *   block             as qsa_oracle_forward_block (1 = slot selection)
 * Every other argument as qsa_oracle_forward.  Steps per (t, KV head j): the valid
 * selected slots (width, -1 and range rules of the slot-level definition, blocks
 * expanded), their K and V rows dequantised into float, then for each query head of
 * the group: scores scale * <q, k_i>, softmax over the selected slots, P V.
 */
int qsa_oracle_forward_fp8kv(const uint16_t* q, int64_t q_stride_t, int64_t q_stride_h,
                             const uint8_t* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                             const uint8_t* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                             const int32_t* slot_idx, int64_t idx_stride_t, const int32_t* width,
                             int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int64_t S, int32_t W,
                             int32_t block, float scale, float k_scale, float v_scale,
                             const int64_t* rows, int64_t nrows, float* out, uint32_t* err_bits) {
  if (Tq < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || S < 0 || W < 0 || block < 1) return -1;
  if (Hq % Hkv != 0) return -1;
  const int32_t G = Hq / Hkv;
  const int64_t n_out = rows ? nrows : (int64_t)Tq;
  const int64_t cap = (int64_t)W * block;
  const size_t cap1 = (size_t)(cap > 0 ? cap : 1);
  uint32_t all_bits = 0;

#pragma omp parallel reduction(| : all_bits)
  {
    int64_t* sel = (int64_t*)malloc(sizeof(int64_t) * cap1);
    float* kf = (float*)malloc(sizeof(float) * cap1 * (size_t)D);
    float* vf = (float*)malloc(sizeof(float) * cap1 * (size_t)D);
    float* sc = (float*)malloc(sizeof(float) * cap1);
    uint32_t bits = 0;
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_out; ++r) {
      const int64_t t = rows ? rows[r] : r;
      int32_t width_t = width ? width[t] : W;
      if (width_t < 0 || width_t > W) {
        bits |= 2u;
        width_t = width_t < 0 ? 0 : W;
      }
      /* 1. the valid selected slots of the row (blocks expanded, -1 skipped) */
      const int32_t* idx_row = slot_idx + t * idx_stride_t;
      int64_t n = 0;
      for (int32_t w = 0; w < width_t; ++w) {
        const int32_t b = idx_row[w];
        if (b == -1) continue;
        if (b < -1 || ((int64_t)b + 1) * block > S) {
          bits |= 1u;
          continue;
        }
        for (int32_t e = 0; e < block; ++e) sel[n++] = (int64_t)b * block + e;
      }
      for (int32_t j = 0; j < Hkv; ++j) {
        /* 2. dequantise the selected K and V rows of KV head j */
        for (int64_t i = 0; i < n; ++i) {
          const uint8_t* k_row = k_cache + sel[i] * k_stride_s + (int64_t)j * k_stride_h;
          const uint8_t* v_row = v_cache + sel[i] * v_stride_s + (int64_t)j * v_stride_h;
          for (int32_t d = 0; d < D; ++d) {
            kf[i * D + d] = e4m3_value(k_row[d]) * k_scale;
            vf[i * D + d] = e4m3_value(v_row[d]) * v_scale;
          }
        }
        for (int32_t h = j * G; h < (j + 1) * G; ++h) {
          const uint16_t* q_row = q + t * q_stride_t + (int64_t)h * q_stride_h;
          float* out_row = out + (r * Hq + h) * (int64_t)D;
          for (int32_t d = 0; d < D; ++d) out_row[d] = 0.0f;
          if (n == 0) continue; /* fully masked row or zero width: exactly zero */
          /* 3. scores */
          for (int64_t i = 0; i < n; ++i) {
            float acc = 0.0f;
            for (int32_t d = 0; d < D; ++d) acc += bf16_to_float(q_row[d]) * kf[i * D + d];
            sc[i] = scale * acc;
          }
          /* 4. softmax over the selected slots */
          float m = sc[0];
          for (int64_t i = 1; i < n; ++i)
            if (sc[i] > m) m = sc[i];
          float l = 0.0f;
          for (int64_t i = 0; i < n; ++i) {
            sc[i] = expf(sc[i] - m);
            l += sc[i];
          }
          /* 5. P V, normalised */
          for (int64_t i = 0; i < n; ++i)
            for (int32_t d = 0; d < D; ++d) out_row[d] += sc[i] * vf[i * D + d];
          for (int32_t d = 0; d < D; ++d) out_row[d] = out_row[d] / l;
        }
      }
    }
    free(sel);
    free(kf);
    free(vf);
    free(sc);
    all_bits |= bits;
  }
  if (err_bits) *err_bits |= all_bits;
  return 0;
}

/* Number of OpenMP threads a parallel region of this library uses (1 without OpenMP). */
int qsa_oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
