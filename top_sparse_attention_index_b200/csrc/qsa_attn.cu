// qsa_attn.cu -- sm_100a kernels for selected-slot sparse attention (QSA prefill).
//
// Operation (article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in
// CANN prefill PR", section "What the pull request actually adds"): for every query row
// t and KV head j, gather the row's selected physical slots of K and V, form
// scale * Q K^T for the whole GQA group of G = Hq / Hkv query heads, take the softmax
// over the selected slots only and return P V; a row without a valid slot returns 0.
//
// K1 qsa_sparse_attn_fwd_kernel -- one CTA per (t, j, split) work unit, several CTAs
// resident per SM so that one CTA's prologue and epilogue overlap the others' gathers
// (bf16: two, or three of two slot lanes each when the cache has at most 65,536 rows so
// the compacted row list is 16-bit and the launch has many waves; E4M3 caches in such
// launches: eight of one slot lane for G <= 8, six for G > 8; units ordered KV head
// slowest when one head's slice of the cache fits L2 and the whole cache does not):
//   1. stage the split's slot indices in shared memory and compact away -1 (and
//      out-of-range) entries with a block scan, so masked slots cost no bandwidth;
//   2. gather K and V rows of the compacted slots with 16-byte cp.async (or, in builds
//      that ask for it, TMA tile::gather4, measured slower) into shared
//      memory: each 16-slot sub-tile of a stage belongs to one slot lane (a warp pair)
//      that loads it, waits for it and consumes it, so the lanes run STAGES-deep
//      pipelines of their own with no block-wide barrier in the loop (row = 512
//      contiguous bytes; the 16-byte chunks of a row are XOR-swizzled by the row index
//      so ldmatrix reads are conflict-free);
//   3. per slot lane and 16-slot sub-tile: S^T = K Q^T with the slots as the MMA M
//      dimension and the (up to 8) heads of one n8 tile as N, so the group shares every
//      gathered row and G = 3/6/8/12/16 needs no padding of the head ratio in memory
//      (the warp pair splits D for both products and exchanges partial scores; for
//      G > 8 each warp handles both n8 head tiles); online softmax in fp32 registers
//      (base 2, lazy rescaling); P rounded to bf16 and transposed in registers
//      (movmatrix) into the B operand of O^T += V^T P^T with D = 256 as M;
//   4. merge the per-warp (m, l, O) states through shared memory and write bf16 out
//      (exact zeros for empty rows), or fp32 partials + base-2 LSE when split.
// K2 qsa_lse_combine_kernel -- one warp per (t, h): log-sum-exp weighted sum of the
//   split partials (or of context-parallel records, fp32 or bf16); empty splits carry
//   LSE = -inf and weight 0; all empty -> exact 0.
// qsa_shard_compact_kernel -- context-parallel shards: each row's local entries copied in
//   order before K1, which then scans only those.
//
// fp8_e4m3 KV cache (the format named in section "Where this sits in the Qwen4Exp serving
// build-out" of the same article): K1 with KV8 gathers 256-byte rows of E4M3 codes (half
// the bytes), keeps them 8-bit in shared memory and converts them to f16 in registers
// after ldmatrix; Q, P and both MMAs are f16 with fp32 accumulation; k_scale is folded
// into the softmax scale and v_scale into the final normalisation, so the result is the
// attention over the dequantised cache up to rounding.
#include <cuda.h>  // CUtensorMap (the TMA gather's tensor maps)
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <type_traits>

#include "qsa_internal.h"
#include "qsa_ptx.cuh"

namespace qsa {
namespace {

constexpr int kRowBytes = kHeadDim * 2;     // one (slot, head) row: 512 bytes
constexpr int kChunks = kRowBytes / 16;     // 32 16-byte chunks per row
constexpr int kMergeStride = kHeadDim + 4;  // padded fp32 row of the epilogue merge
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (base-2 exponent)
constexpr uint32_t kMaxPolls = 1u << 20;  // bound of one mbarrier wait (TMA gathers)
// E4M3 shapes with this many slot lanes read all of a warp's V code pairs early (the
// eight-CTA shape of one lane: 1.482 vs 1.489 ms with two pairs)
#ifndef QSA_FP8_EARLY_ALL_LANES
#define QSA_FP8_EARLY_ALL_LANES 1
#endif


// Tensor maps of the TMA gather, one per KV head for K and for V: a 2-D view [S rows,
// 256 elements] of that head's slice of the cache (row pitch = the slot stride), a box of
// one 128-byte column block of one row, 128-byte swizzle (tile::gather4 row gathers).
constexpr int kMaxTmaHeads = 4;
struct TmaMaps {
  CUtensorMap k[kMaxTmaHeads];
  CUtensorMap v[kMaxTmaHeads];
};

template <int NTILE, int DSPLIT, int SL, int STAGES, bool KV8 = false, bool SLOT16 = false,
          int QROWS = NTILE * 8, bool TMA = false>
struct Cfg {
  // warps serving one slot lane: a D-split pair (each warp handles every head tile over
  // its half of D) or one warp per head tile
  static constexpr int kParts = DSPLIT > 1 ? DSPLIT : NTILE;
  static constexpr int kTPW = DSPLIT > 1 ? NTILE : 1;  // head tiles per warp
  static constexpr int kWarps = kParts * SL;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr int kRows = 16 * SL;                      // slots per stage
  static constexpr int kKvRow = KV8 ? kHeadDim : kRowBytes;  // one gathered K or V row (bytes)
  static constexpr int kSubBytes = 16 * kKvRow * 2;          // one sub-tile: 16 K rows, 16 V rows
  static constexpr int kStageBytes = SL * kSubBytes;
  static constexpr int kRingBytes = STAGES * kStageBytes;    // [slot lane][stage][sub-tile]
  // the group's Q rows in shared memory: NTILE * 8, or fewer for a shape serving G <= QROWS
  static constexpr int kQRows = QROWS;
  static_assert(QROWS > (NTILE - 1) * 8 && QROWS <= NTILE * 8 && (!KV8 || QROWS == NTILE * 8),
                "Q tile rows");
  static constexpr int kQBytes = QROWS * kRowBytes;
  // compacted row numbers: 16-bit when the cache of the call has at most 65,536 rows
  static constexpr int kIdxBytes = kMaxSlotsPerSplit * (SLOT16 ? 2 : 4);
  static constexpr int kScanBytes = 32 * 4;
  // partial scores a D-split pair exchanges when it also splits Q K^T: [lane][warp][32][4]
  static constexpr int kXchgBytes = (DSPLIT > 1) ? SL * DSPLIT * kTPW * 32 * 16 : 0;
  static constexpr int kTileFloats = 8 * kMergeStride + 16;  // one head tile's merge record
  static constexpr int kMergeBytes = kWarps * kTPW * kTileFloats * 4;
  // the exchange buffer overlays the Q tile, which is dead once the Q fragments are in
  // registers
  static constexpr bool kXchgOverQ = DSPLIT > 1;
  static_assert(!kXchgOverQ || kXchgBytes <= kQBytes, "exchange buffer fits the Q tile");
  // TMA gathers: one full barrier per (slot lane, stage), after the scan words
  static_assert(!TMA || DSPLIT == 2, "the TMA gather serves the D-split pair shapes");
  static constexpr int kBarBytes = TMA ? SL * STAGES * 8 : 0;
  static constexpr size_t kSmem = size_t(kRingBytes) + kQBytes + kIdxBytes + kScanBytes +
                                  (kXchgOverQ ? 0 : kXchgBytes) + kBarBytes;
  // Layout of a gathered sub-tile in shared memory.  cp.async: 16 rows of kKvRow bytes,
  // 16-byte chunk c of row r at r * kKvRow + ((c ^ (r & 7)) << 4).  TMA tile::gather4
  // (128-byte swizzle): kKvRow / 128 column blocks of [16 rows x 128 bytes], chunk c of
  // row r at (c / 8) * 2048 + r * 128 + (((c % 8) ^ (r & 7)) << 4).  Both are the same
  // XOR of the chunk's low three bits; only the row and block pitches differ.
  static constexpr int kRowPitch = TMA ? 128 : kKvRow;
  static constexpr int kBlkPitch = TMA ? 16 * 128 : 128;
  // the epilogue's merge buffer reuses the ring and, after it, the Q tile and the slot
  // list (all dead once the main loop is over)
  static_assert(kMergeBytes <= kRingBytes + kQBytes + kIdxBytes, "merge buffer fits");
  static_assert(kMaxSlotsPerSplit * 4 <= kRingBytes, "raw index staging reuses the ring");
  static_assert(kMaxSlotsPerSplit % 16 == 0, "the offset list pads to whole sub-tiles");
  // shared memory one SM gives its resident CTAs (228 KiB, 1 KiB reserved per CTA)
  static constexpr size_t kSmPerCta(int ctas) { return 233472 / ctas - 1024; }
};

// NTILE n8 tiles cover the head group (G <= 8: 1; G <= 16: 2).  The warps of one slot
// lane split either the head tiles (DSPLIT = 1: one warp per tile) or, with DSPLIT = 2,
// the D rows of the PV product, each warp handling every head tile (and with QSPLIT also
// the D range of Q K^T, the pair exchanging partial scores), so every gathered row is
// read from shared memory once.
// KV8: the cache holds E4M3 codes (256-byte rows).  The gathered codes stay 8-bit in
// shared memory and become f16 in registers right after ldmatrix (cvt.f16x2.e4m3x2, exact);
// Q and P are f16 too, so both products are f16 MMAs with fp32 accumulation.  The order
// of the D index inside a k-step (Q K^T) or an m-tile (P V) is permuted to match what
// ldmatrix delivers for 8-bit data; a sum over D does not depend on that order, and the
// epilogue maps the m-tile rows back.
template <int NTILE, int DSPLIT, int SL, int STAGES, int MINB, bool QSPLIT, bool KV8, bool SLOT16,
          int QROWS, bool TMA>
__global__ void __launch_bounds__(32 * (DSPLIT > 1 ? DSPLIT : NTILE) * SL, MINB)
    qsa_sparse_attn_fwd_kernel(const FwdParams p, const __grid_constant__ TmaMaps maps) {
  static_assert(!QSPLIT || DSPLIT == 2 || (DSPLIT == 4 && !KV8),
                "splitting Q K^T needs a D-split pair (or a bf16 D-split quad)");
  constexpr int kKS = QSPLIT ? 16 / DSPLIT : 16;  // k-steps of Q K^T per warp
  using C = Cfg<NTILE, DSPLIT, SL, STAGES, KV8, SLOT16, QROWS, TMA>;
  using SlotT = std::conditional_t<SLOT16, uint16_t, uint32_t>;
  constexpr int kKvRow = C::kKvRow;
  constexpr int kMT = 16 / DSPLIT;  // m16 tiles of D per warp in the PV product
  constexpr int TPW = C::kTPW;      // n8 head tiles per warp
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* ring = smem;
  uint8_t* sQ = smem + C::kRingBytes;
  // Compacted valid slot numbers of the split, padded to whole 16-slot sub-tiles.
  SlotT* sSlot = reinterpret_cast<SlotT*>(sQ + C::kQBytes);
  int32_t* sScan = reinterpret_cast<int32_t*>(sSlot + kMaxSlotsPerSplit);
  float4* sXchg = C::kXchgOverQ ? reinterpret_cast<float4*>(sQ)  // (QSPLIT only)
                                 : reinterpret_cast<float4*>(sScan + 32);
  // TMA: full barrier of (slot lane, stage); both warps of the lane's pair arrive on it
  // with the byte count of their half of the sub-tile
  uint64_t* sBar = reinterpret_cast<uint64_t*>(sScan + 32);
  auto full_bar = [&](int lane_i, int stage) { return smem_addr(sBar + lane_i * STAGES + stage); };

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int wslot = warp % SL;  // which 16-slot sub-tile of a stage
  const int wpart = warp / SL;             // which warp of the slot lane
  const int wn = DSPLIT == 1 ? wpart : 0;  // first n8 tile of this warp
  const int wd = DSPLIT > 1 ? wpart : 0;   // which D range of the PV product (and of
                                           // Q K^T with QSPLIT)

  // ---- work unit -------------------------------------------------------------------
  // head_major: KV head slowest, so the CTAs resident at any time gather from one head's
  // slice of the cache (S rows per tensor) instead of all Hkv heads'; otherwise the
  // heads of a query row are neighbours and share its index row in L2.
  int u = blockIdx.x;
  const int split = u % p.nsplit;
  u /= p.nsplit;
  const int j = p.head_major ? u / p.Tq : u % p.Hkv;
  const int t = p.head_major ? u % p.Tq : u / p.Hkv;

  int width_t = p.W;
  if (p.width != nullptr) {
    int wv = p.width[t];
    if (wv < 0 || wv > p.W) {
      if (tid == 0 && p.err_word != nullptr) atomicOr(p.err_word, 2u);
      wv = wv < 0 ? 0 : p.W;
    }
    width_t = wv;
  }
  if constexpr (TMA) {
    // the 128-byte swizzle of the TMA destinations repeats every 1024 bytes: the ring must
    // start on that boundary (it does with no static shared memory; checked, not assumed)
    if ((smem_addr(smem) & 1023u) != 0) {
      if (tid == 0 && p.err_word != nullptr) atomicOr(p.err_word, 8u);
      return;
    }
    if (tid == 0) {
      for (int i = 0; i < SL * STAGES; ++i) mbar_init(smem_addr(sBar + i), C::kParts);
      mbar_init_fence();
    }
  }
  // ---- 0. the group's Q rows (commit group 0): in flight during the index work ---------
  const int G = p.G;
  const int64_t head0 = int64_t(j) * G;
  const uint32_t ring_s = smem_addr(ring);
  const uint32_t q_s = smem_addr(sQ);
  for (int i = tid; i < C::kQRows * kChunks; i += C::kThreads) {
    const int g = i / kChunks, c = i % kChunks;
    const bool ok = g < G;
    const uint16_t* src =
        p.q + int64_t(t) * p.q_stride_t + (head0 + (ok ? g : 0)) * p.q_stride_h + c * 8;
    cp_async_16(q_s + g * kRowBytes + ((c ^ (g & 7)) << 4), src, ok);
  }
  cp_async_commit();

  const int w0 = split * p.split_len;
  const int n_raw = max(min(w0 + p.split_len, width_t) - w0, 0);

  // ---- 1. stage and compact the slot indices -----------------------------------------
  int32_t* sRaw = reinterpret_cast<int32_t*>(ring);
  {
    const int32_t* idx_row = p.slot_idx + int64_t(t) * p.idx_stride_t + w0;
    for (int i = tid; i < n_raw; i += C::kThreads) sRaw[i] = __ldg(idx_row + i);
  }
  __syncthreads();
  const int per = (n_raw + C::kThreads - 1) / C::kThreads;
  const int b_i = min(tid * per, n_raw);
  const int e_i = min(b_i + per, n_raw);
  // An entry is valid when its whole block of p.block slots lies in the cache's global
  // extent (0 <= v < ent_total) and local when that block is held here (ent_lo <= v <
  // ent_hi); unsigned compares cover the negative values.
  const int block = p.block;
  const uint32_t ent_lo = uint32_t(p.ent_lo), ent_n = uint32_t(p.ent_hi - p.ent_lo);
  auto local = [&](int v) { return uint32_t(v) - ent_lo < ent_n; };
  int cnt = 0;
  bool bad = false;
  for (int i = b_i; i < e_i; ++i) {
    const int v = sRaw[i];
    bad |= v != -1 && uint32_t(v) >= uint32_t(p.ent_total);
    cnt += local(v) ? block : 0;
  }
  if (bad && p.err_word != nullptr) atomicOr(p.err_word, 1u);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sScan[warp] = incl;
  __syncthreads();
  int n_valid = 0, warp_off = 0;
#pragma unroll
  for (int w = 0; w < C::kWarps; ++w) {
    const int s = sScan[w];
    warp_off += (w < warp) ? s : 0;
    n_valid += s;
  }
  {
    int pos = warp_off + incl - cnt;
    for (int i = b_i; i < e_i; ++i) {
      const int v = sRaw[i];
      if (local(v)) {
        const uint32_t row = (uint32_t(v) - ent_lo) * uint32_t(block);  // row of this cache
        for (int e = 0; e < block; ++e) sSlot[pos++] = SlotT(row + uint32_t(e));
      }
    }
  }
  __syncthreads();  // sSlot complete, the ring is free again

  if (n_valid == 0) {  // fully masked row, zero width or an empty split (block-uniform)
    cp_async_wait<0>();  // the Q copy lands before this CTA's shared memory is released
    if (p.nsplit == 1 && !p.partial_out) {
      for (int i = tid; i < G * kChunks; i += C::kThreads) {
        const int g = i / kChunks, c = i % kChunks;
        uint16_t* dst = p.out + int64_t(t) * p.out_stride_t + (head0 + g) * p.out_stride_h + c * 8;
        *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
    } else {
      for (int g = tid; g < G; g += C::kThreads)
        p.ws_lse[(int64_t(split) * p.Tq + t) * p.Hq + head0 + g] = kNegInf;
      if (p.nsplit == 1) {  // a partial record (the combine skips it): O written as zeros
        // (the group's G rows are contiguous; 2- or 4-byte elements)
        const int64_t esz = p.rec_bf16 ? 2 : 4;
        uint4* z = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.part_o) +
                                            (int64_t(t) * p.Hq + head0) * kHeadDim * esz);
        const int n16 = int(G * kHeadDim * esz / 16);
        for (int i = tid; i < n16; i += C::kThreads) z[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }

  // ---- 2. the pipeline prologue -------------------------------------------------------

  const int n_stages = (n_valid + C::kRows - 1) / C::kRows;
  // Pad the offset list to whole 16-slot sub-tiles with the first slot: padding rows
  // hold finite data and are masked out of the softmax.
  for (int i = n_valid + tid; i < ((n_valid + 15) & ~15); i += C::kThreads) sSlot[i] = sSlot[0];
  // Gather addressing: global-space row bases, a row = base + slot * stride in bytes (one
  // 32x32->64-bit mad per row and tensor in the loop) and, per lane, the eight swizzled
  // chunk offsets (row & 7 is a compile-time
  // constant in the unrolled loop up to the warp's first row, 0, 4 or 8), so a
  // destination is a register plus an immediate.
  // An E4M3 row is 16 chunks: lanes 0-15 copy one row, lanes 16-31 the next.
  constexpr int kElem = KV8 ? 1 : 2;
  const uint32_t lchunk = KV8 ? uint32_t(lane & 15) : uint32_t(lane);
  const int lhalf = KV8 ? (lane >> 4) : 0;
  const uint64_t kg = static_cast<uint64_t>(__cvta_generic_to_global(
                          static_cast<const uint8_t*>(p.k_cache) + int64_t(j) * p.k_stride_h * kElem)) +
                      uint64_t(lchunk) * 16;
  const uint64_t vg = static_cast<uint64_t>(__cvta_generic_to_global(
                          static_cast<const uint8_t*>(p.v_cache) + int64_t(j) * p.v_stride_h * kElem)) +
                      uint64_t(lchunk) * 16;
  const uint32_t kstride = p.k_row_bytes, vstride = p.v_row_bytes;
  const uint32_t lane16 = lchunk << 4;
  // this lane's sub-tiles: [wslot][stage]; a warp pair splits the 16 rows 8 / 8
  const uint32_t sub_s = ring_s + wslot * STAGES * C::kSubBytes;
  constexpr int kLoadRows = 16 / C::kParts;
  const int row0 = wpart * kLoadRows;
  const uint32_t sub_rows = sub_s + (row0 + lhalf) * kKvRow;

  auto load_stage = [&](int s, int buf) {
    const int base = s * C::kRows + wslot * 16;
    if (base >= n_valid) return;  // an empty sub-tile is neither loaded nor read
    // rows i .. i + 3 of this warp's part of the sub-tile (one 16- or 8-byte read)
    auto slots4 = [&](int i, uint32_t (&sl)[4]) {
      if constexpr (SLOT16) {
        const uint2 s2 = reinterpret_cast<const uint2*>(sSlot + base + row0)[i / 4];
        sl[0] = s2.x & 0xffffu; sl[1] = s2.x >> 16; sl[2] = s2.y & 0xffffu; sl[3] = s2.y >> 16;
      } else {
        const uint4 s4 = reinterpret_cast<const uint4*>(sSlot + base + row0)[i / 4];
        sl[0] = s4.x; sl[1] = s4.y; sl[2] = s4.z; sl[3] = s4.w;
      }
    };
    if constexpr (TMA) {
      // each warp of the pair gathers its rows of K and V with TMA tile::gather4 (four
      // rows of one 128-byte column block per instruction), one instruction per lane, all
      // issued at once; lane 0 first announces the warp's bytes on the stage's full
      // barrier (which expects both warps of the pair)
      constexpr int kBlk = kKvRow / 128;
      constexpr int kBoxElems = KV8 ? 128 : 64;
      constexpr int kIssue = (kLoadRows / 4) * kBlk * 2;  // (row group, block, K or V)
      static_assert(kIssue <= 32, "one gather4 per lane");
      const uint32_t bar = full_bar(wslot, buf);
      if (lane == 0) mbar_arrive_expect_tx(bar, kLoadRows * kKvRow * 2);
      __syncwarp();
      if (lane < kIssue) {
        const int tv = lane & 1;               // 0: K, 1: V
        const int b = (lane >> 1) % kBlk;      // column block
        const int gi = (lane >> 1) / kBlk;     // row group of the warp's rows
        uint32_t sl[4];
        slots4(4 * gi, sl);
        const uint32_t d = sub_s + buf * C::kSubBytes + (row0 + 4 * gi) * C::kRowPitch +
                           b * C::kBlkPitch + tv * 16 * kKvRow;
        fence_proxy_async_smem();  // the pair's earlier reads of this buffer come first
        tma_gather4(d, tv ? &maps.v[j] : &maps.k[j], bar, b * kBoxElems, int32_t(sl[0]),
                    int32_t(sl[1]), int32_t(sl[2]), int32_t(sl[3]));
      }
    } else if constexpr (!KV8) {
      uint32_t kd[8];
#pragma unroll
      for (int m = 0; m < 8; ++m)  // (row0 & 7 is 0 for a pair's warps, 0 or 4 for a quad's)
        kd[m] = sub_rows + buf * C::kSubBytes + (lane16 ^ (uint32_t((m + row0) & 7) << 4));
#pragma unroll
      for (int i = 0; i < kLoadRows; i += 4) {
        uint32_t sl[4];
        slots4(i, sl);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t d = kd[(i + e) & 7] + (i + e) * kRowBytes;
          cp_async_16_global(d, kg + uint64_t(sl[e]) * kstride);
          cp_async_16_global(d + 16 * kRowBytes, vg + uint64_t(sl[e]) * vstride);
        }
      }
    } else {
      // instruction ip copies rows 2 ip + lhalf; their swizzle key is (2 ip + lhalf) & 7
      uint32_t kd[4];
#pragma unroll
      for (int m = 0; m < 4; ++m)
        kd[m] = sub_rows + buf * C::kSubBytes + (lane16 ^ (uint32_t((2 * m + lhalf) & 7) << 4));
#pragma unroll
      for (int i = 0; i < kLoadRows; i += 4) {
        uint32_t sl[4];
        slots4(i, sl);
        const uint32_t sa = lhalf ? sl[1] : sl[0];  // row i + lhalf
        const uint32_t sb = lhalf ? sl[3] : sl[2];  // row i + 2 + lhalf
        const int ip = i / 2;
        uint32_t d = kd[ip & 3] + ip * 2 * kKvRow;
        cp_async_16_global(d, kg + uint64_t(sa) * kstride);
        cp_async_16_global(d + 16 * kKvRow, vg + uint64_t(sa) * vstride);
        d = kd[(ip + 1) & 3] + (ip + 1) * 2 * kKvRow;
        cp_async_16_global(d, kg + uint64_t(sb) * kstride);
        cp_async_16_global(d + 16 * kKvRow, vg + uint64_t(sb) * vstride);
      }
    }
  };
  // makes a stage's sub-tile, loaded by one warp or a warp pair, visible to it
  auto lane_sync = [&]() {
    if constexpr (C::kParts == 1) {
      __syncwarp();
    } else {
      named_barrier_sync(1 + wslot, 32 * C::kParts);
    }
  };
  __syncthreads();  // the padded offset list is complete

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < n_stages) load_stage(s, s);
    cp_async_commit();
  }
  cp_async_wait<STAGES - 1>();  // the Q group is the oldest
  __syncthreads();

  // B fragments of Q^T for this warp's n8 tile, all 16 k-steps of D = 256.
  // (with QSPLIT, warp wd of a pair keeps the k-steps of its half of D only)
  uint32_t qf[TPW][kKS][2];
  const int ks0 = QSPLIT ? wd * kKS : 0;
  if constexpr (!KV8) {
#pragma unroll
    for (int nt = 0; nt < TPW; ++nt) {
#pragma unroll
      for (int kp = 0; kp < kKS / 2; ++kp) {
        const int g = lane & 7;
        const int c = 4 * kp + 2 * ks0 + (lane >> 3);
        uint32_t r[4];
        if constexpr (C::kQRows < NTILE * 8) {
          // heads past the tile (>= QROWS >= G) are padding: their fragments are zero, and
          // their row addresses stay inside the tile
          ldmatrix_x4(r, q_s + min((wn + nt) * 8 + g, C::kQRows - 1) * kRowBytes + ((c ^ g) << 4));
          if ((wn + nt) * 8 + (lane >> 2) >= C::kQRows) r[0] = r[1] = r[2] = r[3] = 0u;
        } else {
          ldmatrix_x4(r, q_s + ((wn + nt) * 8 + g) * kRowBytes + ((c ^ g) << 4));
        }
        qf[nt][2 * kp][0] = r[0];
        qf[nt][2 * kp][1] = r[1];
        qf[nt][2 * kp + 1][0] = r[2];
        qf[nt][2 * kp + 1][1] = r[3];
      }
    }
  } else {
    // f16 B fragments in the permuted k order of the E4M3 A fragments: for k-step ks
    // (D range 16 ks .. 16 ks + 15) lane l holds head l/4, elements 16 ks + 4 (l%4) + 0..3.
    bool q_big = false;
#pragma unroll
    for (int nt = 0; nt < TPW; ++nt) {
      const int n = (wn + nt) * 8 + (lane >> 2);
#pragma unroll
      for (int ks = 0; ks < kKS; ++ks) {
        const int c8 = 2 * (ks0 + ks) + ((lane & 3) >> 1);
        const uint2 v = *reinterpret_cast<const uint2*>(sQ + n * kRowBytes +
                                                        ((c8 ^ (n & 7)) << 4) + 8 * (lane & 1));
        const float f0 = bf16lo_to_f32(v.x), f1 = bf16hi_to_f32(v.x);
        const float f2 = bf16lo_to_f32(v.y), f3 = bf16hi_to_f32(v.y);
        q_big |= fmaxf(fmaxf(fabsf(f0), fabsf(f1)), fmaxf(fabsf(f2), fabsf(f3))) >= 65536.f;
        qf[nt][ks][0] = pack_f16x2(f0, f1);
        qf[nt][ks][1] = pack_f16x2(f2, f3);
      }
    }
    if (__any_sync(0xffffffffu, q_big) && lane == 0 && p.err_word != nullptr)
      atomicOr(p.err_word, 4u);
  }
  if constexpr (C::kXchgOverQ) __syncthreads();  // Q fragments loaded: the exchange may reuse sQ

  // ---- 3. main loop ------------------------------------------------------------------
  // per head tile nt of this warp: reference max (base 2) and this lane's share of the
  // running sums of heads 2(l%4), 2(l%4)+1, and the O^T accumulators
  float m0[TPW], m1[TPW], l0[TPW], l1[TPW];
  float o[TPW][kMT][4];
#pragma unroll
  for (int nt = 0; nt < TPW; ++nt) {
    m0[nt] = m1[nt] = kNegInf;
    l0[nt] = l1[nt] = 0.f;
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
  }

  // ldmatrix addressing.  Chunk c of a row sits at ((c ^ key) << 4), key = row & 7 =
  // lane & 7 for every row this lane addresses.  With c = 2 * step + hi (step = k-step
  // for K, m-tile for V; hi in {0, 1}) the XOR only touches the low three bits, so
  // (c ^ key) << 4 = 128 * (step >> 2) + swz[step & 3] (128 is the block pitch kBlkPitch
  // of the cp.async layout; the TMA layout has 2048): four per-lane offsets computed
  // once, and every ldmatrix address in the loop is a register plus an immediate.
  const int key = lane & 7;
  const int krow = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int khi = lane >> 4;
  const int vrow = (lane & 7) + ((lane >> 4) << 3);
  const int vhi = (lane >> 3) & 1;
  uint32_t kswz[4], vswz[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    kswz[m] = uint32_t(krow * C::kRowPitch + (((2 * m + khi) ^ key) << 4));
    // E4M3 V: the transposed loads use the K lane pattern (one chunk is one m-tile)
    vswz[m] = KV8 ? kswz[m] + 16 * kKvRow
                  : uint32_t(16 * kRowBytes + vrow * C::kRowPitch + (((2 * m + vhi) ^ key) << 4));
  }
  const float sl2 = p.scale_log2;
  bool tma_failed = false;

  for (int s = 0; s < n_stages; ++s) {
    cp_async_wait<STAGES - 2>();
    lane_sync();  // stage s landed for the whole slot lane; stage s-1 is consumed
    {
      const int sn = s + STAGES - 1;
      if (sn < n_stages) load_stage(sn, sn % STAGES);
      cp_async_commit();
    }
    const int buf = s % STAGES;
    const int base = s * C::kRows + wslot * 16;
    if (base >= n_valid) continue;  // warp-uniform: no valid slot in this sub-tile
    const uint32_t sub = sub_s + buf * C::kSubBytes;
    if constexpr (TMA) {
      // the stage's K and V rows of both warps have landed (use s / STAGES of the buffer);
      // a bounded wait: on a time-out the error bit is set, later waits are skipped and
      // the rows' outputs are not valid, but no warp leaves the pair's barriers (the
      // lanes agree on the outcome, so the warp stays converged)
      const bool landed =
          !tma_failed && mbar_wait(full_bar(wslot, buf), (s / STAGES) & 1, kMaxPolls);
      if (!__all_sync(0xffffffffu, landed)) tma_failed = true;
    }

    // S^T (16 slots x 8 heads) = K (16 x 256) * Q^T (256 x 8) per head tile; each K
    // fragment feeds every tile of the warp; two chains for ILP.
    uint32_t kt[4];
#pragma unroll
    for (int m = 0; m < 4; ++m)  // a k-step is 32 (16) bytes of a row: whole 128-byte blocks
      kt[m] = sub + kswz[m] + (ks0 * (KV8 ? 16 : 32) / 128) * C::kBlkPitch;
    float sa[TPW][4], sb[TPW][4];
#pragma unroll
    for (int nt = 0; nt < TPW; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = 0.f;
    if constexpr (!KV8) {
#pragma unroll
      for (int ks = 0; ks < kKS; ks += 2) {
        uint32_t a[4];
        ldmatrix_x4(a, kt[ks & 3] + C::kBlkPitch * (ks >> 2));
#pragma unroll
        for (int nt = 0; nt < TPW; ++nt) mma_bf16_16816(sa[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
        ldmatrix_x4(a, kt[(ks + 1) & 3] + C::kBlkPitch * ((ks + 1) >> 2));
#pragma unroll
        for (int nt = 0; nt < TPW; ++nt)
          mma_bf16_16816(sb[nt], a, qf[nt][ks + 1][0], qf[nt][ks + 1][1]);
      }
    } else {
      // one ldmatrix.x4 = two k-steps of 8-bit codes: r0 / r1 = rows 0-7 / 8-15 of
      // chunk 2 kq, r2 / r3 of chunk 2 kq + 1; lane l holds 4 codes of row l/4
#pragma unroll
      for (int kq = 0; kq < kKS / 2; ++kq) {
        uint32_t r[4], a[4];
        ldmatrix_x4(r, kt[kq & 3] + C::kBlkPitch * (kq >> 2));
        e4m3x4_to_f16x2x2(r[0], a[0], a[2]);
        e4m3x4_to_f16x2x2(r[1], a[1], a[3]);
#pragma unroll
        for (int nt = 0; nt < TPW; ++nt)
          mma_f16_16816(sa[nt], a, qf[nt][2 * kq][0], qf[nt][2 * kq][1]);
        e4m3x4_to_f16x2x2(r[2], a[0], a[2]);
        e4m3x4_to_f16x2x2(r[3], a[1], a[3]);
#pragma unroll
        for (int nt = 0; nt < TPW; ++nt)
          mma_f16_16816(sb[nt], a, qf[nt][2 * kq + 1][0], qf[nt][2 * kq + 1][1]);
      }
    }
    float sc[TPW][4];
#pragma unroll
    for (int nt = 0; nt < TPW; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = sa[nt][e] + sb[nt][e];
    // With one head tile per warp the first kVEarly V fragments of the sub-tile (bf16: m-tiles;
    // E4M3: raw codes of m-tile pairs) are read here, before the score exchange and the
    // softmax, so their shared-memory latency is hidden behind that work (the stage has
    // landed; the registers fit under the cap).  The E4M3 shape of one slot lane has the
    // registers for all of its pairs.  With two head tiles per
    // warp the registers are already at the cap and the early reads cost more than they hide.
    constexpr int kVEarly = TPW == 1 ? (KV8 ? (SL == QSA_FP8_EARLY_ALL_LANES ? kMT / 2 : 2) : 4) : 0;
    uint32_t vt[4];
    uint32_t vearly[kVEarly > 0 ? kVEarly : 1][4];
#pragma unroll
    for (int m = 0; m < 4; ++m) vt[m] = sub + vswz[m] + wd * (kMT / (KV8 ? 8 : 4)) * C::kBlkPitch;
#pragma unroll
    for (int mt = 0; mt < kVEarly; ++mt)
      ldmatrix_x4_trans(vearly[mt], vt[mt & 3] + C::kBlkPitch * (mt >> 2));
    if constexpr (QSPLIT && DSPLIT == 2) {
      // each warp of the pair holds the scores over its half of D: exchange and add in
      // a fixed order (low half + high half) so both warps hold the same scores
#pragma unroll
      for (int nt = 0; nt < TPW; ++nt)
        sXchg[((wslot * 2 + wd) * TPW + nt) * 32 + lane] =
            make_float4(sc[nt][0], sc[nt][1], sc[nt][2], sc[nt][3]);
      named_barrier_sync(1 + wslot, 64);
#pragma unroll
      for (int nt = 0; nt < TPW; ++nt) {
        const float4 t = sXchg[((wslot * 2 + (wd ^ 1)) * TPW + nt) * 32 + lane];
        if (wd == 0) {
          sc[nt][0] += t.x; sc[nt][1] += t.y; sc[nt][2] += t.z; sc[nt][3] += t.w;
        } else {
          sc[nt][0] = t.x + sc[nt][0]; sc[nt][1] = t.y + sc[nt][1];
          sc[nt][2] = t.z + sc[nt][2]; sc[nt][3] = t.w + sc[nt][3];
        }
      }
    } else if constexpr (QSPLIT) {
      // a quad: every warp holds the scores over its quarter of D; all four partial
      // scores are summed in the order of the quarters, so every warp holds the same sums
#pragma unroll
      for (int nt = 0; nt < TPW; ++nt)
        sXchg[((wslot * DSPLIT + wd) * TPW + nt) * 32 + lane] =
            make_float4(sc[nt][0], sc[nt][1], sc[nt][2], sc[nt][3]);
      named_barrier_sync(1 + wslot, 32 * DSPLIT);
#pragma unroll
      for (int nt = 0; nt < TPW; ++nt) {
        float4 a = sXchg[((wslot * DSPLIT) * TPW + nt) * 32 + lane];
#pragma unroll
        for (int w = 1; w < DSPLIT; ++w) {
          const float4 b = sXchg[((wslot * DSPLIT + w) * TPW + nt) * 32 + lane];
          a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        sc[nt][0] = a.x; sc[nt][1] = a.y; sc[nt][2] = a.z; sc[nt][3] = a.w;
      }
    }
    float x[TPW][4];
#pragma unroll
    for (int nt = 0; nt < TPW; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) x[nt][e] = sc[nt][e] * sl2;
    if (base + 16 > n_valid) {  // warp-uniform: only the last sub-tile has padding rows
      const int r0 = base + (lane >> 2);
#pragma unroll
      for (int nt = 0; nt < TPW; ++nt) {
        if (r0 >= n_valid) x[nt][0] = x[nt][1] = kNegInf;
        if (r0 + 8 >= n_valid) x[nt][2] = x[nt][3] = kNegInf;
      }
    }

    // Online softmax over the slot axis (rows); lanes sharing l%4 hold one head pair.
    // Lazy rescaling: the reference max m only moves when the chunk max exceeds it by
    // more than kRescaleLog2 (weights stay <= 2^kRescaleLog2, exact in fp32 and within
    // bf16 range); the final normalisation uses the same m for O and l, so the result
    // is unchanged.  A vote on the lanes' own maxima decides whether any head moves;
    // only then is the exact chunk max reduced over the slot axis (the decision is the
    // same as comparing the exact max).  The max is finite: row `base` is valid.
    bool need = false;
#pragma unroll
    for (int nt = 0; nt < TPW; ++nt)
      need |= fmaxf(x[nt][0], x[nt][2]) > m0[nt] + kRescaleLog2 ||
              fmaxf(x[nt][1], x[nt][3]) > m1[nt] + kRescaleLog2;
    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
      for (int nt = 0; nt < TPW; ++nt) {
        float mx0 = fmaxf(x[nt][0], x[nt][2]), mx1 = fmaxf(x[nt][1], x[nt][3]);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = (mx0 > m0[nt] + kRescaleLog2) ? mx0 : m0[nt];
        const float mn1 = (mx1 > m1[nt] + kRescaleLog2) ? mx1 : m1[nt];
        const float al0 = fast_exp2(m0[nt] - mn0), al1 = fast_exp2(m1[nt] - mn1);  // -inf -> 0
        l0[nt] *= al0;
        l1[nt] *= al1;
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt) {
          o[nt][mt][0] *= al0;
          o[nt][mt][1] *= al1;
          o[nt][mt][2] *= al0;
          o[nt][mt][3] *= al1;
        }
        m0[nt] = mn0;
        m1[nt] = mn1;
      }
    }
    uint32_t b0[TPW], b1[TPW];
#pragma unroll
    for (int nt = 0; nt < TPW; ++nt) {
      uint32_t p01, p23;
      if constexpr (!KV8) {
        p01 = pack_bf16x2(fast_exp2(x[nt][0] - m0[nt]), fast_exp2(x[nt][1] - m1[nt]));
        p23 = pack_bf16x2(fast_exp2(x[nt][2] - m0[nt]), fast_exp2(x[nt][3] - m1[nt]));
        // the denominators sum the same bf16-rounded weights that multiply V
        l0[nt] += bf16lo_to_f32(p01) + bf16lo_to_f32(p23);
        l1[nt] += bf16hi_to_f32(p01) + bf16hi_to_f32(p23);
      } else {
        // f16 weights (<= 2^kRescaleLog2, in range) for the f16 P V product
        p01 = pack_f16x2(fast_exp2(x[nt][0] - m0[nt]), fast_exp2(x[nt][1] - m1[nt]));
        p23 = pack_f16x2(fast_exp2(x[nt][2] - m0[nt]), fast_exp2(x[nt][3] - m1[nt]));
        l0[nt] += f16lo_to_f32(p01) + f16lo_to_f32(p23);
        l1[nt] += f16hi_to_f32(p01) + f16hi_to_f32(p23);
      }
      // P^T as the B operand of the P V product
      b0[nt] = movmatrix_trans(p01);
      b1[nt] = movmatrix_trans(p23);
    }

    // O^T (this warp's D rows x 8) += V^T (D rows x 16) * P^T (16 x 8) per head tile;
    // each V fragment feeds every tile of the warp
    if constexpr (!KV8) {
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt) {
        uint32_t a[4];
        if (mt < kVEarly) {
          a[0] = vearly[mt][0]; a[1] = vearly[mt][1]; a[2] = vearly[mt][2]; a[3] = vearly[mt][3];
        } else {
          ldmatrix_x4_trans(a, vt[mt & 3] + C::kBlkPitch * (mt >> 2));
        }
#pragma unroll
        for (int nt = 0; nt < TPW; ++nt) mma_bf16_16816(o[nt][mt], a, b0[nt], b1[nt]);
      }
    } else {
      // m-tile = one 16-byte chunk of D.  Transposed 8-bit loads give lane l the codes
      // (slot 2(l%4) and 2(l%4)+1) x (d = 16 c + 2(l/4) and + 1); a byte permute pairs
      // the two slots of each d, so tile row l/4 is d = 16 c + 2(l/4) and row l/4 + 8
      // is d + 1.  r0 / r1: slots 0-7 / 8-15 of chunk 2 mq, r2 / r3 of chunk 2 mq + 1.
#pragma unroll
      for (int mq = 0; mq < kMT / 2; ++mq) {
        uint32_t r[4], a[4];
        if (mq < kVEarly) {
          r[0] = vearly[mq][0]; r[1] = vearly[mq][1]; r[2] = vearly[mq][2]; r[3] = vearly[mq][3];
        } else {
          ldmatrix_x4_trans(r, vt[mq & 3] + C::kBlkPitch * (mq >> 2));
        }
        e4m3x4_to_f16x2x2(byte_perm(r[0], 0u, 0x3120u), a[0], a[1]);
        e4m3x4_to_f16x2x2(byte_perm(r[1], 0u, 0x3120u), a[2], a[3]);
#pragma unroll
        for (int nt = 0; nt < TPW; ++nt) mma_f16_16816(o[nt][2 * mq], a, b0[nt], b1[nt]);
        e4m3x4_to_f16x2x2(byte_perm(r[2], 0u, 0x3120u), a[0], a[1]);
        e4m3x4_to_f16x2x2(byte_perm(r[3], 0u, 0x3120u), a[2], a[3]);
#pragma unroll
        for (int nt = 0; nt < TPW; ++nt) mma_f16_16816(o[nt][2 * mq + 1], a, b0[nt], b1[nt]);
      }
    }
  }
  cp_async_wait<0>();
  if constexpr (TMA) {
    if (tma_failed) {
      // bounded drain of this lane's gathers that may still be in flight, then report
      const int lane_stages = n_valid > wslot * 16 ? (n_valid - wslot * 16 + C::kRows - 1) / C::kRows : 0;
      for (int s = lane_stages > STAGES ? lane_stages - STAGES : 0; s < lane_stages; ++s)
        mbar_wait(full_bar(wslot, s % STAGES), (s / STAGES) & 1, kMaxPolls / 64);
      if (lane == 0 && p.err_word != nullptr) atomicOr(p.err_word, 8u);
    }
  }
  __syncthreads();  // every warp is done with the ring: reuse it for the merge

  // ---- 4. merge the warps of each n8 tile and write ------------------------------------
#pragma unroll
  for (int nt = 0; nt < TPW; ++nt) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0[nt] += __shfl_xor_sync(0xffffffffu, l0[nt], off);
      l1[nt] += __shfl_xor_sync(0xffffffffu, l1[nt], off);
    }
  }
  float* mbuf = reinterpret_cast<float*>(ring);
  constexpr int kTileFloats = C::kTileFloats;   // [8 heads][kMergeStride] O, then m[8], l[8]
  constexpr int kWarpFloats = TPW * kTileFloats;
  {
    const int g0 = 2 * (lane & 3);
    const int r8 = lane >> 2;
#pragma unroll
    for (int nt = 0; nt < TPW; ++nt) {
      float* mine = mbuf + warp * kWarpFloats + nt * kTileFloats;
#pragma unroll
      for (int mt = 0; mt < kMT; ++mt) {
        // rows r8 / r8 + 8 of the m-tile are d = 16 mt' + r8 / + 8 (bf16), or
        // d = 16 mt' + 2 r8 / + 1 (E4M3 order)
        constexpr int kHi = KV8 ? 1 : 8;
        const int d = 16 * (wd * kMT + mt) + (KV8 ? 2 * r8 : r8);
        mine[g0 * kMergeStride + d] = o[nt][mt][0];
        mine[(g0 + 1) * kMergeStride + d] = o[nt][mt][1];
        mine[g0 * kMergeStride + d + kHi] = o[nt][mt][2];
        mine[(g0 + 1) * kMergeStride + d + kHi] = o[nt][mt][3];
      }
      if (r8 == 0) {
        mine[8 * kMergeStride + g0] = m0[nt];
        mine[8 * kMergeStride + g0 + 1] = m1[nt];
        mine[8 * kMergeStride + 8 + g0] = l0[nt];
        mine[8 * kMergeStride + 8 + g0 + 1] = l1[nt];
      }
    }
  }
  __syncthreads();

  for (int it = tid; it < NTILE * 8 * 32; it += C::kThreads) {
    const int gg = it >> 5;  // head within the group (n-tile major)
    const int dg = it & 31;  // 8-wide d group
    if (gg >= G) continue;
    const int nt = gg >> 3, g = gg & 7;
    // the warps holding this (head, d) range, one per slot lane: the D-half's warp
    // (tile record nt) or the tile's warp (its only record)
    const int part = DSPLIT > 1 ? (dg * 8) / (kHeadDim / DSPLIT) : nt;
    const int trec = DSPLIT > 1 ? nt * kTileFloats : 0;
    float mstar = kNegInf;
#pragma unroll
    for (int w = 0; w < SL; ++w)
      mstar = fmaxf(mstar, mbuf[(part * SL + w) * kWarpFloats + trec + 8 * kMergeStride + g]);
    float lsum = 0.f;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int w = 0; w < SL; ++w) {
      const float* src = mbuf + (part * SL + w) * kWarpFloats + trec;
      const float sc = fast_exp2(src[8 * kMergeStride + g] - mstar);  // -inf -> 0
      lsum += sc * src[8 * kMergeStride + 8 + g];
      const float4 a = *reinterpret_cast<const float4*>(src + g * kMergeStride + dg * 8);
      const float4 b = *reinterpret_cast<const float4*>(src + g * kMergeStride + dg * 8 + 4);
      acc[0] += sc * a.x; acc[1] += sc * a.y; acc[2] += sc * a.z; acc[3] += sc * a.w;
      acc[4] += sc * b.x; acc[5] += sc * b.y; acc[6] += sc * b.z; acc[7] += sc * b.w;
    }
    const float inv = (KV8 ? p.v_scale : 1.f) / lsum;
    const int64_t h = head0 + gg;
    if (p.nsplit == 1 && !p.partial_out) {
      uint4 v;
      v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      v.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
      v.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
      *reinterpret_cast<uint4*>(p.out + int64_t(t) * p.out_stride_t + h * p.out_stride_h + dg * 8) = v;
    } else {
      const int64_t row = (int64_t(split) * p.Tq + t) * p.Hq + h;
      if (p.nsplit == 1 && p.rec_bf16) {  // the record itself, O in bf16 (RNE)
        uint4 v;
        v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        v.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
        v.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
        *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.part_o) + row * kHeadDim + dg * 8) = v;
      } else {
        float4* dst = reinterpret_cast<float4*>(p.ws_o + row * kHeadDim + dg * 8);
        dst[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        dst[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
      }
      if (dg == 0) p.ws_lse[row] = mstar + fast_log2(lsum);
    }
  }
}

// K2: out[t, h, :] = sum_s 2^(lse_s - lse*) O_s / sum_s 2^(lse_s - lse*), one warp per row.
// The lanes read the splits' LSEs side by side (lane i: splits i, i + 32, ...) and reduce
// their maximum; the weighted sum then runs over the splits in order, every lane adding
// its eight elements of D, with the partial rows read regardless of their weight (the
// buffers hold every split's row) so that the reads of several splits are in flight at
// once; a split with lse = -inf (empty, its row never written) is left out by a select.
// IN_BF16: the partial rows are bf16 (gathered context-parallel records), else fp32.
// With partial_out the result is one record (O fp32, or bf16 with rec_bf16, and its LSE).
// records whose rows a warp reads at once (8: the bf16 records of 8 ranks combine in 117 us
// instead of 134 at the long-prefill shape; fp32 records and split workspaces unchanged)
#ifndef QSA_COMBINE_UNROLL
#define QSA_COMBINE_UNROLL 8
#endif
constexpr int kCombineUnroll = QSA_COMBINE_UNROLL;
template <bool IN_BF16>
__global__ void __launch_bounds__(128) qsa_lse_combine_kernel(const FwdParams p) {
  const int64_t rows = int64_t(p.Tq) * p.Hq;
  const int64_t row = int64_t(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int ns = p.nsplit;
  float mstar = kNegInf;
  for (int s = lane; s < ns; s += 32) mstar = fmaxf(mstar, p.ws_lse[s * rows + row]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mstar = fmaxf(mstar, __shfl_xor_sync(0xffffffffu, mstar, off));
  const int64_t t = row / p.Hq, h = row % p.Hq;
  // writes eight elements of this lane: a record (fp32 or bf16) or the bf16 output
  auto store8 = [&](const float (&x)[8]) {
    uint4 v;
    v.x = pack_bf16x2(x[0], x[1]);
    v.y = pack_bf16x2(x[2], x[3]);
    v.z = pack_bf16x2(x[4], x[5]);
    v.w = pack_bf16x2(x[6], x[7]);
    if (p.partial_out && !p.rec_bf16) {
      float4* po = reinterpret_cast<float4*>(static_cast<float*>(p.part_o) + row * kHeadDim + lane * 8);
      po[0] = make_float4(x[0], x[1], x[2], x[3]);
      po[1] = make_float4(x[4], x[5], x[6], x[7]);
    } else if (p.partial_out) {
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.part_o) + row * kHeadDim + lane * 8) = v;
    } else {
      *reinterpret_cast<uint4*>(p.out + t * p.out_stride_t + h * p.out_stride_h + lane * 8) = v;
    }
  };
  if (mstar == kNegInf) {  // no valid slot in any split
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    store8(z);
    if (p.partial_out && lane == 0) p.part_lse[row] = kNegInf;
    return;
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  for (int s0 = 0; s0 < ns; s0 += 32) {
    const float lse_l = s0 + lane < ns ? p.ws_lse[(s0 + lane) * rows + row] : kNegInf;
    const int cnt = min(32, ns - s0);
#pragma unroll kCombineUnroll
    for (int i = 0; i < cnt; ++i) {
      const float lse = __shfl_sync(0xffffffffu, lse_l, i);
      const int64_t off = ((s0 + i) * rows + row) * kHeadDim + lane * 8;
      float x[8];
      if constexpr (IN_BF16) {
        const uint4 r = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(p.ws_o) + off);
        x[0] = bf16lo_to_f32(r.x); x[1] = bf16hi_to_f32(r.x);
        x[2] = bf16lo_to_f32(r.y); x[3] = bf16hi_to_f32(r.y);
        x[4] = bf16lo_to_f32(r.z); x[5] = bf16hi_to_f32(r.z);
        x[6] = bf16lo_to_f32(r.w); x[7] = bf16hi_to_f32(r.w);
      } else {
        const float4 a = reinterpret_cast<const float4*>(p.ws_o + off)[0];
        const float4 b = reinterpret_cast<const float4*>(p.ws_o + off)[1];
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
      }
      if (lse != kNegInf) {  // warp-uniform
        const float w = fast_exp2(lse - mstar);
        wsum += w;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += w * x[e];
      }
    }
  }
  const float inv = 1.f / wsum;
  float res[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) res[e] = acc[e] * inv;
  store8(res);
  // one normalised record of all splits: O and lse* + log2(sum of weights)
  if (p.partial_out && lane == 0) p.part_lse[row] = mstar + fast_log2(wsum);
}

// Shard compaction (context parallelism): one warp per query row reads the row's selected
// entries (up to its width, clamped as K1 does) 32 at a time, flags invalid values, and
// appends the entries held by this shard in their original order (a ballot and a prefix
// count per 32 entries).  K1 then runs on the compacted rows with the counts as widths and
// sees exactly the local entries it would have kept itself, in the same order.
__global__ void __launch_bounds__(128) qsa_shard_compact_kernel(const FwdParams p, int32_t* idx,
                                                                int32_t* count) {
  const int64_t t = int64_t(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (t >= p.Tq) return;
  const int lane = threadIdx.x & 31;
  int wv = p.W;
  if (p.width != nullptr) {
    wv = p.width[t];
    if (wv < 0 || wv > p.W) {
      if (lane == 0 && p.err_word != nullptr) atomicOr(p.err_word, 2u);
      wv = wv < 0 ? 0 : p.W;
    }
  }
  const int32_t* src = p.slot_idx + t * p.idx_stride_t;
  int32_t* dst = idx + t * int64_t(p.W);
  const uint32_t ent_lo = uint32_t(p.ent_lo), ent_n = uint32_t(p.ent_hi - p.ent_lo);
  const uint32_t below = (1u << lane) - 1u;
  // 256 entries per step: each lane's eight loads are in flight together, then the eight
  // 32-entry groups are appended in order
  constexpr int kUnroll = 8;
  int n = 0;
  bool bad = false;
  for (int base = 0; base < wv; base += 32 * kUnroll) {
    int v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = base + 32 * u + lane;
      v[u] = i < wv ? __ldg(src + i) : -1;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      bad |= v[u] != -1 && uint32_t(v[u]) >= uint32_t(p.ent_total);
      const bool loc = uint32_t(v[u]) - ent_lo < ent_n;
      const uint32_t m = __ballot_sync(0xffffffffu, loc);
      if (loc) dst[n + __popc(m & below)] = v[u];
      n += __popc(m);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0 && p.err_word != nullptr) atomicOr(p.err_word, 1u);
  if (lane == 0) count[t] = n;
}

template <int NTILE, int DSPLIT, int SL, int STAGES, int MINB, bool QSPLIT, bool KV8,
          bool SLOT16 = false, int QROWS = NTILE * 8, bool TMA = false>
cudaError_t launch_fwd(const FwdParams& p, cudaStream_t stream) {
  using C = Cfg<NTILE, DSPLIT, SL, STAGES, KV8, SLOT16, QROWS, TMA>;
  if (p.G > QROWS) return cudaErrorInvalidValue;  // the Q tile holds the whole group
  auto kern =
      qsa_sparse_attn_fwd_kernel<NTILE, DSPLIT, SL, STAGES, MINB, QSPLIT, KV8, SLOT16, QROWS, TMA>;
  TmaMaps maps{};
  if constexpr (TMA) {
    if (p.Hkv > kMaxTmaHeads || p.S <= 0) return cudaErrorInvalidValue;
    const int64_t elem = KV8 ? 1 : 2;
    for (int jh = 0; jh < p.Hkv; ++jh) {
      cudaError_t e = encode_row_gather_map(
          &maps.k[jh], static_cast<const uint8_t*>(p.k_cache) + jh * p.k_stride_h * elem,
          uint64_t(p.S), uint32_t(kHeadDim * elem), p.k_row_bytes);
      if (e == cudaSuccess)
        e = encode_row_gather_map(
            &maps.v[jh], static_cast<const uint8_t*>(p.v_cache) + jh * p.v_stride_h * elem,
            uint64_t(p.S), uint32_t(kHeadDim * elem), p.v_row_bytes);
      if (e != cudaSuccess) return e;
    }
  }
  // The shared-memory opt-in is a function attribute that lives in the CUDA context: set
  // it on the first launch in each context only (keyed by the context's unique ID, so a
  // device reset or a new context sets it again), so later calls (e.g. under stream
  // capture) are launches and nothing else.
  static std::atomic<uint64_t> configured_ctx[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t ctx = current_context_id();
  const bool cached = dev >= 0 && dev < 64 && ctx != 0 &&
                      configured_ctx[dev].load(std::memory_order_acquire) == ctx;
  if (!cached) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(C::kSmem));
    if (e != cudaSuccess) return e;
    // (the attribute call made the context current if no call had before)
    const uint64_t now = current_context_id();
    if (dev >= 0 && dev < 64 && now != 0) configured_ctx[dev].store(now, std::memory_order_release);
  }
  const unsigned grid = static_cast<unsigned>(int64_t(p.Tq) * p.Hkv * p.nsplit);
  kern<<<grid, C::kThreads, C::kSmem, stream>>>(p, maps);
  return cudaGetLastError();
}

// The same shape with the rows gathered by TMA tile::gather4 (use_tma) or by cp.async.
// Gather of the K / V rows per cache format: TMA tile::gather4 (1) or cp.async (0).
// Measured on the long prefill (bf16 2.03 vs 3.10 ms, E4M3 1.74 vs 2.56 ms, G = 12 4.52 vs
// 6.53 ms): cp.async for both; the TMA kernels stay buildable for measurement.
#ifndef QSA_TMA_E4M3
#define QSA_TMA_E4M3 0
#endif
#ifndef QSA_TMA_BF16
#define QSA_TMA_BF16 0
#endif

// (The TMA kernels are only compiled in when a build asks for them.)
template <int NTILE, int DSPLIT, int SL, int STAGES, int MINB, bool QSPLIT, bool KV8,
          bool SLOT16 = false, int QROWS = NTILE * 8>
cudaError_t launch_gather(const FwdParams& p, cudaStream_t stream, bool use_tma) {
  if constexpr ((KV8 && QSA_TMA_E4M3) || (!KV8 && QSA_TMA_BF16)) {
    if (use_tma)
      return launch_fwd<NTILE, DSPLIT, SL, STAGES, MINB, QSPLIT, KV8, SLOT16, QROWS, true>(p,
                                                                                          stream);
  }
  return launch_fwd<NTILE, DSPLIT, SL, STAGES, MINB, QSPLIT, KV8, SLOT16, QROWS, false>(p, stream);
}

// The two shapes (slot lanes x pipeline stages per lane x resident CTAs per SM, chosen by
// measurement): G <= 8: one n8 tile, slot lanes of one warp each; 8 < G <= 16: two n8
// tiles, slot lanes of a warp pair each.  Two CTAs per SM hide each other's prologue
// (index compaction, Q load, pipeline fill) and epilogue (warp merge, output write).
#ifndef QSA_SMALL_SL
#define QSA_SMALL_SL 3
#endif
#ifndef QSA_SMALL_STAGES
#define QSA_SMALL_STAGES 2
#endif
#ifndef QSA_SMALL_CTAS
#define QSA_SMALL_CTAS 2  // CTAs resident per SM
#endif
#ifndef QSA_FP8_SMALL_CTAS
#define QSA_FP8_SMALL_CTAS 2
#endif
#ifndef QSA_LARGE_SL
#define QSA_LARGE_SL 3
#endif
#ifndef QSA_LARGE_STAGES
#define QSA_LARGE_STAGES 2
#endif
#ifndef QSA_LARGE_CTAS
#define QSA_LARGE_CTAS 2
#endif
#ifndef QSA_SMALL_DSPLIT
#define QSA_SMALL_DSPLIT 2
#endif
#ifndef QSA_SMALL_QSPLIT
#define QSA_SMALL_QSPLIT true
#endif
// E4M3 caches: a sub-tile is half the bytes, so the same shared memory holds more slot
// lanes (G <= 8: four lanes of three stages, 16 warps per SM, measured best) or a deeper
// pipeline per lane.
#ifndef QSA_FP8_SMALL_SL
#define QSA_FP8_SMALL_SL 4
#endif
#ifndef QSA_FP8_SMALL_STAGES
#define QSA_FP8_SMALL_STAGES 3
#endif
#ifndef QSA_FP8_LARGE_SL
#define QSA_FP8_LARGE_SL 3
#endif
#ifndef QSA_FP8_LARGE_STAGES
#define QSA_FP8_LARGE_STAGES 4
#endif
using CfgSmall = Cfg<1, QSA_SMALL_DSPLIT, QSA_SMALL_SL, QSA_SMALL_STAGES>;
#ifndef QSA_LARGE_DSPLIT
#define QSA_LARGE_DSPLIT 2  // 8 < G <= 16: the pair splits D (2) or the head tiles (1)
#endif
constexpr bool kLargeQsplit = QSA_LARGE_DSPLIT == 2;
using CfgLarge = Cfg<2, QSA_LARGE_DSPLIT, QSA_LARGE_SL, QSA_LARGE_STAGES>;
using CfgSmall8 = Cfg<1, 2, QSA_FP8_SMALL_SL, QSA_FP8_SMALL_STAGES, true>;
using CfgLarge8 = Cfg<2, QSA_LARGE_DSPLIT, QSA_FP8_LARGE_SL, QSA_FP8_LARGE_STAGES, true>;
static_assert(CfgSmall::kSmem <= CfgSmall::kSmPerCta(QSA_SMALL_CTAS), "small shape: CTAs per SM");
static_assert(CfgLarge::kSmem <= CfgLarge::kSmPerCta(QSA_LARGE_CTAS), "large shape: CTAs per SM");
static_assert(CfgSmall8::kSmem <= CfgSmall8::kSmPerCta(QSA_FP8_SMALL_CTAS), "E4M3 small shape: CTAs per SM");
static_assert(CfgLarge8::kSmem <= CfgLarge8::kSmPerCta(QSA_LARGE_CTAS), "E4M3 large shape: CTAs per SM");

// Caches of at most 65,536 rows (the long prefill's among them): the compacted row list is
// 16-bit, which brings a CTA of two slot lanes of two stages to 73 KB, so three such CTAs
// (12 warps, as before) fit on an SM and hide one another's per-unit prologue and epilogue
// better than two CTAs of three lanes (measured: long prefill 2.016 vs 2.096 ms, 512-slot
// rows 0.317 vs 0.356 ms).  A CTA of two lanes takes ~1.4x as long per unit, so with few
// units the coarser waves lose: the shape is used from five waves of three CTAs per SM on
// (Hq 16, Hkv 2, W 2,051, S 65,536: 2,048 units 314 vs 306 us, 2,560 units 363 vs 381,
// 3,072 units 432 vs 454).  E4M3 caches take a shape of their own there (below), from four
// such waves on (2,048 units 227 vs 253 us, 1,280 units 191 vs 168); with fewer waves
// they keep four lanes of three stages, with the 16-bit list.
constexpr int64_t kRows16 = 65536;
#ifndef QSA_SHAPE16_MIN_WAVES
#define QSA_SHAPE16_MIN_WAVES 5
#endif
#ifndef QSA_FP8_SHAPE16_MIN_WAVES
#define QSA_FP8_SHAPE16_MIN_WAVES 4
#endif
constexpr int64_t kShape16MinWaves = QSA_SHAPE16_MIN_WAVES;
constexpr int64_t kFp8Shape16MinWaves = QSA_FP8_SHAPE16_MIN_WAVES;
#ifndef QSA_SMALL16_SL
#define QSA_SMALL16_SL 2
#endif
#ifndef QSA_SMALL16_STAGES
#define QSA_SMALL16_STAGES 2
#endif
#ifndef QSA_SMALL16_CTAS
#define QSA_SMALL16_CTAS 3
#endif
#ifndef QSA_SMALL16_DSPLIT
#define QSA_SMALL16_DSPLIT 2  // warps of a slot lane splitting D: a pair (2) or a quad (4)
#endif
// E4M3 caches in such launches: one slot lane (a warp pair) of two stages, 25 KB, eight
// CTAs per SM (long prefill 1.495 ms; two lanes of two stages at three or four CTAs 1.595,
// of four stages 1.738; one lane of three stages at six CTAs 1.684, of four at five 1.749)
#ifndef QSA_FP8_SMALL16_SL
#define QSA_FP8_SMALL16_SL 1
#endif
#ifndef QSA_FP8_SMALL16_STAGES
#define QSA_FP8_SMALL16_STAGES 2
#endif
#ifndef QSA_FP8_SMALL16_CTAS
#define QSA_FP8_SMALL16_CTAS 8
#endif
#ifndef QSA_LARGE16_CTAS
#define QSA_LARGE16_CTAS 3
#endif
// E4M3 caches, 8 < G <= 16, many-wave launches on caches of at most 65,536 rows: one slot
// lane of three stages (the merge buffer of two head tiles needs the third), 37 KB, six
// CTAs per SM (the causal batch with an E4M3 cache 4.005 vs 4.571 ms with the two-CTA
// shape of three lanes of four stages; one lane of three stages at five CTAs 4.081, of
// four stages at five 4.320, two lanes of four stages at two 4.961)
#ifndef QSA_FP8_LARGE16
#define QSA_FP8_LARGE16 1
#endif
#ifndef QSA_FP8_LARGE16_SL
#define QSA_FP8_LARGE16_SL 1
#endif
#ifndef QSA_FP8_LARGE16_STAGES
#define QSA_FP8_LARGE16_STAGES 3
#endif
#ifndef QSA_FP8_LARGE16_CTAS
#define QSA_FP8_LARGE16_CTAS 6
#endif
using CfgSmall16 = Cfg<1, QSA_SMALL16_DSPLIT, QSA_SMALL16_SL, QSA_SMALL16_STAGES, false, true>;
using CfgSmall8r16 = Cfg<1, 2, QSA_FP8_SMALL_SL, QSA_FP8_SMALL_STAGES, true, true>;
using CfgSmall8s16 = Cfg<1, 2, QSA_FP8_SMALL16_SL, QSA_FP8_SMALL16_STAGES, true, true>;
static_assert(CfgSmall16::kSmem <= CfgSmall16::kSmPerCta(QSA_SMALL16_CTAS), "16-bit shape: CTAs per SM");
static_assert(CfgSmall8s16::kSmem <= CfgSmall8s16::kSmPerCta(QSA_FP8_SMALL16_CTAS),
              "E4M3 three-CTA shape: CTAs per SM");
// 8 < G <= 12 on such caches: two slot lanes of two stages with a 12-row Q tile, three CTAs
// per SM (G = 12: 2.518 vs 2.609 ms for 8,000 query rows of a 12,288-slot cache, 1.289 vs
// 1.334 ms for 4,000 rows of 65,536 slots; G = 10 2.515 vs 2.604 ms).
#ifndef QSA_LARGE16_SL
#define QSA_LARGE16_SL 2
#endif
#ifndef QSA_LARGE16_STAGES
#define QSA_LARGE16_STAGES 2
#endif
#ifndef QSA_LARGE16_QROWS
#define QSA_LARGE16_QROWS 12
#endif
using CfgLarge16 = Cfg<2, 2, QSA_LARGE16_SL, QSA_LARGE16_STAGES, false, true, QSA_LARGE16_QROWS>;
static_assert(CfgLarge16::kSmem <= CfgLarge16::kSmPerCta(QSA_LARGE16_CTAS),
              "12-row two-tile shape: CTAs per SM");
static_assert(CfgSmall8r16::kSmem <= CfgSmall8r16::kSmPerCta(QSA_FP8_SMALL_CTAS),
              "E4M3 16-bit shape: CTAs per SM");

}  // namespace

KernelShape kernel_shape(int G) {
  if (G <= 8)
    return {1, QSA_SMALL_SL, CfgSmall::kThreads, CfgSmall::kRows, QSA_SMALL_STAGES, CfgSmall::kSmem,
            QSA_SMALL_CTAS};
  return {2, QSA_LARGE_SL, CfgLarge::kThreads, CfgLarge::kRows, QSA_LARGE_STAGES, CfgLarge::kSmem,
          QSA_LARGE_CTAS};
}

size_t workspace_lse_offset(int32_t Tq, int32_t Hq, int32_t nsplit) {
  const size_t o_bytes = size_t(nsplit) * size_t(Tq) * size_t(Hq) * kHeadDim * sizeof(float);
  return (o_bytes + 255) / 256 * 256;
}

size_t workspace_bytes_for(int32_t Tq, int32_t Hq, int32_t nsplit) {
  if (nsplit <= 1) return 0;
  const size_t lse_bytes = size_t(nsplit) * size_t(Tq) * size_t(Hq) * sizeof(float);
  return workspace_lse_offset(Tq, Hq, nsplit) + (lse_bytes + 255) / 256 * 256;
}

// Kernel shape of a call: by cache format and group size G; caches of at most 65,536 rows
// take the 16-bit row list, and with it, in launches of at least five (E4M3: four) waves of
// three CTAs per SM, the shapes of more resident CTAs (G <= 8, and 8 < G <= 12 for bf16
// caches).
cudaError_t launch_sparse_prefill(const FwdParams& p, cudaStream_t stream) {
  cudaError_t e;
  // every compacted row number is below the row count of this call's cache
  const bool rows16 = p.S <= kRows16;
  const int64_t grid = int64_t(p.Tq) * p.Hkv * p.nsplit;
  const bool shape16 = rows16 && p.num_sms > 0 &&
                       grid >= (p.kv_fp8 ? kFp8Shape16MinWaves : kShape16MinWaves) * p.num_sms * 3;
  // TMA tile::gather4 for the rows where it is the faster gather (per cache format; one
  // tensor map per KV head for K and V, so at most kMaxTmaHeads heads; an empty shard
  // (S == 0) gathers nothing and takes the cp.async kernel)
  const bool tma_shape = p.S > 0 && p.Hkv <= kMaxTmaHeads;
  const bool tma = tma_shape && (p.kv_fp8 ? QSA_TMA_E4M3 : QSA_TMA_BF16);
  if (p.kv_fp8) {
    if (p.G <= 8)
      e = shape16 ? launch_gather<1, 2, QSA_FP8_SMALL16_SL, QSA_FP8_SMALL16_STAGES,
                                  QSA_FP8_SMALL16_CTAS, true, true, true>(p, stream, tma)
          : rows16 ? launch_gather<1, 2, QSA_FP8_SMALL_SL, QSA_FP8_SMALL_STAGES, QSA_FP8_SMALL_CTAS,
                                   true, true, true>(p, stream, tma)
                   : launch_gather<1, 2, QSA_FP8_SMALL_SL, QSA_FP8_SMALL_STAGES, QSA_FP8_SMALL_CTAS,
                                   true, true>(p, stream, tma);
#if QSA_FP8_LARGE16
    else if (shape16)
      e = launch_gather<2, 2, QSA_FP8_LARGE16_SL, QSA_FP8_LARGE16_STAGES, QSA_FP8_LARGE16_CTAS,
                        true, true, true>(p, stream, tma);
#endif
    else if constexpr (QSA_LARGE_DSPLIT == 2)
      e = launch_gather<2, 2, QSA_FP8_LARGE_SL, QSA_FP8_LARGE_STAGES, QSA_LARGE_CTAS, true,
                        true>(p, stream, tma);
    else
      e = launch_fwd<2, QSA_LARGE_DSPLIT, QSA_FP8_LARGE_SL, QSA_FP8_LARGE_STAGES, QSA_LARGE_CTAS,
                     kLargeQsplit, true>(p, stream);
  } else {
    if (p.G <= 8)
      e = shape16 ? launch_gather<1, QSA_SMALL16_DSPLIT, QSA_SMALL16_SL, QSA_SMALL16_STAGES,
                                  QSA_SMALL16_CTAS, QSA_SMALL_QSPLIT, false, true>(p, stream, tma)
                  : launch_gather<1, 2, QSA_SMALL_SL, QSA_SMALL_STAGES, QSA_SMALL_CTAS,
                                  QSA_SMALL_QSPLIT, false>(p, stream, tma);
    else if (shape16 && p.G <= QSA_LARGE16_QROWS)
      e = launch_gather<2, 2, QSA_LARGE16_SL, QSA_LARGE16_STAGES, QSA_LARGE16_CTAS, true, false,
                        true, QSA_LARGE16_QROWS>(p, stream, tma);
    else if constexpr (QSA_LARGE_DSPLIT == 2)
      e = launch_gather<2, 2, QSA_LARGE_SL, QSA_LARGE_STAGES, QSA_LARGE_CTAS, true, false>(
          p, stream, tma);
    else
      e = launch_fwd<2, QSA_LARGE_DSPLIT, QSA_LARGE_SL, QSA_LARGE_STAGES, QSA_LARGE_CTAS,
                     kLargeQsplit, false>(p, stream);
  }
  if (e != cudaSuccess || p.nsplit == 1) return e;
  return launch_combine(p, stream);
}

size_t shard_compact_bytes(int32_t Tq, int32_t W) {
  const size_t idx_bytes = (size_t(Tq) * size_t(W) * 4 + 255) / 256 * 256;
  return idx_bytes + (size_t(Tq) * 4 + 255) / 256 * 256;
}

cudaError_t launch_shard_compact(const FwdParams& p, int32_t* idx, int32_t* count,
                                 cudaStream_t stream) {
  if (p.Tq == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((int64_t(p.Tq) + 3) / 4);
  qsa_shard_compact_kernel<<<grid, 128, 0, stream>>>(p, idx, count);
  return cudaGetLastError();
}

cudaError_t launch_combine(const FwdParams& p, cudaStream_t stream) {
  const int64_t rows = int64_t(p.Tq) * p.Hq;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((rows + 3) / 4);
  if (p.in_bf16)
    qsa_lse_combine_kernel<true><<<grid, 128, 0, stream>>>(p);
  else
    qsa_lse_combine_kernel<false><<<grid, 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace qsa
