// qsa_probe.cu -- the gather-rate probe: the data movement of K1 with no arithmetic, used
// to measure the SM-side roofline of the sparse-attention gather on the device at hand.
//
// Once the selected K/V rows are L2 hits (the long-prefill cache is about the size of
// B200's L2), the bound of the gather is not HBM but the rate at which the SMs can pull
// random 512-byte rows (256 for E4M3 codes) out of L2 into shared memory and read them
// back once for the tensor-core fragments.  This kernel does exactly that and nothing
// else: every warp runs a pipeline of 16-row sub-tiles (the sub-tile of K1's slot lanes)
// over rows drawn at random from an L2-resident buffer, lands each sub-tile in shared
// memory with the swizzle K1 uses, and (optionally) reads it back with ldmatrix.x4.
// Three ways of moving the rows are measured:
//   method 0  cp.async.cg, 16 bytes per lane (K1's loader);
//   method 1  TMA tile::gather4 (four rows x 128 bytes per instruction, 128-byte swizzle),
//             issued by one lane of each consumer warp, mbarrier completion;
//   method 2  the same TMA gathers issued by one dedicated producer warp per CTA for all
//             consumer warps, with full / empty mbarrier rings;
//   method 3  the TMA gathers of a sub-tile issued by several lanes of the consumer warp in
//             one warp instruction (one gather4 per lane).
// The caller times a launch with CUDA events; bytes moved = warps x iters x 16 x row bytes.
// Every mbarrier wait is bounded: on a time-out the kernel sets bit 0 of sink[0], waits
// (bounded) for the copies it has in flight and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "qsa_internal.h"
#include "qsa_probe.h"
#include "qsa_ptx.cuh"

namespace qsa {
namespace {

constexpr uint32_t kMaxPolls = 1u << 22;

struct ProbeParams {
  const uint8_t* src;
  uint32_t rows;        // rows of the source buffer
  uint32_t pitch;       // bytes between consecutive rows
  int32_t iters;        // sub-tiles per consumer warp
  int32_t warps;        // consumer warps per CTA
  uint32_t seed;
  uint32_t* sink;       // [0]: error bits; [1 + ...]: reduction sink (never equal in practice)
};

// Row numbers: a warp-uniform linear congruential sequence mapped onto [0, rows).
__device__ __forceinline__ uint32_t next_row(uint32_t& h, uint32_t rows) {
  h = h * 1664525u + 1013904223u;
  return __umulhi(h, rows);
}

template <int METHOD, int READ, int ROWB, int STAGES>
__global__ void __launch_bounds__(512, 1)
    qsa_probe_gather_kernel(const ProbeParams p, const __grid_constant__ CUtensorMap tmap) {
  constexpr int kSub = 16 * ROWB;     // one 16-row sub-tile
  constexpr int kCpr = ROWB / 16;     // 16-byte chunks per row
  constexpr int kBlk = ROWB / 128;    // 128-byte column blocks per row (TMA layout)
  constexpr int kBoxElems = 128 / (ROWB / 256);  // one block in elements (bf16 or bytes)
  extern __shared__ __align__(1024) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const bool producer = METHOD == 2 && warp == p.warps;
  const int cw = producer ? 0 : warp;  // consumer warp index
  uint8_t* ring = smem + size_t(cw) * STAGES * kSub;
  // barriers after all rings: full[warp][stage], then empty[warp][stage]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(p.warps) * STAGES * kSub);
  auto full = [&](int w, int s) { return smem_addr(bars + w * STAGES + s); };
  auto empty = [&](int w, int s) { return smem_addr(bars + (p.warps + w) * STAGES + s); };
  if (METHOD != 0) {
    // the TMA destinations need the 1024-byte alignment of the 128-byte swizzle pattern;
    // anything else is reported and nothing is issued
    if ((smem_addr(smem) & 1023u) != 0) {
      if (threadIdx.x == 0) atomicOr(p.sink, 2u);
      return;
    }
    for (int i = threadIdx.x; i < p.warps * STAGES; i += blockDim.x) {
      mbar_init(full(i / STAGES, i % STAGES), 1);
      mbar_init(empty(i / STAGES, i % STAGES), 1);
    }
    mbar_init_fence();
  }
  __syncthreads();

  const uint32_t ring_s = smem_addr(ring);
  const uint64_t gsrc = static_cast<uint64_t>(__cvta_generic_to_global(p.src));
  uint32_t acc = 0;
  bool failed = false;

  // TMA issue of one sub-tile of consumer warp w into stage s (16 rows, kBlk blocks each)
  auto issue = [&](int w, int s, uint32_t& h) {
    const uint32_t dst = smem_addr(smem) + uint32_t((w * STAGES + s) * kSub);
    mbar_arrive_expect_tx(full(w, s), kSub);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const int32_t y0 = next_row(h, p.rows), y1 = next_row(h, p.rows);
      const int32_t y2 = next_row(h, p.rows), y3 = next_row(h, p.rows);
#pragma unroll
      for (int b = 0; b < kBlk; ++b)
        tma_gather4(dst + b * (16 * 128) + g * 512, &tmap, full(w, s), b * kBoxElems, y0, y1, y2,
                    y3);
    }
  };
  // Lane-parallel TMA issue (method 3): lane i < 4 * kBlk issues gather4 number i (row
  // group i / kBlk, column block i % kBlk) of the sub-tile, all in one warp instruction;
  // lane 0 announces the bytes first.  Every lane draws the sub-tile's 16 rows.
  auto issue_lanes = [&](int w, int s, uint32_t& h) {
    const uint32_t dst = smem_addr(smem) + uint32_t((w * STAGES + s) * kSub);
    uint32_t rv[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) rv[r] = next_row(h, p.rows);
    if (lane == 0) mbar_arrive_expect_tx(full(w, s), kSub);
    __syncwarp();
    if (lane < 4 * kBlk) {
      const int g = lane / kBlk, b = lane % kBlk;
      uint32_t y[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t v = rv[e];
#pragma unroll
        for (int gg = 1; gg < 4; ++gg) v = g == gg ? rv[4 * gg + e] : v;
        y[e] = v;
      }
      tma_gather4(dst + b * (16 * 128) + g * 512, &tmap, full(w, s), b * kBoxElems, int32_t(y[0]),
                  int32_t(y[1]), int32_t(y[2]), int32_t(y[3]));
    }
  };
  // read back one landed sub-tile with ldmatrix.x4 (16 rows, every chunk once).  With
  // READ == 2 every fragment is also compared with the source bytes of its row (the
  // warp replays the row sequence in `hv`), which checks the shared-memory layout; the
  // mismatches are counted in sink[1].
  uint32_t mismatches = 0;
  auto read_back = [&](uint32_t stage, uint32_t& hv) {
    uint32_t rowv[16];
    if constexpr (READ == 2) {
#pragma unroll
      for (int r = 0; r < 16; ++r) rowv[r] = next_row(hv, p.rows);
    }
#pragma unroll
    for (int m = 0; m < kCpr / 2; ++m) {
      const int r = lane & 15;
      const int c = 2 * m + (lane >> 4);
      uint32_t addr;
      if constexpr (METHOD == 0) {
        addr = stage + r * ROWB + ((c ^ (r & 7)) << 4);
      } else {
        addr = stage + (c >> 3) * (16 * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4);
      }
      uint32_t x[4];
      ldmatrix_x4(x, addr);
      acc ^= x[0] ^ x[1] ^ x[2] ^ x[3];
      if constexpr (READ == 2) {
        // fragment i of lane t: row 8 (i & 1) + t / 4, chunk 2 m + i / 2, bytes 4 (t % 4)..
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t row = rowv[8 * (i & 1) + (lane >> 2)];
          const uint32_t want = *reinterpret_cast<const uint32_t*>(
              p.src + uint64_t(row) * p.pitch + (2 * m + (i >> 1)) * 16 + 4 * (lane & 3));
          mismatches += want != x[i];
        }
      }
    }
  };

  if constexpr (METHOD == 0) {
    // K1's loader: lane l copies chunk l % kCpr of rows (l / kCpr) + (32 / kCpr) i
    uint32_t h = p.seed ^ (0x9e3779b9u * (blockIdx.x * p.warps + cw + 1));
    uint32_t hv = h;
    auto load = [&](int s) {
      const uint32_t st = ring_s + s * kSub;
      const int rsub = lane / kCpr, ch = lane % kCpr;
#pragma unroll
      for (int i = 0; i < 16; i += 32 / kCpr) {
        uint32_t rows_i[32 / kCpr];
#pragma unroll
        for (int e = 0; e < 32 / kCpr; ++e) rows_i[e] = next_row(h, p.rows);
        const int r = i + rsub;
        const uint32_t row = rows_i[rsub];
        cp_async_16_global(st + r * ROWB + ((ch ^ (r & 7)) << 4),
                           gsrc + uint64_t(row) * p.pitch + ch * 16);
      }
    };
#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
      if (s < p.iters) load(s);
      cp_async_commit();
    }
    for (int it = 0; it < p.iters; ++it) {
      cp_async_wait<STAGES - 2>();
      __syncwarp();
      const int nx = it + STAGES - 1;
      if (nx < p.iters) load(nx % STAGES);
      cp_async_commit();
      if (READ) read_back(ring_s + (it % STAGES) * kSub, hv);
    }
    cp_async_wait<0>();
  } else if constexpr (METHOD == 3) {
    uint32_t h = p.seed ^ (0x9e3779b9u * (blockIdx.x * p.warps + cw + 1));
    uint32_t hv = h;
    for (int s = 0; s < STAGES && s < p.iters; ++s) issue_lanes(cw, s, h);
    int it = 0;
    for (; it < p.iters; ++it) {
      const int s = it % STAGES;
      // every lane waits; the warp acts on the outcome as one (no lane leaves alone)
      if (!__all_sync(0xffffffffu, mbar_wait(full(cw, s), (it / STAGES) & 1, kMaxPolls))) {
        failed = true;
        break;
      }
      if (READ) read_back(ring_s + s * kSub, hv);
      __syncwarp();
      if (it + STAGES < p.iters) {
        fence_proxy_async_smem();
        issue_lanes(cw, s, h);
      }
    }
    if (failed) {  // drain what is still in flight (bounded)
      for (int k = it + 1; k < p.iters && k < it + STAGES; ++k)
        mbar_wait(full(cw, k % STAGES), (k / STAGES) & 1, kMaxPolls);
    }
  } else if constexpr (METHOD == 1) {
    uint32_t h = p.seed ^ (0x9e3779b9u * (blockIdx.x * p.warps + cw + 1));
    uint32_t hv = h;
    if (lane == 0)
      for (int s = 0; s < STAGES && s < p.iters; ++s) issue(cw, s, h);
    int it = 0;
    for (; it < p.iters; ++it) {
      const int s = it % STAGES;
      // every lane waits; the warp acts on the outcome as one (no lane leaves alone)
      if (!__all_sync(0xffffffffu, mbar_wait(full(cw, s), (it / STAGES) & 1, kMaxPolls))) {
        failed = true;
        break;
      }
      if (READ) read_back(ring_s + s * kSub, hv);
      __syncwarp();
      if (lane == 0 && it + STAGES < p.iters) {
        fence_proxy_async_smem();
        issue(cw, s, h);
      }
    }
    if (failed) {  // drain what is still in flight (bounded)
      for (int k = it + 1; k < p.iters && k < it + STAGES; ++k)
        mbar_wait(full(cw, k % STAGES), (k / STAGES) & 1, kMaxPolls);
    }
  } else {
    if (producer) {
      if (lane == 0) {
        uint32_t hs[16];
        for (int w = 0; w < p.warps; ++w) hs[w] = p.seed ^ (0x9e3779b9u * (blockIdx.x * p.warps + w + 1));
        int issued = 0;
        for (int it = 0; it < p.iters && !failed; ++it) {
          const int s = it % STAGES;
          for (int w = 0; w < p.warps; ++w) {
            if (!mbar_wait(empty(w, s), ((it / STAGES) & 1) ^ 1, kMaxPolls)) {
              failed = true;
              break;
            }
            issue(w, s, hs[w]);
          }
          issued = it + 1;
        }
        (void)issued;
      }
    } else {
      uint32_t hv = p.seed ^ (0x9e3779b9u * (blockIdx.x * p.warps + cw + 1));
      for (int it = 0; it < p.iters; ++it) {
        const int s = it % STAGES;
        if (!__all_sync(0xffffffffu, mbar_wait(full(cw, s), (it / STAGES) & 1, kMaxPolls))) {
          failed = true;
          break;
        }
        if (READ) read_back(ring_s + s * kSub, hv);
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(cw, s));
      }
      if (failed)  // the producer may still have this warp's next stages in flight (bounded)
        for (int s = 0; s < STAGES; ++s) mbar_wait(full(cw, s), 0, kMaxPolls / 64);
    }
  }
  if (failed && lane == 0) atomicOr(p.sink, 1u);
  if (READ == 2 && mismatches != 0) atomicAdd(p.sink + 1, mismatches);
  __syncthreads();  // nothing of this CTA is in flight past here on the normal path
  if (acc == 0x9e3779b9u) p.sink[2 + (threadIdx.x & 255)] = acc;
}

using ProbeKernel = void (*)(const ProbeParams, const CUtensorMap);

template <int METHOD, int READ, int ROWB>
ProbeKernel pick_stages(int stages) {
  switch (stages) {
    case 2: return qsa_probe_gather_kernel<METHOD, READ, ROWB, 2>;
    case 3: return qsa_probe_gather_kernel<METHOD, READ, ROWB, 3>;
    case 4: return qsa_probe_gather_kernel<METHOD, READ, ROWB, 4>;
  }
  return nullptr;
}

template <int METHOD, int ROWB>
ProbeKernel pick_read(int read, int stages) {
  return read == 0   ? pick_stages<METHOD, 0, ROWB>(stages)
         : read == 1 ? pick_stages<METHOD, 1, ROWB>(stages)
                     : pick_stages<METHOD, 2, ROWB>(stages);
}

template <int METHOD>
ProbeKernel pick(int read, int row_bytes, int stages) {
  return row_bytes == 512 ? pick_read<METHOD, 512>(read, stages) : pick_read<METHOD, 256>(read, stages);
}

}  // namespace

// 2-D tensor map over `rows` rows of `row_bytes` bytes, `pitch` bytes apart: elements of
// 2 bytes (512-byte rows) or 1 byte (256-byte rows), a box of one 128-byte block of one
// row, 128-byte swizzle -- the map of tile::gather4 row gathers.
cudaError_t encode_row_gather_map(CUtensorMap* map, const void* base, uint64_t rows,
                                  uint32_t row_bytes, uint64_t pitch) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static const EncodeFn encode = [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult r{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &r) != cudaSuccess ||
        r != cudaDriverEntryPointSuccess)
      fn = nullptr;
    return reinterpret_cast<EncodeFn>(fn);
  }();
  if (encode == nullptr) return cudaErrorNotSupported;
  const uint32_t elem = row_bytes / 256;  // 2 (bf16) or 1 (E4M3 codes)
  const cuuint64_t dims[2] = {256, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {128 / elem, 1};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                            2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace qsa

extern "C" qsa_status_t qsa_probe_gather(int32_t method, int32_t read_back, const void* src,
                                         int64_t rows, int64_t pitch_bytes, int32_t row_bytes,
                                         int32_t warps_per_cta, int32_t stages, int32_t ctas,
                                         int32_t iters, uint32_t seed, uint32_t* sink,
                                         void* stream) {
  using namespace qsa;
  if (method < 0 || method > 3 || read_back < 0 || read_back > 2 ||
      (row_bytes != 512 && row_bytes != 256) || stages < 2 ||
      stages > 4 || warps_per_cta < 1 || warps_per_cta > 15 || ctas < 1 || iters < 1 ||
      rows < 1 || rows > (int64_t(1) << 31) || pitch_bytes < row_bytes || pitch_bytes % 16 != 0 ||
      src == nullptr || sink == nullptr || (reinterpret_cast<uintptr_t>(src) & 15u) != 0) {
    set_error_detail("qsa_probe_gather: invalid arguments");
    return QSA_ERR_INVALID_ARG;
  }
  if (pitch_bytes > int64_t(UINT32_MAX) || rows * pitch_bytes > (int64_t(1) << 40)) {
    set_error_detail("qsa_probe_gather: buffer too large");
    return QSA_ERR_UNSUPPORTED;
  }
  const size_t smem = size_t(warps_per_cta) * stages * 16 * row_bytes +
                      (method != 0 ? size_t(2) * warps_per_cta * stages * 8 : 0);
  if (smem > 227 * 1024) {
    set_error_detail("qsa_probe_gather: %zu bytes of shared memory needed", smem);
    return QSA_ERR_INVALID_ARG;
  }
  CUtensorMap map{};
  if (method != 0) {
    const cudaError_t e = encode_row_gather_map(&map, src, uint64_t(rows), uint32_t(row_bytes),
                                                uint64_t(pitch_bytes));
    if (e != cudaSuccess) {
      set_error_detail("qsa_probe_gather: tensor map: %s", cudaGetErrorString(e));
      return QSA_ERR_CUDA;
    }
  }
  ProbeKernel k = method == 0   ? pick<0>(read_back, row_bytes, stages)
                  : method == 1 ? pick<1>(read_back, row_bytes, stages)
                  : method == 2 ? pick<2>(read_back, row_bytes, stages)
                                : pick<3>(read_back, row_bytes, stages);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) {
    set_error_detail("qsa_probe_gather: %s", cudaGetErrorString(e));
    return QSA_ERR_CUDA;
  }
  ProbeParams p{};
  p.src = static_cast<const uint8_t*>(src);
  p.rows = uint32_t(rows);
  p.pitch = uint32_t(pitch_bytes);
  p.iters = iters;
  p.warps = warps_per_cta;
  p.seed = seed;
  p.sink = sink;
  const int threads = 32 * (warps_per_cta + (method == 2 ? 1 : 0));
  k<<<ctas, threads, smem, static_cast<cudaStream_t>(stream)>>>(p, map);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error_detail("qsa_probe_gather: launch: %s", cudaGetErrorString(e));
    return QSA_ERR_CUDA;
  }
  return QSA_OK;
}
