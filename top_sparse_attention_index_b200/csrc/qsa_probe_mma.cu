// qsa_probe_mma.cu -- the shared-memory operand rate of the two MMA forms sm_100a offers
// the fused kernel: the warp-level form, whose operands a warp reads from shared memory
// with ldmatrix into registers (what K1 does with every gathered K and V row), and
// tcgen05.mma, issued by one thread, whose operands the tensor core reads from shared
// memory through matrix descriptors and whose accumulator lives in tensor memory.  The
// gathered rows are read from shared memory exactly once either way, so the form that
// reads shared memory faster at this path's shapes (slots x a group of 8-16 heads) is the
// one that can move the kernel's bound.  Entry point: include/qsa_probe.h.
#include <cuda_runtime.h>

#include <cstdint>

#include "qsa_internal.h"
#include "qsa_probe.h"

namespace {

constexpr int kUmmaM = 128;                  // rows of A (and of the accumulator)
constexpr int kUmmaSmem = 200 * 1024;        // 16 K-slices of A and B, one CTA per SM
constexpr uint32_t kUmmaMaxPolls = 1u << 26;  // bound of the completion wait
constexpr int kLdsmWarps = 16;
constexpr int kLdsmBytes = 64 * 1024;

__device__ __forceinline__ uint32_t sm_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor of a K-major bf16 tile without swizzle (core matrices of
// 8 rows x 16 bytes stored contiguously): start address, the byte distance between the two
// 16-byte K halves of a K = 16 slice (leading) and between 8-row groups (stride), all in
// 16-byte units, and the descriptor version bit of this architecture.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr, uint32_t lead, uint32_t stride) {
  return uint64_t((addr >> 4) & 0x3FFFu) | (uint64_t((lead >> 4) & 0x3FFFu) << 16) |
         (uint64_t((stride >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46);
}

// Instruction descriptor of kind::f16: fp32 accumulator, A and B bf16, both K-major, no
// negation, N / 8 and M / 16 in their fields.
__device__ __forceinline__ uint32_t f16_instr_desc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// One thread issues `rounds` x 16 MMAs of M = 128, N, K = 16 (one per K-slice of the tiles)
// back to back, accumulating into one tensor-memory tile; tcgen05.commit signals an
// mbarrier when they are done (bounded wait).  A and B hold bf16 ones, so every
// accumulator element ends at rounds x 256, which each thread checks for its lane.
template <int N>
__global__ void __launch_bounds__(128, 1) qsa_probe_umma_kernel(int rounds, long long* out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ uint32_t tmem_base;
  __shared__ __align__(8) uint64_t done_bar;
  constexpr int kAStep = kUmmaM * 32, kBStep = N * 32;  // one K-slice: rows x 16 bf16
  constexpr uint32_t kCols = N < 32 ? 32 : N;           // allocation: a power of two >= 32
  static_assert(16 * (kAStep + kBStep) <= kUmmaSmem, "16 K-slices of A and B fit");
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < 16 * (kAStep + kBStep) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem)[i] = 0x3F803F80u;  // two bf16 ones
  if (tid == 0) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sm_addr(&done_bar)));
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // operands visible to the MMA
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     sm_addr(&tmem_base)), "r"(kCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tacc = tmem_base;
  if (tid == 0) {
    const uint32_t idesc = f16_instr_desc(kUmmaM, N);
    const uint32_t a0 = sm_addr(smem), b0 = a0 + 16 * kAStep;
    const long long c0 = clock64();
    for (int r = 0; r < rounds; ++r) {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const uint64_t ad = kmajor_desc(a0 + k * kAStep, 128, 256);
        const uint64_t bd = kmajor_desc(b0 + k * kBStep, 128, 256);
        const uint32_t accumulate = (r | k) != 0;
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(
                tacc), "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate), "r"(0u));  // no lane disabled
      }
    }
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            sm_addr(&done_bar))
        : "memory");
    uint32_t done = 0;
    for (uint32_t n = 0; !done && n < kUmmaMaxPolls; ++n)
      asm volatile(
          "{\n\t.reg .pred q;\n\tmbarrier.try_wait.parity.shared::cta.b64 q, [%1], 0;\n\t"
          "selp.u32 %0, 1, 0, q;\n\t}\n"
          : "=r"(done)
          : "r"(sm_addr(&done_bar)));
    if (!done) atomicOr(reinterpret_cast<unsigned long long*>(out), 1ull);
    out[2 + blockIdx.x] = clock64() - c0;
  }
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  uint32_t v;  // column 0 of this thread's lane (warp w reads lanes 32 w .. 32 w + 31)
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];"
               : "=r"(v)
               : "r"(tacc + (uint32_t(warp * 32) << 16)));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  if (__uint_as_float(v) != float(rounds) * 256.f)
    atomicAdd(reinterpret_cast<unsigned long long*>(out + 1), 1ull);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tacc), "r"(kCols));
}

// 16 warps read a 64 KiB window with ldmatrix.x4 (512 bytes per warp instruction), each
// warp starting at its own 4 KiB offset, `rounds` passes of 64 KiB per warp.
__global__ void __launch_bounds__(32 * kLdsmWarps, 1) qsa_probe_ldsm_kernel(int rounds, long long* out) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kLdsmBytes / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(smem)[i] = i;
  __syncthreads();
  const uint32_t base = sm_addr(smem) + lane * 16;
  uint32_t x = 0;
  const long long c0 = clock64();
  for (int r = 0; r < rounds; ++r) {
#pragma unroll 8
    for (int j = 0; j < kLdsmBytes / 512; ++j) {
      uint32_t a, b, c, d;
      asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                   : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
                   : "r"(base + ((j * 512 + warp * 4096) & (kLdsmBytes - 1))));
      x ^= a ^ b ^ c ^ d;
    }
  }
  __syncthreads();
  if (tid == 0) out[2 + blockIdx.x] = clock64() - c0;
  if (x == 0x9E3779B9u) atomicAdd(reinterpret_cast<unsigned long long*>(out + 1), 0ull);  // keeps x live
}

template <int N>
cudaError_t launch_umma(int rounds, int ctas, long long* out, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(qsa_probe_umma_kernel<N>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kUmmaSmem);
  if (e != cudaSuccess) return e;
  qsa_probe_umma_kernel<N><<<ctas, 128, kUmmaSmem, stream>>>(rounds, out);
  return cudaGetLastError();
}

}  // namespace

extern "C" qsa_status_t qsa_probe_mma_operands(int32_t method, int32_t n, int32_t rounds,
                                               int32_t ctas, int64_t* out, void* stream) {
  const bool n_ok = method == 0 ? n == 0 : (n == 16 || n == 32 || n == 64 || n == 128 || n == 256);
  if (method < 0 || method > 1 || !n_ok || rounds < 1 || rounds > 65536 || ctas < 1 ||
      ctas > 4096 || out == nullptr || (reinterpret_cast<uintptr_t>(out) & 7u) != 0) {
    qsa::set_error_detail("qsa_probe_mma_operands: invalid arguments");
    return QSA_ERR_INVALID_ARG;
  }
  const auto st = static_cast<cudaStream_t>(stream);
  auto* o = reinterpret_cast<long long*>(out);
  cudaError_t e;
  if (method == 0) {
    e = cudaFuncSetAttribute(qsa_probe_ldsm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kLdsmBytes);
    if (e == cudaSuccess) {
      qsa_probe_ldsm_kernel<<<ctas, 32 * kLdsmWarps, kLdsmBytes, st>>>(rounds, o);
      e = cudaGetLastError();
    }
  } else {
    e = n == 16    ? launch_umma<16>(rounds, ctas, o, st)
        : n == 32  ? launch_umma<32>(rounds, ctas, o, st)
        : n == 64  ? launch_umma<64>(rounds, ctas, o, st)
        : n == 128 ? launch_umma<128>(rounds, ctas, o, st)
                   : launch_umma<256>(rounds, ctas, o, st);
  }
  if (e != cudaSuccess) {
    qsa::set_error_detail("qsa_probe_mma_operands: %s", cudaGetErrorString(e));
    (void)cudaGetLastError();  // not reported again by a later launch's check
    return QSA_ERR_CUDA;
  }
  return QSA_OK;
}
