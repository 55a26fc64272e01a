// mma_peak.cu - dense tensor-core throughput of single tcgen05.mma shapes on
// one B200, for the roofline denominators of the block-scaled expert FFN
// (MXFP8 x MXFP4 on kind::mxf8f6f4) and of an all-FP4 path (kind::mxf4).
//
// One CTA per SM issues back-to-back MMAs on operands that stay in shared
// memory (no loads inside the timed loop), into `chains` accumulators in
// turn, and commits once at the end; the caller times the launch with CUDA
// events. The result is the instruction throughput of the shape: the ceiling
// a GEMM kernel of that kind can approach, not a GEMM measurement. Run at the
// bf16 kind as well, it gives the ratio by which a measured bf16 GEMM peak
// scales to the other kinds.
//
// Shapes: M = 128 (cta_group::1), N = n, K = 16 (kind::f16, bf16 x bf16),
// 32 (kind::mxf8f6f4, e2m1 x e4m3, one e8m0 scale per 32 along K) or 64
// (kind::mxf4, e2m1 x e2m1 packed two per byte, one e8m0 scale per 32).
// Operand bytes are a fixed pattern (finite in every format); scales 2^0.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// K-major operand rows of 128 bytes with the 128-byte swizzle, 8-row groups
// 1024 bytes apart (start >> 4, stride >> 4, version 1, layout 128B swizzle).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (1ull << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
// 32 rows x 16 bytes without swizzle: the source of a scale-atom copy.
__device__ __forceinline__ uint64_t desc_rows16(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128u >> 4) << 32) |
         (1ull << 46);
}

// Instruction descriptors (fields of the tcgen05 instruction descriptor:
// formats at bits 7-9 / 10-12, N >> 3 at 17-22, scale type at 23, M >> 4 at
// 24-28; K-major operands, dense).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {  // D fp32, A/B bf16
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_mxf8f6f4_e2m1_e4m3(int M, int N) {  // e8m0 scales
  return (5u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_mxf4_e2m1(int M, int N) {  // e8m0 scales, K = 64
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

constexpr long long kWaitLimit = 8000000000LL;  // cycles (about 4 s): the commit wait gives up after

template <int KIND>
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc,
                                    uint32_t sfa, uint32_t sfb) {
  if constexpr (KIND == 0) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
  } else if constexpr (KIND == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
        : "memory");
  }
}

// Shared memory: A 128 rows x 128 B, B 256 rows x 128 B, three 512-byte
// scale atoms (A, B rows 0-127, B rows 128-255), 1024-byte aligned.
constexpr int kABytes = 128 * 128, kBBytes = 256 * 128, kAtom = 512;
constexpr int kSmem = kABytes + kBBytes + 3 * kAtom + 1024 + 64;
// TMEM: 512 columns; accumulators from column 0 (chains x n <= 512, or 384
// for the block-scaled kinds), scale atoms at 384 (A), 392 and 396 (B).
constexpr uint32_t kSfA = 384, kSfB = 392;

// Operand patterns (`mode` bits 0-3) that replay how the expert-FFN kernels
// issue their MMAs; bit 4 adds a commit after every 8 MMAs (as a pipeline
// releases its stages):
//   0  every chain reads the same A and B, the K step rotating per round;
//   1  two 128-row A tiles (one per chain) against one B tile of n rows, the
//      same K step for both chains (gate and up of one token tile);
//   2  the K step rotating per MMA, so chain c takes every chains-th step (a
//      K split into partial sums).
constexpr int kModeCommit = 16;

template <int KIND>
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int n, int chains, int iters, int mode,
                                                          int* status) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = sm;
  uint8_t* sB = sm + kABytes;
  uint8_t* atoms = sB + kBBytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(atoms + 3 * kAtom);  // [0] final, [1] per-8 commits
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 2);
  const int tid = threadIdx.x;
  // operands: 0x22 bytes (e2m1 1.0 in each nibble; e4m3 2^-6 x 1.25), bf16 1.0
  const uint32_t fill = KIND == 0 ? 0x3F803F80u : 0x22222222u;
  for (int i = tid; i < (kABytes + kBBytes) / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(sm)[i] = fill;
  for (int i = tid; i < 3 * kAtom / 4; i += blockDim.x) reinterpret_cast<uint32_t*>(atoms)[i] = 0x7F7F7F7Fu;
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar + 1)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (tid < 32) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tslot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tbase = *tslot;
  if (tid == 0) {
    if (KIND != 0) {
      for (int a = 0; a < 3; ++a) {
        const uint32_t col = a == 0 ? kSfA : kSfB + 4 * (a - 1);
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tbase + col),
                     "l"(desc_rows16(smem_u32(atoms + a * kAtom)))
                     : "memory");
      }
    }
    const uint32_t idesc = KIND == 0 ? idesc_f16(128, n)
                         : KIND == 1 ? idesc_mxf8f6f4_e2m1_e4m3(128, n)
                                     : idesc_mxf4_e2m1(128, n);
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    const int pattern = mode & 15;
    int issued = 0;
    for (int i = 0; i < iters; ++i) {
      for (int c = 0; c < chains; ++c) {
        // the four K steps of a 128-byte row
        const uint32_t koff = static_cast<uint32_t>((pattern == 2 ? i * chains + c : i) & 3) * 32;
        uint32_t a = a0, b = b0;
        if (pattern == 1) {  // chain c's 128-row tile in the 256-row region, the n-row tile in the other
          a = b0 + static_cast<uint32_t>(c & 1) * (128 * 128);
          b = a0;
        }
        mma<KIND>(tbase + static_cast<uint32_t>(c * n), desc_sw128(a + koff), desc_sw128(b + koff), idesc,
                  i > 0 ? 1u : 0u, tbase + kSfA, tbase + kSfB);
        if ((mode & kModeCommit) && (++issued & 7) == 0)
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           smem_u32(bar + 1))
                       : "memory");
      }
    }
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
    // bounded wait for the MMAs to retire
    const long long t0 = clock64();
    uint32_t ok = 0;
    while (!ok) {
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}\n"
          : "=r"(ok)
          : "r"(smem_u32(bar))
          : "memory");
      if (!ok && clock64() - t0 > kWaitLimit) {
        atomicExch(status, 1);
        break;
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (tid < 32) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tbase) : "memory");
  }
}

}  // namespace

extern "C" {

// Launches `ctas` CTAs (one per SM) of the probe: kind 0 = bf16 (kind::f16),
// 1 = e2m1 x e4m3 (kind::mxf8f6f4), 2 = e2m1 x e2m1 (kind::mxf4); M = 128,
// `mode` an operand pattern (above; pattern 1 needs n <= 128),
// N = n (16..256, a multiple of 16), `chains` accumulators in turn
// (chains * n <= 512 for bf16, <= 384 for the block-scaled kinds), `iters`
// MMAs per chain. status (device int, zeroed by
// the caller) becomes 1 if a CTA gave up waiting for its MMAs. Returns a
// cudaError_t value (0 = launched); asynchronous on `stream`.
__attribute__((visibility("default"))) int sgl_mma_peak(int kind, int n, int chains, int iters, int ctas,
                                                        int mode, int* status, void* stream) {
  // block-scaled kinds keep TMEM columns 384-399 for their scale atoms
  const int max_cols = kind == 0 ? 512 : 384;
  const int pattern = mode & 15;
  if (kind < 0 || kind > 2 || n < 16 || n > 256 || n % 16 != 0 || chains < 1 || chains * n > max_cols ||
      iters < 1 || ctas < 1 || status == nullptr || pattern > 2 || (mode & ~(15 | kModeCommit)) != 0 ||
      (pattern == 1 && n > 128))
    return static_cast<int>(cudaErrorInvalidValue);
  void (*k)(int, int, int, int, int*) =
      kind == 0 ? mma_peak_kernel<0> : kind == 1 ? mma_peak_kernel<1> : mma_peak_kernel<2>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return static_cast<int>(e);
  k<<<ctas, 128, kSmem, static_cast<cudaStream_t>(stream)>>>(n, chains, iters, mode, status);
  return static_cast<int>(cudaGetLastError());
}

}  // extern "C"
