// microbench.cu -- the library's own peak probes, so that every roofline
// fraction can also be stated against a number this code measured on the
// GPU at hand:
//   * a dense FP8 tensor-core loop: one CTA per SM issuing back-to-back
//     tcgen05.mma.kind::f8f6f4 (M 128, N 256, K 32, e4m3 x e4m3 -> fp32)
//     from operands resident in shared memory, no data movement.  The
//     tensor pipe's rate depends on the operand values (its power draw sets
//     the clock under the power limit), so the operands are chosen: the e4m3
//     codes of Gaussian values scaled like statically quantised activations
//     and weights (amax near 448: sigma 100, random signs, every mantissa
//     bit in play), or low-toggle codes (non-negative, one exponent bit
//     cleared), which draw less power and run faster;
//   * a device-to-device copy over buffers far larger than L2.
// The caller times the launches (CUDA events) and converts: the MMA loop does
// 2 * 128 * 256 * 32 * 4 * iters flops per CTA; the copy moves 2 * bytes.

#include "frt_common.cuh"
#include "frt_sm100.cuh"

namespace frt {
namespace {

constexpr int kMbThreads = 128;
constexpr int kMbA = 128 * 128;  // 128 rows x 128 K-bytes
constexpr int kMbB = 256 * 128;  // 256 rows x 128 K-bytes
constexpr uint64_t kMbWaitNs = 4000000000ull;

__global__ void __launch_bounds__(kMbThreads, 1) mma_peak_kernel(int iters, int operands,
                                                                 int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kMbA;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sB + kMbB);
  uint32_t* holder = reinterpret_cast<uint32_t*>(bar + 1);
  // operands: pseudo-random finite e4m3 codes (the tensor pipe's power
  // draw, hence its clock, depends on the data)
  for (int i = threadIdx.x; i < (kMbA + kMbB) / 4; i += kMbThreads) {
    uint32_t h = uint32_t(i) * 2654435761u + blockIdx.x * 40503u;
    h ^= h >> 15;
    h *= 2246822519u;
    h ^= h >> 13;
    if (operands == FRT_PEAK_OPERANDS_GAUSSIAN) {
      // four codes of N(0, 100^2) values: each the sum of four uniform
      // bytes (Irwin-Hall, mean 510, sd 147.8) standardised and scaled,
      // rounded to e4m3 with saturation at +-448 (never NaN)
      float z[8];
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        uint32_t g = h * 0x9E3779B1u + uint32_t(b + 1) * 0x85EBCA77u;
        g ^= g >> 15;
        g *= 0x2C1B3C6Du;
        g ^= g >> 12;
        g *= 0x297A2D39u;
        g ^= g >> 15;
        const float u = float(g & 0xFFu) + float((g >> 8) & 0xFFu) + float((g >> 16) & 0xFFu) +
                        float(g >> 24);
        z[b] = (u - 510.0f) * (100.0f / 147.8f);
      }
      h = pack8_e4m3(z).x;
    } else {
      h &= 0x6F6F6F6Fu;  // clears bits 4 and 7 of every byte: never 0x7F/0xFF (NaN)
    }
    reinterpret_cast<uint32_t*>(smem)[i] = h;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(holder, 256);
    tmem_relinquish();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *holder;
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = idesc_e4m3_f32(128, 256);
    const uint64_t ad = sdesc_k_sw128(smem_u32(sA)), bd = sdesc_k_sw128(smem_u32(sB));
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        umma_e4m3(tmem, ad + 2 * k, bd + 2 * k, idesc, (it > 0 || k > 0) ? 1u : 0u);
    }
    umma_commit(bar);
    if (!mbar_wait_bounded(bar, 0, kMbWaitNs, nullptr) && status)
      atomicExch(status, FRT_ETIMEOUT);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

#ifndef FRT_COPY_UNROLL
#define FRT_COPY_UNROLL 8
#endif
#ifndef FRT_COPY_BLOCKS_PER_SM
#define FRT_COPY_BLOCKS_PER_SM 16
#endif
#ifndef FRT_COPY_MODE
#define FRT_COPY_MODE 0
#endif
__device__ __forceinline__ uint4 cp_ld(const uint4* p) {
  if (FRT_COPY_MODE == 0) return __ldcs(p);
  if (FRT_COPY_MODE == 1) return *p;
  return __ldg(p);
}
__device__ __forceinline__ void cp_st(uint4* p, uint4 v) {
  if (FRT_COPY_MODE == 1) *p = v;
  else __stcs(p, v);
}
constexpr int kCopyUnroll = FRT_COPY_UNROLL;

__global__ void __launch_bounds__(256) copy_peak_kernel(const uint4* __restrict__ src,
                                                        uint4* __restrict__ dst, size_t n16) {
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + (kCopyUnroll - 1) * stride < n16; i += kCopyUnroll * stride) {
    uint4 v[kCopyUnroll];
#pragma unroll
    for (int k = 0; k < kCopyUnroll; ++k) v[k] = cp_ld(src + i + k * stride);
#pragma unroll
    for (int k = 0; k < kCopyUnroll; ++k) cp_st(dst + i + k * stride, v[k]);
  }
  for (; i < n16; i += stride) __stcs(dst + i, __ldcs(src + i));
}

}  // namespace
}  // namespace frt

extern "C" int frt_peak_fp8_mma(int ctas, int iters, int operands, void* stream) {
  frt::clear_error();
  FRT_REQUIRE(ctas >= 1 && ctas <= 4096 && iters >= 1, FRT_EINVAL,
              "ctas must be in [1, 4096] and iters >= 1");
  FRT_REQUIRE(operands == FRT_PEAK_OPERANDS_GAUSSIAN || operands == FRT_PEAK_OPERANDS_LOW_TOGGLE,
              FRT_EINVAL, "operands must be FRT_PEAK_OPERANDS_GAUSSIAN or _LOW_TOGGLE");
  constexpr int smem = frt::kMbA + frt::kMbB + 1024 + 64;
  auto kern = frt::mma_peak_kernel;
  if (frt::first_use(reinterpret_cast<const void*>(kern)) &&
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess)
    return frt::fail(FRT_ECUDA, "cudaFuncSetAttribute(mma_peak_kernel)");
  kern<<<ctas, frt::kMbThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      iters, operands, frt::device_status_ptr());
  return frt::check_launch("mma_peak_kernel");
}

extern "C" int frt_peak_copy(const void* src, void* dst, size_t bytes, void* stream) {
  frt::clear_error();
  FRT_REQUIRE(src && dst, FRT_EINVAL, "src and dst are required");
  FRT_REQUIRE(frt::aligned(src, 16) && frt::aligned(dst, 16) && bytes % 16 == 0, FRT_EALIGN,
              "src, dst and bytes must be 16-byte aligned");
  if (bytes == 0) return FRT_OK;
  const int grid = frt::num_sms() * FRT_COPY_BLOCKS_PER_SM;
  frt::copy_peak_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), bytes / 16);
  return frt::check_launch("copy_peak_kernel");
}
