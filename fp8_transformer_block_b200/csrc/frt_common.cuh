// frt_common.cuh -- host error plumbing and device numeric helpers shared by
// the library's translation units.  Everything here is this library's own;
// nothing is shared with the CPU oracle.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/frt.h"

// ------------------------------------------------------------------ host --

namespace frt {

// Record a reason for the calling thread (read back by frt_last_error) and
// return `code`, so validation reads `return fail(FRT_ESHAPE, "...")`.
int fail(int code, const char* fmt, ...);
void clear_error();
// Map a CUDA error from a launch to FRT_ECUDA with the call site named.
int check_launch(const char* what);
// Device address of the library's device-side status word for the current
// device (bounded waits that run out record their code there).
int* device_status_ptr();
// Streaming multiprocessors of the current device (cached per device).
int num_sms();
// True the first time it is called for this kernel on the current device.
bool first_use(const void* kernel);

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

}  // namespace frt

#define FRT_REQUIRE(cond, code, ...) \
  do { if (!(cond)) return ::frt::fail((code), __VA_ARGS__); } while (0)

namespace frt {

// Launch with programmatic dependent launch allowed: the kernel may begin
// (prologue, loads of data no earlier kernel writes) while its predecessor in
// the stream finishes.  Every kernel launched this way executes pdl_wait()
// before it touches memory an earlier kernel may read or write.
template <typename... KArgs, typename... Args>
int launch_pdl(const char* what, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
               cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // every kernel of the chain asks for the same L1 / shared-memory split as
  // the GEMM, so an SM never has to drain to reconfigure between them
  if (first_use(reinterpret_cast<const void*>(kern)))
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FRT_ECUDA, "%s: %s", what, cudaGetErrorString(e));
  }
  return FRT_OK;
}

}  // namespace frt

// ---------------------------------------------------------------- device --

namespace frt {

__device__ __forceinline__ float bf2f(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

// fp32 -> bf16 bits, round to nearest even (the CUDA conversion intrinsic).
__device__ __forceinline__ uint16_t f2bf(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two fp32 -> two e4m3fn codes (lo in the low byte), round to nearest even,
// saturating to +-448: the hardware conversion, which equals clamp-then-round.
__device__ __forceinline__ uint16_t pack_e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// ---- paired fp32 arithmetic (sm_100 f32x2 instructions) --------------------
// A uint64_t holds two fp32 lanes (lo, hi).  add2 / sub2 / mul2 round each
// lane to nearest even exactly like the scalar __fadd_rn / __fsub_rn /
// __fmul_rn, so swapping a scalar pair for one paired instruction leaves
// every result bit unchanged while halving the instructions issued.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(uint32_t(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float(uint32_t(v >> 32)); }
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// a * b + c per lane with one rounding (fused multiply-add)
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
// Two bf16 in one 32-bit word (lo in the low half) -> an fp32 pair.
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
  return (uint64_t(w & 0xFFFF0000u) << 32) | uint64_t(w << 16);
}
// 8 bf16 in a uint4 -> 4 fp32 pairs.
__device__ __forceinline__ void unpack8_f2(const uint4& v, uint64_t (&f)[4]) {
  f[0] = bf16x2_to_f2(v.x);
  f[1] = bf16x2_to_f2(v.y);
  f[2] = bf16x2_to_f2(v.z);
  f[3] = bf16x2_to_f2(v.w);
}
// 4 fp32 pairs -> 8 bf16 (round to nearest even) in a uint4.
__device__ __forceinline__ uint4 pack8_bf16_f2(const uint64_t (&f)[4]) {
  return make_uint4(pack_bf16x2(f2_lo(f[0]), f2_hi(f[0])), pack_bf16x2(f2_lo(f[1]), f2_hi(f[1])),
                    pack_bf16x2(f2_lo(f[2]), f2_hi(f[2])), pack_bf16x2(f2_lo(f[3]), f2_hi(f[3])));
}
// 4 fp32 pairs -> 8 e4m3fn codes in a uint2.
__device__ __forceinline__ uint2 pack8_e4m3_f2(const uint64_t (&q)[4]) {
  const uint32_t lo = pack_e4m3x2(f2_lo(q[0]), f2_hi(q[0])) |
                      (uint32_t(pack_e4m3x2(f2_lo(q[1]), f2_hi(q[1]))) << 16);
  const uint32_t hi = pack_e4m3x2(f2_lo(q[2]), f2_hi(q[2])) |
                      (uint32_t(pack_e4m3x2(f2_lo(q[3]), f2_hi(q[3]))) << 16);
  return make_uint2(lo, hi);
}
// max(m, |lo|, |hi|)
__device__ __forceinline__ float absmax2(float m, uint64_t v) {
  return fmaxf(fmaxf(m, fabsf(f2_lo(v))), fabsf(f2_hi(v)));
}

// 8 bf16 packed in a uint4 -> 8 floats.
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                    pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
}

// Adjacent-pair rotation of 8 bf16 values x (4 pairs) with 4 (cos, sin)
// pairs r (the rope table's interleaved layout): (x0, x1) -> (x0*c - x1*s,
// x0*s + x1*c) in fp32, each product and sum rounded once, then bf16.  The
// fused GEMM epilogue and the standalone split kernel both use this, so
// their results agree bit for bit.
__device__ __forceinline__ uint4 rope_rotate8(const uint4& xv, const uint4& rv) {
  float x[8], r[8], o[8];
  unpack8(xv, x);
  unpack8(rv, r);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float x0 = x[2 * p], x1 = x[2 * p + 1], c = r[2 * p], s = r[2 * p + 1];
    o[2 * p] = __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, s));
    o[2 * p + 1] = __fadd_rn(__fmul_rn(x0, s), __fmul_rn(x1, c));
  }
  return pack8_bf16(o);
}

// 8 floats already divided by the scale -> 8 e4m3 codes in a uint2.
__device__ __forceinline__ uint2 pack8_e4m3(const float (&q)[8]) {
  uint32_t lo = pack_e4m3x2(q[0], q[1]) | (uint32_t(pack_e4m3x2(q[2], q[3])) << 16);
  uint32_t hi = pack_e4m3x2(q[4], q[5]) | (uint32_t(pack_e4m3x2(q[6], q[7])) << 16);
  return make_uint2(lo, hi);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// |y| max into a device float holding non-negative values: the bit patterns
// of non-negative floats order like unsigned integers.
__device__ __forceinline__ void atomic_max_nonneg(float* dst, float v) {
  atomicMax(reinterpret_cast<unsigned int*>(dst), __float_as_uint(v));
}

// Programmatic dependent launch: wait for the preceding kernel's completion
// (and the visibility of its writes); allow the next kernel to start early.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// c * gelu_tanh(g) [* u] on two lanes at once, with gelu_tanh(x) = 0.5 x
// (1 + tanh(y)), y = sqrt(2/pi) (x + 0.044715 x^3) (the tanh form of
// Hendrycks & Gimpel's GELU), every step an explicitly rounded fp32
// operation issued as a paired instruction.  half_c holds 0.5 c in both
// lanes (c: the output scale's reciprocal, or 1).
//   * -2 log2(e) y = g (A0 + A1 g^2), the constants folded (one fma, one
//     multiply); the hardware base-2 exponential of 1 - 2 log2(e) |y| gives
//     2E directly, E = exp(-2|y|) (ex2.approx.ftz: 0 once E underflows);
//   * r = 1 / (1 + E), an argument d in [1, 2]: two Newton steps r <- r + r
//     (1 - d r) from the minimax quadratic seed (70 - 48 d + 32 d^2 / 3) / 33
//     (relative error at most 1/99, squared by each step: within one ulp
//     after two, and exactly 1 at d = 1);
//   * tanh|y| = 1 - 2E r, its sign that of y (= that of g), then 1 + tanh(y)
//     formed as the fp32 formula 0.5 g (1 + tanh(y)) forms it -- cancelling
//     where y << 0 just as that evaluation does (an accurate 2E / (1 + E)
//     there moves e4m3 codes away from it);
//   * gelu_one_plus_tanh2 returns 1 + tanh(y); gelu_tanh_scaled2 the result
//     (0.5 c g) (1 + tanh y) [u]: exactly c g once tanh saturates (E = 0), a
//     zero of g's sign at g = +-0.
__device__ __forceinline__ uint64_t gelu_one_plus_tanh2(uint64_t g) {
  constexpr float kA0 = -2.0f * 0.7978845608028654f * 1.4426950408889634f;
  constexpr float kA1 = -2.0f * 0.7978845608028654f * 0.044715f * 1.4426950408889634f;
  const uint64_t one = f2_pack(1.0f, 1.0f);
  constexpr uint64_t kSign = 0x8000000080000000ull;
  const uint64_t q = fma2(mul2(g, g), f2_pack(kA1, kA1), f2_pack(kA0, kA0));
  const uint64_t x = add2(mul2(q, g) | kSign, one);  // 1 - 2 log2(e) |y|
  float e_lo, e_hi;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e_lo) : "f"(f2_lo(x)));
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e_hi) : "f"(f2_hi(x)));
  const uint64_t e2 = f2_pack(e_lo, e_hi);  // 2E
  const uint64_t d = fma2(e2, f2_pack(0.5f, 0.5f), one);
  uint64_t r = fma2(fma2(d, f2_pack(32.0f / 99.0f, 32.0f / 99.0f),
                         f2_pack(-48.0f / 33.0f, -48.0f / 33.0f)),
                    d, f2_pack(70.0f / 33.0f, 70.0f / 33.0f));
#pragma unroll
  for (int i = 0; i < 2; ++i) r = fma2(r, fma2(d ^ kSign, r, one), r);
  const uint64_t t = sub2(one, mul2(e2, r)) | (g & kSign);  // tanh(y): y has g's sign
  return add2(one, t);
}
template <bool GATED>
__device__ __forceinline__ uint64_t gelu_tanh_scaled2(uint64_t g, uint64_t u, uint64_t half_c) {
  const uint64_t v = mul2(mul2(g, half_c), gelu_one_plus_tanh2(g));
  if constexpr (GATED) return mul2(v, u);
  return v;
}

}  // namespace frt
