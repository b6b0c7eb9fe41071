// geglu.cu -- a5 (standalone form): merged GEGLU + static FP8 requant, and
// the plain GELU + requant of the DiT FFN (fp8_ptok_table.py).
//
// flashrt-structures 0.2.0, impls/adarms_stack/fp8_chain.py `down_project`
// (the merged gate/up output gu [S, 2H] becomes hid8 [S, H] in one kernel,
// quantized with the down projection's static input scale) and the bind
// check that the FFN activation is the tanh-approximate GELU.
// gelu_tanh(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), the tanh
// form of Hendrycks & Gimpel's GELU (frt::gelu_one_plus_tanh2, shared with
// the fused GEMM epilogue, whose arithmetic these kernels repeat step for
// step so both forms give the same codes).
#include "frt_common.cuh"

namespace frt {

namespace {

__global__ void geglu_kernel(int M, int H, const uint16_t* gu, long ld, const float* out_scale,
                             uint8_t* hid8, float* amax) {
  const int h8 = H / 8;
  const long total = long(M) * h8;
  pdl_trigger();
  pdl_wait();
  // quantize: h * (1 / scale), the reciprocal folded into the GELU's 0.5
  const float inv_os = __frcp_rn(__ldg(out_scale));
  const uint64_t half_c = f2_pack(0.5f * inv_os, 0.5f * inv_os), half = f2_pack(0.5f, 0.5f);
  float mx = 0.0f;
  for (long g = blockIdx.x * long(blockDim.x) + threadIdx.x; g < total;
       g += long(gridDim.x) * blockDim.x) {
    const long m = g / h8;
    const int c = int(g % h8);
    float gv[8], uv[8], q[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(gu + m * ld + 8 * c)), gv);
    unpack8(__ldg(reinterpret_cast<const uint4*>(gu + m * ld + H + 8 * c)), uv);
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const uint64_t gp = f2_pack(gv[j], gv[j + 1]), up = f2_pack(uv[j], uv[j + 1]);
      const uint64_t opt = gelu_one_plus_tanh2(gp);
      const uint64_t h = mul2(mul2(mul2(gp, half_c), opt), up);
      if (amax) mx = absmax2(mx, mul2(mul2(mul2(gp, half), opt), up));
      q[j] = f2_lo(h);
      q[j + 1] = f2_hi(h);
    }
    *reinterpret_cast<uint2*>(hid8 + m * H + 8 * c) = pack8_e4m3(q);
  }
  if (amax) {
    mx = warp_max(mx);
    if ((threadIdx.x & 31) == 0) atomic_max_nonneg(amax, mx);
  }
}

// GELU + static requant of a bf16 [M, H] tensor (the DiT FFN's
// fp8_gelu_mlp middle step, unfused form; the GEMM's GELU epilogue gives the
// same codes).
__global__ void gelu_kernel(int M, int H, const uint16_t* u, long ld, const float* out_scale,
                            uint8_t* hid8, float* amax) {
  const int h8 = H / 8;
  const long total = long(M) * h8;
  pdl_trigger();
  pdl_wait();
  const float inv_os = __frcp_rn(__ldg(out_scale));
  const uint64_t half_c = f2_pack(0.5f * inv_os, 0.5f * inv_os), half = f2_pack(0.5f, 0.5f);
  float mx = 0.0f;
  for (long g = blockIdx.x * long(blockDim.x) + threadIdx.x; g < total;
       g += long(gridDim.x) * blockDim.x) {
    const long m = g / h8;
    const int c = int(g % h8);
    float uv[8], q[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(u + m * ld + 8 * c)), uv);
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const uint64_t x = f2_pack(uv[j], uv[j + 1]);
      const uint64_t opt = gelu_one_plus_tanh2(x);
      const uint64_t h = mul2(mul2(x, half_c), opt);
      if (amax) mx = absmax2(mx, mul2(mul2(x, half), opt));
      q[j] = f2_lo(h);
      q[j + 1] = f2_hi(h);
    }
    *reinterpret_cast<uint2*>(hid8 + m * H + 8 * c) = pack8_e4m3(q);
  }
  if (amax) {
    mx = warp_max(mx);
    if ((threadIdx.x & 31) == 0) atomic_max_nonneg(amax, mx);
  }
}

// The device GELU on pairs of elements (an odd tail paired with 0).
__global__ void gelu_selftest_kernel(const float* x, float* y, long n) {
  const long pairs = (n + 1) / 2;
  for (long i = blockIdx.x * long(blockDim.x) + threadIdx.x; i < pairs;
       i += long(gridDim.x) * blockDim.x) {
    const bool two = 2 * i + 1 < n;
    const uint64_t h = gelu_tanh_scaled2<false>(f2_pack(x[2 * i], two ? x[2 * i + 1] : 0.0f), 0,
                                                f2_pack(0.5f, 0.5f));
    y[2 * i] = f2_lo(h);
    if (two) y[2 * i + 1] = f2_hi(h);
  }
}

}  // namespace
}  // namespace frt

extern "C" int frt_selftest_gelu(const float* x, float* y, long n, void* stream) {
  frt::clear_error();
  FRT_REQUIRE(n >= 0, FRT_ESHAPE, "n must be >= 0");
  FRT_REQUIRE(n == 0 || (x && y), FRT_EINVAL, "x and y are required");
  FRT_REQUIRE(frt::aligned(x, 4) && frt::aligned(y, 4), FRT_EALIGN, "x and y must be 4-byte aligned");
  if (n == 0) return FRT_OK;
  const long need = ((n + 1) / 2 + 255) / 256;
  const int grid = int(need < frt::num_sms() * 8L ? need : frt::num_sms() * 8L);
  frt::gelu_selftest_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return frt::check_launch("frt_selftest_gelu");
}

extern "C" int frt_geglu_quant_fp8(int M, int H, const frt_bf16* gu, long ld_gu,
                                   const float* out_scale, frt_e4m3* hid8, float* amax_out,
                                   void* stream) {
  using frt::aligned;
  frt::clear_error();
  FRT_REQUIRE(M >= 0 && H > 0 && H % 8 == 0, FRT_ESHAPE, "H must be a positive multiple of 8");
  FRT_REQUIRE(ld_gu >= 2L * H && ld_gu % 8 == 0, FRT_ESHAPE, "ld_gu must be >= 2H and a multiple of 8");
  FRT_REQUIRE(gu && out_scale && hid8, FRT_EINVAL, "gu, out_scale and hid8 are required");
  FRT_REQUIRE(aligned(gu, 16) && aligned(hid8, 8), FRT_EALIGN, "gu 16-byte, hid8 8-byte aligned");
  if (M == 0) return FRT_OK;
  const long total = long(M) * (H / 8);
  const long need = (total + 255) / 256;
  const int grid = int(need < frt::num_sms() * 16L ? need : frt::num_sms() * 16L);
  return frt::launch_pdl("geglu_kernel", frt::geglu_kernel, dim3(grid), dim3(256), 0,
                         static_cast<cudaStream_t>(stream), M, H, gu, ld_gu, out_scale, hid8,
                         amax_out);
}

extern "C" int frt_gelu_quant_fp8(int M, int H, const frt_bf16* u, long ld_u,
                                  const float* out_scale, frt_e4m3* hid8, float* amax_out,
                                  void* stream) {
  using frt::aligned;
  frt::clear_error();
  FRT_REQUIRE(M >= 0 && H > 0 && H % 8 == 0, FRT_ESHAPE, "H must be a positive multiple of 8");
  FRT_REQUIRE(ld_u >= H && ld_u % 8 == 0, FRT_ESHAPE, "ld_u must be >= H and a multiple of 8");
  FRT_REQUIRE(u && out_scale && hid8, FRT_EINVAL, "u, out_scale and hid8 are required");
  FRT_REQUIRE(aligned(u, 16) && aligned(hid8, 8), FRT_EALIGN, "u 16-byte, hid8 8-byte aligned");
  if (M == 0) return FRT_OK;
  const long total = long(M) * (H / 8);
  const long need = (total + 255) / 256;
  const int grid = int(need < frt::num_sms() * 16L ? need : frt::num_sms() * 16L);
  return frt::launch_pdl("gelu_kernel", frt::gelu_kernel, dim3(grid), dim3(256), 0,
                         static_cast<cudaStream_t>(stream), M, H, u, ld_u, out_scale, hid8,
                         amax_out);
}
