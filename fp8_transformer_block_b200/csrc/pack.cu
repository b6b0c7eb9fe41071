// pack.cu -- a0: joint per-tensor FP8 pack of sibling weights (bind time).
//
// flashrt-structures 0.2.0, impls/qkv_pack/fp8_static.py `_pack_weights`:
// concatenate the siblings along N, one scale for the whole stack,
// scale = max(amax / 448, 1e-8), w8 = e4m3(clamp(w / scale)), zero biases for
// siblings without one.  impls/adarms_stack/fp8_chain.py `_quantize` packs
// q and k with their rows interleaved per head (`_interleave_rows`) so the
// adjacent-pair RoPE carries the host's rotate-half rotation; the row map is
// the inverse of the chain's `kperm`.  The gate/up block layout is this
// library's own row order for the fused GEGLU epilogue.
//
// Three launches: amax (max-reduce into the output scale word), finalize
// (one thread turns amax into the scale), quantize (16 weights per thread,
// 32-byte loads, 16-byte stores, each written to its destination row).
#include "frt_common.cuh"

namespace frt {
namespace {

constexpr int kMaxSiblings = 4;

struct PackArgs {
  int n_sib, K, layout, hd;
  const uint16_t* w[kMaxSiblings];
  const uint16_t* bias[kMaxSiblings];
  int n[kMaxSiblings];
  long row0[kMaxSiblings];  // first packed row of sibling i (concat order)
  long total_rows;
  uint8_t* w8;
  float* scale;
  uint16_t* bias_out;
};

__global__ void pack_amax_kernel(PackArgs a) {
  float mx = 0.0f;
  for (int s = 0; s < a.n_sib; ++s) {
    const long n8 = long(a.n[s]) * a.K / 8;
    const uint4* src = reinterpret_cast<const uint4*>(a.w[s]);
    for (long i = blockIdx.x * long(blockDim.x) + threadIdx.x; i < n8;
         i += long(gridDim.x) * blockDim.x) {
      float f[8];
      unpack8(__ldg(src + i), f);
#pragma unroll
      for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(f[j]));
    }
  }
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0) atomic_max_nonneg(a.scale, mx);
}

// Launched (without programmatic overlap) after the quantize kernel so the
// packed weights are complete and visible before any later kernel starts:
// the GEMM may read weights before its own dependency wait.
__global__ void pack_fence_kernel() {}

__global__ void pack_finalize_kernel(float* scale) {
  const float s = __fdiv_rn(*scale, 448.0f);
  *scale = s < 1e-8f ? 1e-8f : s;
}

__device__ __forceinline__ long dest_row(const PackArgs& a, int sib, long i) {
  if (a.layout == FRT_PACK_QK_INTERLEAVE && sib < 2) {
    const long head = i / a.hd, d = i % a.hd, half = a.hd / 2;
    const long dst = d < half ? 2 * d : 2 * (d - half) + 1;
    return a.row0[sib] + head * a.hd + dst;
  }
  if (a.layout == FRT_PACK_GATE_UP_BLOCKS)
    return (i / 128) * 256 + (sib == 1 ? 128 : 0) + (i % 128);
  return a.row0[sib] + i;
}

__global__ void pack_quant_kernel(PackArgs a) {
  const float s = *a.scale;
  const int kc = a.K / 16;  // 16-element chunks per row
  const long total = a.total_rows * kc;
  for (long g = blockIdx.x * long(blockDim.x) + threadIdx.x; g < total;
       g += long(gridDim.x) * blockDim.x) {
    const long prow = g / kc;
    const int c = int(g % kc);
    int sib = 0;
    while (sib + 1 < a.n_sib && prow >= a.row0[sib + 1]) ++sib;
    const long i = prow - a.row0[sib];
    const uint4* src = reinterpret_cast<const uint4*>(a.w[sib] + i * a.K + 16 * c);
    float f0[8], f1[8], q0[8], q1[8];
    unpack8(__ldg(src), f0);
    unpack8(__ldg(src + 1), f1);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      q0[j] = __fdiv_rn(f0[j], s);
      q1[j] = __fdiv_rn(f1[j], s);
    }
    const uint2 lo = pack8_e4m3(q0), hi = pack8_e4m3(q1);
    const long dst = dest_row(a, sib, i);
    *reinterpret_cast<uint4*>(a.w8 + dst * a.K + 16 * c) = make_uint4(lo.x, lo.y, hi.x, hi.y);
    if (c == 0 && a.bias_out) a.bias_out[dst] = a.bias[sib] ? a.bias[sib][i] : uint16_t(0);
  }
}

}  // namespace
}  // namespace frt

extern "C" int frt_pack_weights_fp8(int n_siblings, const frt_bf16* const* w,
                                    const int* n_rows, int K, const frt_bf16* const* bias,
                                    int layout, int hd, frt_e4m3* w8_out, float* w_scale_out,
                                    frt_bf16* bias_out, void* stream) {
  using frt::aligned;
  frt::clear_error();
  FRT_REQUIRE(n_siblings >= 1 && n_siblings <= frt::kMaxSiblings, FRT_EINVAL,
              "n_siblings must be in [1, %d], got %d", frt::kMaxSiblings, n_siblings);
  FRT_REQUIRE(w && n_rows && w8_out && w_scale_out, FRT_EINVAL,
              "w, n_rows, w8_out and w_scale_out are required");
  FRT_REQUIRE(K > 0 && K % 16 == 0, FRT_ESHAPE, "K must be a positive multiple of 16, got %d", K);
  FRT_REQUIRE(layout >= FRT_PACK_CONCAT && layout <= FRT_PACK_GATE_UP_BLOCKS, FRT_EINVAL,
              "unknown layout %d", layout);
  FRT_REQUIRE(aligned(w8_out, 16) && aligned(w_scale_out, 4) && (!bias_out || aligned(bias_out, 2)),
              FRT_EALIGN, "w8_out must be 16-byte aligned");
  frt::PackArgs a{};
  a.n_sib = n_siblings; a.K = K; a.layout = layout; a.hd = hd;
  long rows = 0;
  for (int i = 0; i < n_siblings; ++i) {
    FRT_REQUIRE(w[i] && n_rows[i] > 0, FRT_EINVAL, "sibling %d is empty or NULL", i);
    FRT_REQUIRE(aligned(w[i], 16), FRT_EALIGN, "sibling %d must be 16-byte aligned", i);
    a.w[i] = w[i];
    a.bias[i] = bias ? bias[i] : nullptr;
    a.n[i] = n_rows[i];
    a.row0[i] = rows;
    rows += n_rows[i];
  }
  if (layout == FRT_PACK_QK_INTERLEAVE) {
    FRT_REQUIRE(n_siblings >= 2 && hd >= 2 && hd % 2 == 0, FRT_ESHAPE,
                "q/k interleave needs q and k siblings and an even head size, hd=%d", hd);
    FRT_REQUIRE(n_rows[0] % hd == 0 && n_rows[1] % hd == 0, FRT_ESHAPE,
                "q and k rows must be whole heads of %d", hd);
  }
  if (layout == FRT_PACK_GATE_UP_BLOCKS)
    FRT_REQUIRE(n_siblings == 2 && n_rows[0] == n_rows[1] && n_rows[0] % 128 == 0,
                FRT_ESHAPE, "gate/up blocks need two equal siblings with rows %% 128 == 0");
  a.total_rows = rows;
  a.w8 = w8_out; a.scale = w_scale_out; a.bias_out = bias_out;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(w_scale_out, 0, sizeof(float), s) != cudaSuccess)
    return frt::fail(FRT_ECUDA, "clearing w_scale_out");
  const int sms = frt::num_sms();
  frt::pack_amax_kernel<<<sms * 4, 256, 0, s>>>(a);
  frt::pack_finalize_kernel<<<1, 1, 0, s>>>(w_scale_out);
  frt::pack_quant_kernel<<<sms * 8, 256, 0, s>>>(a);
  frt::pack_fence_kernel<<<1, 32, 0, s>>>();
  return frt::check_launch("frt_pack_weights_fp8");
}
