// tail.cu -- the output side of the AdaRMS layer around the chain:
//   * frt_quantize_fp8_static: static e4m3 quantize of a bf16 activation
//     (impls/adarms_stack/fp8_chain.py `out_project`: the attention output
//     quantized with the site's static scale before the o_proj GEMM);
//   * frt_ada_rms_tail: the stack's final AdaRMS tail (`_make_run`, the
//     "ad:tail" range): h = res + gate * delta in fp32 (not rounded to bf16),
//     RMS norm, (1 + scale) * . + shift with the last norm's fp32 rows, bf16.
// Both are one HBM pass.  The quantize divides (IEEE, round to nearest):
// its inputs are bf16 values, whose ratios to the scale land exactly on e4m3
// rounding midpoints often enough that a reciprocal multiply would move
// about one code in a hundred.  Programmatic dependent launch as every
// kernel of the chain.

#include "frt_common.cuh"

namespace frt {
namespace {

struct QuantArgs {
  int rows, D, C;
  const uint16_t* x;
  long ldx;
  const float* scale;
  uint8_t* x8;
  float* amax;
};

__global__ void __launch_bounds__(256) quant_fp8_kernel(QuantArgs a) {
  pdl_trigger();
  pdl_wait();
  const float sc = __ldg(a.scale);
  const long units = long(a.rows) * a.C;
  float mx = 0.0f;
  for (long u = long(blockIdx.x) * blockDim.x + threadIdx.x; u < units;
       u += long(gridDim.x) * blockDim.x) {
    const long r = u / a.C;
    const int c = int(u - r * a.C);
    float v[8], q[8];
    unpack8(__ldg(reinterpret_cast<const uint4*>(a.x + r * a.ldx + 8 * c)), v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mx = fmaxf(mx, fabsf(v[j]));
      q[j] = __fdiv_rn(v[j], sc);
    }
    *reinterpret_cast<uint2*>(a.x8 + r * a.D + 8 * c) = pack8_e4m3(q);
  }
  if (a.amax) {
    mx = warp_max(mx);
    if ((threadIdx.x & 31) == 0) atomic_max_nonneg(a.amax, mx);
  }
}

struct TailArgs {
  int rows, D, C, G;
  float eps;
  const uint16_t* res;
  const uint16_t* delta;
  const uint16_t* gate;
  long gate_stride;
  const float* fin;
  long fin_stride;
  uint16_t* out;
};

// G threads per row (G == 32: 8 rows per block of 256; else one row per
// block); each thread holds VPT chunks of 8 columns, every input of the row
// requested before the row reduction.
template <int VPT>
__global__ void __launch_bounds__(256) ada_rms_tail_kernel(TailArgs a) {
  __shared__ float red[8];
  pdl_trigger();
  pdl_wait();
  const int G = a.G;
  const int t = threadIdx.x % G;
  const long r = long(blockIdx.x) * (blockDim.x / G) + threadIdx.x / G;
  if (G == 32 && r >= a.rows) return;  // warp-uniform
  const bool ok = r < a.rows;          // G > 32: the whole block
  const int D = a.D, C = a.C;
  float h[VPT][8];
  float ss = 0.0f;
  if (ok) {
    uint4 r4[VPT], d4[VPT], g4[VPT];
    const uint16_t* rr = a.res + r * D;
    const uint16_t* dd = a.delta + r * D;
    const uint16_t* gg = a.gate + r * a.gate_stride;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = t + i * G;
      if (c < C) {
        r4[i] = __ldg(reinterpret_cast<const uint4*>(rr + 8 * c));
        d4[i] = __ldg(reinterpret_cast<const uint4*>(dd + 8 * c));
        g4[i] = __ldg(reinterpret_cast<const uint4*>(gg + 8 * c));
      }
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = t + i * G;
      if (c < C) {
        float rv[8], dv[8], gv[8];
        unpack8(r4[i], rv);
        unpack8(d4[i], dv);
        unpack8(g4[i], gv);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          h[i][j] = __fadd_rn(rv[j], __fmul_rn(gv[j], dv[j]));
          ss = __fadd_rn(ss, __fmul_rn(h[i][j], h[i][j]));
        }
      }
    }
  }
  ss = warp_sum(ss);
  if (G > 32) {
    const int w = threadIdx.x >> 5, nw = G >> 5;
    if ((threadIdx.x & 31) == 0) red[w] = ss;
    __syncthreads();
    ss = 0.0f;
    for (int i = 0; i < nw; ++i) ss = __fadd_rn(ss, red[i]);
  }
  if (!ok) return;
  const float ms = __fdiv_rn(ss, float(D));
  const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = t + i * G;
    if (c < C) {
      const float4* sc = reinterpret_cast<const float4*>(a.fin + 8 * c);
      const float4* sh = reinterpret_cast<const float4*>(a.fin + a.fin_stride + 8 * c);
      const float4 s0 = __ldg(sc), s1 = __ldg(sc + 1), h0 = __ldg(sh), h1 = __ldg(sh + 1);
      const float scale[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      const float shift[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
      float y[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float v = __fmul_rn(__fmul_rn(h[i][j], inv), __fadd_rn(1.0f, scale[j]));
        y[j] = __fadd_rn(v, shift[j]);
      }
      *reinterpret_cast<uint4*>(a.out + r * D + 8 * c) = pack8_bf16(y);
    }
  }
}

}  // namespace
}  // namespace frt

extern "C" int frt_quantize_fp8_static(int rows, int D, const frt_bf16* x, long ldx,
                                       const float* act_scale, frt_e4m3* x8_out,
                                       float* amax_out, void* stream) {
  using frt::aligned;
  frt::clear_error();
  FRT_REQUIRE(rows >= 0 && D > 0 && D % 8 == 0, FRT_ESHAPE,
              "rows must be >= 0 and D a positive multiple of 8 (rows %d, D %d)", rows, D);
  FRT_REQUIRE(ldx >= D && ldx % 8 == 0, FRT_EALIGN, "ldx must be >= D and a multiple of 8");
  FRT_REQUIRE(x && act_scale && x8_out, FRT_EINVAL, "x, act_scale and x8_out are required");
  FRT_REQUIRE(aligned(x, 16) && aligned(x8_out, 8) && aligned(act_scale, 4) &&
                  (!amax_out || aligned(amax_out, 4)),
              FRT_EALIGN, "x must be 16-byte and x8_out 8-byte aligned");
  if (rows == 0) return FRT_OK;
  frt::QuantArgs a{rows, D, D / 8, x, ldx, act_scale, x8_out, amax_out};
  const long units = long(rows) * a.C;
  const long want = (units + 255) / 256;
  const long cap = long(frt::num_sms()) * 8;
  const dim3 grid(unsigned(want < cap ? want : cap));
  return frt::launch_pdl("quant_fp8_kernel", frt::quant_fp8_kernel, grid, dim3(256), 0,
                         static_cast<cudaStream_t>(stream), a);
}

extern "C" int frt_ada_rms_tail(int rows, int D, float eps, const frt_bf16* res,
                                const frt_bf16* delta, const frt_bf16* gate, long gate_row_stride,
                                const float* fin, long fin_row_stride, frt_bf16* out,
                                void* stream) {
  using frt::aligned;
  frt::clear_error();
  FRT_REQUIRE(rows >= 0 && D >= 8 && D <= 8192 && D % 8 == 0, FRT_ESHAPE,
              "D must be a multiple of 8 in [8, 8192], got %d", D);
  FRT_REQUIRE(res && delta && gate && fin && out, FRT_EINVAL,
              "res, delta, gate, fin and out are required");
  FRT_REQUIRE(gate_row_stride == 0 || (gate_row_stride >= D && gate_row_stride % 8 == 0),
              FRT_EALIGN, "gate_row_stride must be 0 or a multiple of 8 >= D");
  FRT_REQUIRE(fin_row_stride >= D && fin_row_stride % 8 == 0, FRT_EALIGN,
              "fin_row_stride must be a multiple of 8 >= D");
  FRT_REQUIRE(aligned(res, 16) && aligned(delta, 16) && aligned(gate, 16) && aligned(fin, 16) &&
                  aligned(out, 16),
              FRT_EALIGN, "res, delta, gate, fin and out must be 16-byte aligned");
  if (rows == 0) return FRT_OK;
  frt::TailArgs a{rows, D, D / 8, 0, eps, res, delta, gate, gate_row_stride, fin,
                  fin_row_stride, out};
  int vpt;
  if (a.C <= 128) {
    a.G = 32;
    vpt = (a.C + 31) / 32;
  } else {
    vpt = (a.C + 255) / 256;
    a.G = ((a.C + vpt - 1) / vpt + 31) / 32 * 32;
  }
  const int rpb = a.G == 32 ? 8 : 1;
  const dim3 grid(unsigned((rows + rpb - 1) / rpb)), block(unsigned(a.G * rpb));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (vpt) {
    case 1: return frt::launch_pdl("ada_rms_tail_kernel", frt::ada_rms_tail_kernel<1>, grid, block, 0, s, a);
    case 2: return frt::launch_pdl("ada_rms_tail_kernel", frt::ada_rms_tail_kernel<2>, grid, block, 0, s, a);
    case 3: return frt::launch_pdl("ada_rms_tail_kernel", frt::ada_rms_tail_kernel<3>, grid, block, 0, s, a);
    default: return frt::launch_pdl("ada_rms_tail_kernel", frt::ada_rms_tail_kernel<4>, grid, block, 0, s, a);
  }
}
