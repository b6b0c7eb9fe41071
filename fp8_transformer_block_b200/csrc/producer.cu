// producer.cu -- a1 / a1': the single-pass producer of the chain's FP8 wire.
//
// AdaRMS form (flashrt-structures 0.2.0, impls/adarms_stack/fp8_chain.py,
// `norm_project`: gated residual add + AdaRMS + static quantize, and the fp32
// tail of `_make_run` that fixes the formula and the (scale, shift, gate)
// chunk order) and the per-token-table LayerNorm form
// (impls/modnorm_qkv_chain/fp8_ptok_table.py, module docstring and
// `PerTokenModChainBlock.forward`: table add + chunk selection + no-affine
// LayerNorm + modulation + static quantize, "the six-chunk materialization
// never exists").
//
// Layout: a group of G threads (G a multiple of 32) owns one row; each thread
// holds VPT chunks of 8 bf16 (16-byte loads) in registers, so every input
// byte is read once and every output byte written once (HBM-bound: 7*D bytes
// per row for the table form, 9*D with the gate output for AdaRMS).  All of a
// row's streamed inputs are loaded before the row reduction so they are in
// flight together.  Few rows (the latency regime) spread a row over more
// threads (VPT = 1); many rows use VPT = 4.  G == 32 packs 4 rows per block;
// larger G uses one row per block and a shared-memory cross-warp reduction.
// Arithmetic is fp32 with explicitly rounded operations (no contraction into
// FMA), IEEE division and square root for the row statistics; the quantizer
// multiplies by the correctly rounded fp32 reciprocal of the static scale
// (y * (1/s) and y / s differ by at most an ulp or two, which changes a code
// only when y / s sits that close to a rounding midpoint).
// Launched with programmatic dependent launch; blocks past the row blocks
// (when the chain passes a prefix) copy the cache prefix in the same grid.

#include "frt_internal.cuh"
#include "frt_sm100.cuh"

namespace frt {
namespace {

struct ProducerArgs {
  int rows, D, C, G, row_blocks;
  float eps;
  uint16_t* res;
  const uint16_t* delta;
  const uint16_t* gate;
  long gate_stride;
  const uint16_t* weight;
  const uint16_t* style;
  long style_stride;
  const uint16_t* x;
  const uint16_t* temb;
  int chunks;
  const float* table;
  int shift_idx, scale_idx;
  const float* act_scale;
  uint8_t* x8;
  uint16_t* gate_out;
  float* amax;
  int* status;
  PrefixArgs pre;  // pre.units == 0: no prefix blocks
};

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// Sum over the G threads of a row.  With G > 32 the block holds one row.
__device__ __forceinline__ float row_sum(float v, int G, float* red) {
  v = warp_sum(v);
  if (G == 32) return v;
  const int w = threadIdx.x >> 5, nw = G >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float s = 0.0f;
  for (int i = 0; i < nw; ++i) s = __fadd_rn(s, red[i]);
  return s;
}

// Blocks past the row blocks copy the prefix (grid-stride over its units).
__device__ __forceinline__ bool prefix_block(const ProducerArgs& a) {
  if (int(blockIdx.x) < a.row_blocks) return false;
  const long nb = long(gridDim.x) - a.row_blocks;
  prefix_units_strided(a.pre, (long(blockIdx.x) - a.row_blocks) * blockDim.x + threadIdx.x,
                       nb * blockDim.x);
  return true;
}

template <int VPT>
__global__ void __launch_bounds__(512) adarms_kernel(ProducerArgs a) {
  __shared__ float red[16];
  pdl_trigger();
  pdl_wait();
  if (prefix_block(a)) return;
  const int G = a.G;
  const int rpb = blockDim.x / G;
  const int t = threadIdx.x % G;
  const long r = long(blockIdx.x) * rpb + threadIdx.x / G;
  if (G == 32 && r >= a.rows) return;          // warp-uniform, no block sync
  const bool ok = r < a.rows;                  // G > 32: whole block uniform
  const int D = a.D, C = a.C;

  float hr[VPT][8];
  float ss = 0.0f;
  // every input of the row is requested up front (one memory round trip)
  uint4 sc4[VPT], sh4[VPT], w4[VPT], go4[VPT];
  const uint16_t* st = a.style + r * a.style_stride;
  if (ok) {
    uint16_t* rr = a.res + r * D;
    const uint16_t* dd = a.delta + r * D;
    const uint16_t* gg = a.gate + r * a.gate_stride;
    uint4 rv4[VPT], dv4[VPT], gv4[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = t + i * G;
      if (c < C) {
        rv4[i] = *reinterpret_cast<const uint4*>(rr + 8 * c);
        dv4[i] = ldg16(dd + 8 * c);
        gv4[i] = ldg16(gg + 8 * c);
        sc4[i] = ldg16(st + 8 * c);
        sh4[i] = ldg16(st + D + 8 * c);
        if (a.weight) w4[i] = ldg16(a.weight + 8 * c);
        if (a.gate_out) go4[i] = ldg16(st + 2 * D + 8 * c);
      }
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = t + i * G;
      if (c < C) {
        float rv[8], dv[8], gv[8], h[8];
        unpack8(rv4[i], rv);
        unpack8(dv4[i], dv);
        unpack8(gv4[i], gv);
#pragma unroll
        for (int j = 0; j < 8; ++j) h[j] = __fadd_rn(rv[j], __fmul_rn(gv[j], dv[j]));
        const uint4 hb = pack8_bf16(h);
        *reinterpret_cast<uint4*>(rr + 8 * c) = hb;
        unpack8(hb, hr[i]);
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = __fadd_rn(ss, __fmul_rn(hr[i][j], hr[i][j]));
      }
    }
  }
  ss = row_sum(ss, G, red);
  if (!ok) return;
  const float ms = __fdiv_rn(ss, float(D));
  const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
  const float inv_as = __frcp_rn(__ldg(a.act_scale));  // quantize: y * (1 / scale)
  float mx = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = t + i * G;
    if (c < C) {
      float wv[8], sc[8], sh[8];
      if (a.weight) unpack8(w4[i], wv);
      else {
#pragma unroll
        for (int j = 0; j < 8; ++j) wv[j] = 1.0f;
      }
      unpack8(sc4[i], sc);
      unpack8(sh4[i], sh);
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = __fmul_rn(hr[i][j], inv);
        v = __fmul_rn(v, wv[j]);
        v = __fmul_rn(v, __fadd_rn(1.0f, sc[j]));
        const float y = __fadd_rn(v, sh[j]);
        mx = fmaxf(mx, fabsf(y));
        q[j] = __fmul_rn(y, inv_as);
      }
      *reinterpret_cast<uint2*>(a.x8 + r * D + 8 * c) = pack8_e4m3(q);
      if (a.gate_out)
        *reinterpret_cast<uint4*>(a.gate_out + r * D + 8 * c) = go4[i];
    }
  }
  if (a.amax) {
    mx = warp_max(mx);
    if ((threadIdx.x & 31) == 0) atomic_max_nonneg(a.amax, mx);
  }
}

template <int VPT>
__global__ void __launch_bounds__(512) ln_table_kernel(ProducerArgs a) {
  __shared__ float red[16];
  pdl_trigger();
  pdl_wait();
  if (prefix_block(a)) return;
  const int G = a.G;
  const int rpb = blockDim.x / G;
  const int t = threadIdx.x % G;
  const long r = long(blockIdx.x) * rpb + threadIdx.x / G;
  if (G == 32 && r >= a.rows) return;
  const bool ok = r < a.rows;
  const int D = a.D, C = a.C;

  float xv[VPT][8];
  uint4 esh4[VPT], esc4[VPT];
  float sum = 0.0f;
  if (ok) {
    const uint16_t* xr = a.x + r * D;
    const uint16_t* tr = a.temb + r * long(a.chunks) * D;
    const uint16_t* tsh = tr + long(a.shift_idx) * D;
    const uint16_t* tsc = tr + long(a.scale_idx) * D;
    uint4 xv4[VPT];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = t + i * G;
      if (c < C) {
        xv4[i] = ldg16(xr + 8 * c);
        esh4[i] = ldg16(tsh + 8 * c);
        esc4[i] = ldg16(tsc + 8 * c);
      }
    }
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = t + i * G;
      if (c < C) {
        unpack8(xv4[i], xv[i]);
#pragma unroll
        for (int j = 0; j < 8; ++j) sum = __fadd_rn(sum, xv[i][j]);
      }
    }
  }
  sum = row_sum(sum, G, red);
  const float mu = __fdiv_rn(sum, float(D));
  float sq = 0.0f;
  if (ok) {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int c = t + i * G;
      if (c < C) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float d = __fsub_rn(xv[i][j], mu);
          sq = __fadd_rn(sq, __fmul_rn(d, d));
        }
      }
    }
  }
  sq = row_sum(sq, G, red);
  if (!ok) return;
  const float var = __fdiv_rn(sq, float(D));
  const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, a.eps)));
  const float inv_as = __frcp_rn(__ldg(a.act_scale));  // quantize: y * (1 / scale)
  const float* bsh = a.table + long(a.shift_idx) * D;
  const float* bsc = a.table + long(a.scale_idx) * D;
  float mx = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int c = t + i * G;
    if (c < C) {
      float esh[8], esc[8];
      unpack8(esh4[i], esh);
      unpack8(esc4[i], esc);
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(bsh + 8 * c));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(bsh + 8 * c + 4));
      const float4 c0 = __ldg(reinterpret_cast<const float4*>(bsc + 8 * c));
      const float4 c1 = __ldg(reinterpret_cast<const float4*>(bsc + 8 * c + 4));
      const float tsh8[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
      const float tsc8[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      float q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float shift = __fadd_rn(tsh8[j], esh[j]);
        const float scale = __fadd_rn(tsc8[j], esc[j]);
        float v = __fmul_rn(__fsub_rn(xv[i][j], mu), inv);
        v = __fmul_rn(v, __fadd_rn(1.0f, scale));
        const float y = __fadd_rn(v, shift);
        mx = fmaxf(mx, fabsf(y));
        q[j] = __fmul_rn(y, inv_as);
      }
      *reinterpret_cast<uint2*>(a.x8 + r * D + 8 * c) = pack8_e4m3(q);
    }
  }
  if (a.amax) {
    mx = warp_max(mx);
    if ((threadIdx.x & 31) == 0) atomic_max_nonneg(a.amax, mx);
  }
}

// ------------------------------------------------ staged (bandwidth) form --
//
// Many rows: persistent CTAs of T threads walk rows r = blockIdx.x,
// + row_blocks, ...; thread 0 keeps the next kStages rows' streamed inputs
// in flight as bulk copies into a shared-memory ring (one mbarrier per
// stage).  Thread t owns the column chunks c = t + i*T (i < CPT, 8 columns
// each): per row it moves its chunks from the ring into registers once, so
// the stage is handed back to the copy engine right after the first row
// reduction, and the per-column constants (table rows, norm weight) stay in
// registers for the CTA's lifetime.  Two block barriers per row, one per
// row statistic; the first also carries the consensus on a timed-out wait.
// Same operations as the register kernels, issued two lanes at a time
// (f32x2: identical rounding per lane, half the instructions); the row sums
// keep two running partials per thread, a different summation order that
// moves the statistics by a few ulps at most.
#ifndef FRT_PRODUCER_STAGES
#define FRT_PRODUCER_STAGES 3
#endif
#ifndef FRT_PRODUCER_MAX_THREADS
#define FRT_PRODUCER_MAX_THREADS 128
#endif
constexpr int kStages = FRT_PRODUCER_STAGES;        // rows in flight per CTA
constexpr int kMaxThreads = FRT_PRODUCER_MAX_THREADS;  // threads per row (CTA)
constexpr int kMaxCpt = 4;
constexpr uint64_t kRowWaitNs = 2000000000ull;   // 2 s per wait
constexpr uint64_t kRowDrainNs = 200000000ull;

// Sum over the block of one value per thread; `red` holds one slot per warp.
__device__ __forceinline__ float block_sum_into(float v, float* red, bool& ok) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  ok = __syncthreads_and(ok) != 0;
  float s = 0.0f;
  const int nw = int(blockDim.x >> 5);
  for (int i = 0; i < nw; ++i) s = __fadd_rn(s, red[i]);
  return s;
}

template <int MODE, int CPT>
__global__ void __launch_bounds__(256)
producer_staged_kernel(ProducerArgs a) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ float red1[8], red2[8];
  constexpr int NS = MODE == FRT_NORM_LAYERNORM_TABLE ? 3 : 2;  // streamed inputs per row
  pdl_trigger();
  pdl_wait();
  if (prefix_block(a)) return;
  const int D = a.D, C = a.C, tid = threadIdx.x, T = blockDim.x;
  const uint32_t row_bytes = 2u * uint32_t(D);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStages * NS * row_bytes);
  const long stride = a.row_blocks;

  auto issue = [&](long r, int st) {
    uint8_t* dst = ring + st * NS * row_bytes;
    mbar_arrive_expect_tx(&full[st], NS * row_bytes);
    if (MODE == FRT_NORM_LAYERNORM_TABLE) {
      const uint16_t* tr = a.temb + r * long(a.chunks) * D;
      bulk_load(dst, a.x + r * D, row_bytes, &full[st]);
      bulk_load(dst + row_bytes, tr + long(a.shift_idx) * D, row_bytes, &full[st]);
      bulk_load(dst + 2 * row_bytes, tr + long(a.scale_idx) * D, row_bytes, &full[st]);
    } else {
      bulk_load(dst, a.res + r * D, row_bytes, &full[st]);
      bulk_load(dst + row_bytes, a.delta + r * D, row_bytes, &full[st]);
    }
  };
  if (tid == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
    fence_barrier_init();
    for (int st = 0; st < kStages; ++st) {
      const long r = blockIdx.x + st * stride;
      if (r < a.rows) issue(r, st);
    }
  }
  __syncthreads();

  // per-column constants of this thread's chunks, as fp32 pairs
  bool has[CPT];
  uint64_t k0[CPT][4], k1[CPT][4];  // table: shift / scale rows; AdaRMS: weight
  const uint64_t one2 = f2_pack(1.0f, 1.0f);
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = tid + i * T;
    has[i] = c < C;
    if (MODE == FRT_NORM_LAYERNORM_TABLE) {
      if (has[i]) {
        const float* bsh = a.table + long(a.shift_idx) * D + 8 * c;
        const float* bsc = a.table + long(a.scale_idx) * D + 8 * c;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float4 t0 = __ldg(reinterpret_cast<const float4*>(bsh + 4 * h));
          const float4 t1 = __ldg(reinterpret_cast<const float4*>(bsc + 4 * h));
          k0[i][2 * h] = f2_pack(t0.x, t0.y);
          k0[i][2 * h + 1] = f2_pack(t0.z, t0.w);
          k1[i][2 * h] = f2_pack(t1.x, t1.y);
          k1[i][2 * h + 1] = f2_pack(t1.z, t1.w);
        }
      }
    } else {
      if (has[i] && a.weight) {
        unpack8_f2(__ldg(reinterpret_cast<const uint4*>(a.weight + 8 * c)), k0[i]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) k0[i][j] = one2;
      }
    }
  }

  const float inv_as = __frcp_rn(__ldg(a.act_scale));  // quantize: y * (1 / scale)
  const uint64_t inv_as2 = f2_pack(inv_as, inv_as);
  const uint64_t zero2 = f2_pack(0.0f, 0.0f);
  float mx = 0.0f;
  int k = 0;
  bool aborted = false;
  for (long r = blockIdx.x; r < a.rows; r += stride, ++k) {
    const int st = k % kStages;
    bool ok = mbar_wait_bounded(&full[st], uint32_t((k / kStages) & 1), kRowWaitNs, nullptr);
    const uint16_t* s0 = reinterpret_cast<const uint16_t*>(ring + st * NS * row_bytes);
    const uint16_t* s1 = s0 + D;
    uint64_t xv[CPT][4];
    if (MODE == FRT_NORM_ADARMS) {
      // s0: residual row, s1: delta row; h = res + gate * delta, written back
      const uint16_t* gg = a.gate + r * a.gate_stride;
      uint16_t* rr = a.res + r * D;
      uint64_t ss2 = zero2;
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = tid + i * T;
        if (has[i]) {
          uint64_t rv[4], dv[4], gv[4], h[4];
          unpack8_f2(*reinterpret_cast<const uint4*>(s0 + 8 * c), rv);
          unpack8_f2(*reinterpret_cast<const uint4*>(s1 + 8 * c), dv);
          unpack8_f2(__ldg(reinterpret_cast<const uint4*>(gg + 8 * c)), gv);
#pragma unroll
          for (int j = 0; j < 4; ++j) h[j] = add2(rv[j], mul2(gv[j], dv[j]));
          const uint4 hb = pack8_bf16_f2(h);
          if (ok) *reinterpret_cast<uint4*>(rr + 8 * c) = hb;
          unpack8_f2(hb, xv[i]);
#pragma unroll
          for (int j = 0; j < 4; ++j) ss2 = add2(ss2, mul2(xv[i][j], xv[i][j]));
        }
      }
      float ss = __fadd_rn(f2_lo(ss2), f2_hi(ss2));
      ss = block_sum_into(ss, red1, ok);   // every thread is done with the stage
      if (!ok) { aborted = true; break; }
      if (tid == 0) {
        const long rn = r + kStages * stride;
        if (rn < a.rows) issue(rn, st);
      }
      const float ms = __fdiv_rn(ss, float(D));
      const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, a.eps)));
      const uint64_t inv2 = f2_pack(inv, inv);
      const uint16_t* sty = a.style + r * a.style_stride;
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = tid + i * T;
        if (has[i]) {
          uint64_t sc[4], sh[4], q[4];
          unpack8_f2(__ldg(reinterpret_cast<const uint4*>(sty + 8 * c)), sc);
          unpack8_f2(__ldg(reinterpret_cast<const uint4*>(sty + D + 8 * c)), sh);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint64_t v = mul2(xv[i][j], inv2);
            v = mul2(v, k0[i][j]);
            v = mul2(v, add2(one2, sc[j]));
            const uint64_t y = add2(v, sh[j]);
            mx = absmax2(mx, y);
            q[j] = mul2(y, inv_as2);
          }
          *reinterpret_cast<uint2*>(a.x8 + r * D + 8 * c) = pack8_e4m3_f2(q);
          if (a.gate_out)
            *reinterpret_cast<uint4*>(a.gate_out + r * D + 8 * c) =
                __ldg(reinterpret_cast<const uint4*>(sty + 2 * D + 8 * c));
        }
      }
    } else {
      // s0: x row, s1: shift chunk of temb, s2: scale chunk of temb
      const uint16_t* s2 = s1 + D;
      uint4 esh4[CPT], esc4[CPT];
      uint64_t sum2 = zero2;
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = tid + i * T;
        if (has[i]) {
          unpack8_f2(*reinterpret_cast<const uint4*>(s0 + 8 * c), xv[i]);
          esh4[i] = *reinterpret_cast<const uint4*>(s1 + 8 * c);
          esc4[i] = *reinterpret_cast<const uint4*>(s2 + 8 * c);
#pragma unroll
          for (int j = 0; j < 4; ++j) sum2 = add2(sum2, xv[i][j]);
        }
      }
      float sum = __fadd_rn(f2_lo(sum2), f2_hi(sum2));
      sum = block_sum_into(sum, red1, ok);  // every thread is done with the stage
      if (!ok) { aborted = true; break; }
      if (tid == 0) {
        const long rn = r + kStages * stride;
        if (rn < a.rows) issue(rn, st);
      }
      const float mu = __fdiv_rn(sum, float(D));
      const uint64_t mu2 = f2_pack(mu, mu);
      uint64_t sq2 = zero2;
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        if (has[i]) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t d = sub2(xv[i][j], mu2);
            sq2 = add2(sq2, mul2(d, d));
          }
        }
      }
      float sq = __fadd_rn(f2_lo(sq2), f2_hi(sq2));
      bool ok2 = true;
      sq = block_sum_into(sq, red2, ok2);
      const float var = __fdiv_rn(sq, float(D));
      const float inv = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, a.eps)));
      const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = tid + i * T;
        if (has[i]) {
          uint64_t esh[4], esc[4], q[4];
          unpack8_f2(esh4[i], esh);
          unpack8_f2(esc4[i], esc);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t shift = add2(k0[i][j], esh[j]);
            const uint64_t scale = add2(k1[i][j], esc[j]);
            uint64_t v = mul2(sub2(xv[i][j], mu2), inv2);
            v = mul2(v, add2(one2, scale));
            const uint64_t y = add2(v, shift);
            mx = absmax2(mx, y);
            q[j] = mul2(y, inv_as2);
          }
          *reinterpret_cast<uint2*>(a.x8 + r * D + 8 * c) = pack8_e4m3_f2(q);
        }
      }
    }
  }
  if (aborted && tid == 0) {
    if (a.status) atomicExch(a.status, FRT_ETIMEOUT);
    // drain the copies still in flight (bounded)
    for (int j = 0; j < kStages; ++j) {
      const long r = blockIdx.x + long(k + j) * stride;
      if (r >= a.rows) break;
      mbar_wait_bounded(&full[(k + j) % kStages], uint32_t(((k + j) / kStages) & 1), kRowDrainNs,
                        nullptr);
    }
  }
  if (a.amax) {
    mx = warp_max(mx);
    if ((threadIdx.x & 31) == 0) atomic_max_nonneg(a.amax, mx);
  }
}
}  // namespace

int producer_call(int mode, int rows, int D, float eps, uint16_t* res, const uint16_t* delta,
                  const uint16_t* prev_gate, long gate_row_stride, const uint16_t* weight,
                  const uint16_t* style, long style_row_stride, const uint16_t* x,
                  const uint16_t* temb, int chunks, const float* table, int shift_idx,
                  int scale_idx, const float* act_scale, uint8_t* x8_out, uint16_t* gate_out,
                  float* amax_out, const PrefixArgs* pre, cudaStream_t s) {
  FRT_REQUIRE(mode == FRT_NORM_ADARMS || mode == FRT_NORM_LAYERNORM_TABLE, FRT_EINVAL,
              "mode %d is not FRT_NORM_ADARMS or FRT_NORM_LAYERNORM_TABLE", mode);
  FRT_REQUIRE(rows >= 0, FRT_ESHAPE, "rows must be >= 0, got %d", rows);
  FRT_REQUIRE(D >= 8 && D <= 16384 && D % 8 == 0, FRT_ESHAPE,
              "D must be a multiple of 8 in [8, 16384], got %d", D);
  FRT_REQUIRE(eps >= 0.0f, FRT_EINVAL, "eps must be >= 0");
  FRT_REQUIRE(act_scale && x8_out, FRT_EINVAL, "act_scale and x8_out are required");
  FRT_REQUIRE(aligned(x8_out, 8), FRT_EALIGN, "x8_out must be 8-byte aligned");
  FRT_REQUIRE(aligned(act_scale, 4), FRT_EALIGN, "act_scale must be 4-byte aligned");
  if (mode == FRT_NORM_ADARMS) {
    FRT_REQUIRE(res && delta && prev_gate && style, FRT_EINVAL,
                "AdaRMS needs res, delta, prev_gate and style");
    FRT_REQUIRE(aligned(res, 16) && aligned(delta, 16) && aligned(prev_gate, 16) &&
                    aligned(style, 16) && (!weight || aligned(weight, 16)) &&
                    (!gate_out || aligned(gate_out, 16)),
                FRT_EALIGN, "bf16 tensors must be 16-byte aligned");
    FRT_REQUIRE(gate_row_stride >= 0 && gate_row_stride % 8 == 0 && style_row_stride >= 0 &&
                    style_row_stride % 8 == 0,
                FRT_EALIGN, "row strides must be non-negative multiples of 8");
    FRT_REQUIRE(gate_row_stride == 0 || gate_row_stride >= D, FRT_ESHAPE,
                "gate_row_stride must be 0 or >= D");
    FRT_REQUIRE(style_row_stride == 0 || style_row_stride >= 3L * D, FRT_ESHAPE,
                "style_row_stride must be 0 or >= 3*D");
  } else {
    FRT_REQUIRE(x && temb && table, FRT_EINVAL, "LayerNorm-table needs x, temb and table");
    FRT_REQUIRE(chunks >= 1 && shift_idx >= 0 && shift_idx < chunks && scale_idx >= 0 &&
                    scale_idx < chunks,
                FRT_EINVAL, "chunk indices (%d, %d) outside [0, %d)", shift_idx, scale_idx, chunks);
    FRT_REQUIRE(aligned(x, 16) && aligned(temb, 16) && aligned(table, 16), FRT_EALIGN,
                "x, temb and table must be 16-byte aligned");
  }
  FRT_REQUIRE(!amax_out || aligned(amax_out, 4), FRT_EALIGN, "amax_out must be 4-byte aligned");
  const long pre_units = pre ? pre->units : 0;
  if (rows == 0 && pre_units == 0) return FRT_OK;

  ProducerArgs a{};
  a.rows = rows; a.D = D; a.C = D / 8; a.eps = eps;
  a.res = res; a.delta = delta; a.gate = prev_gate; a.gate_stride = gate_row_stride;
  a.weight = weight; a.style = style; a.style_stride = style_row_stride;
  a.x = x; a.temb = temb; a.chunks = chunks; a.table = table;
  a.shift_idx = shift_idx; a.scale_idx = scale_idx;
  a.act_scale = act_scale; a.x8 = x8_out; a.gate_out = gate_out; a.amax = amax_out;
  if (pre) a.pre = *pre;
  a.status = device_status_ptr();
  const int sms = num_sms();
  const int ns = mode == FRT_NORM_LAYERNORM_TABLE ? 3 : 2;
  const size_t staged_smem = size_t(kStages) * ns * 2 * D + 64;
  const int cpt = (a.C + kMaxThreads - 1) / kMaxThreads;
  constexpr size_t kStagedSmemMax = size_t(kStages) * 24 * 1024 + 64;
  // the staged form pays for rows of at least a few KB; narrow rows in
  // large numbers (D <= 1024, >= 16 rows per SM) run faster as register
  // groups with every load of the row up front (measured: 4096 x 512 rows,
  // 6.1 -> 5.2 us; 1024 x 512 keeps the staged form)
  const bool narrow_many = D <= 1024 && rows >= 16L * sms;
  if (rows > 2 * sms && !narrow_many && staged_smem <= kStagedSmemMax && cpt <= kMaxCpt) {
    // bandwidth regime: persistent CTAs with a bulk-copy row ring; each
    // thread owns cpt chunks of 8 columns
    using Kern = void (*)(ProducerArgs);
    static const Kern kerns[2][kMaxCpt] = {
        {producer_staged_kernel<FRT_NORM_ADARMS, 1>, producer_staged_kernel<FRT_NORM_ADARMS, 2>,
         producer_staged_kernel<FRT_NORM_ADARMS, 3>, producer_staged_kernel<FRT_NORM_ADARMS, 4>},
        {producer_staged_kernel<FRT_NORM_LAYERNORM_TABLE, 1>,
         producer_staged_kernel<FRT_NORM_LAYERNORM_TABLE, 2>,
         producer_staged_kernel<FRT_NORM_LAYERNORM_TABLE, 3>,
         producer_staged_kernel<FRT_NORM_LAYERNORM_TABLE, 4>}};
    const Kern kern = kerns[mode == FRT_NORM_ADARMS ? 0 : 1][cpt - 1];
    const int block = ((a.C + cpt - 1) / cpt + 31) / 32 * 32;
    if (first_use(reinterpret_cast<const void*>(kern)) &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kStagedSmemMax)) != cudaSuccess)
      return fail(FRT_ECUDA, "cudaFuncSetAttribute(producer smem)");
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, block, staged_smem) !=
            cudaSuccess ||
        per_sm < 1) {
      cudaGetLastError();
      per_sm = 1;
    }
    a.row_blocks = rows < sms * per_sm ? rows : sms * per_sm;
    int pre_blocks = 0;
    if (pre_units > 0) {
      const long need = (pre_units + block - 1) / block;
      pre_blocks = int(need < 2L * sms ? need : 2L * sms);
    }
    const dim3 grid(a.row_blocks + pre_blocks);
    return launch_pdl("producer_staged_kernel", kern, grid, dim3(block), staged_smem, s, a);
  }
  int vpt;
  if (rows <= 2 * sms) {  // latency regime: many threads per row
    vpt = a.C <= 512 ? 1 : a.C <= 1024 ? 2 : 4;
    a.G = ((a.C + vpt - 1) / vpt + 31) / 32 * 32;
  } else if (a.C <= 128) {
    a.G = 32;
    vpt = (a.C + 31) / 32;
  } else {
    vpt = 4;
    a.G = ((a.C + 127) / 128) * 32;
  }
  const int rpb = a.G == 32 ? 4 : 1;
  a.row_blocks = (rows + rpb - 1) / rpb;
  const int block = a.G * rpb;
  int pre_blocks = 0;
  if (pre_units > 0) {
    const long need = (pre_units + block - 1) / block;
    pre_blocks = int(need < 2L * sms ? need : 2L * sms);
  }
  const dim3 grid(a.row_blocks + pre_blocks);
  if (mode == FRT_NORM_ADARMS) {
    switch (vpt) {
      case 1: return launch_pdl("adarms_kernel", adarms_kernel<1>, grid, block, 0, s, a);
      case 2: return launch_pdl("adarms_kernel", adarms_kernel<2>, grid, block, 0, s, a);
      case 3: return launch_pdl("adarms_kernel", adarms_kernel<3>, grid, block, 0, s, a);
      default: return launch_pdl("adarms_kernel", adarms_kernel<4>, grid, block, 0, s, a);
    }
  }
  switch (vpt) {
    case 1: return launch_pdl("ln_table_kernel", ln_table_kernel<1>, grid, block, 0, s, a);
    case 2: return launch_pdl("ln_table_kernel", ln_table_kernel<2>, grid, block, 0, s, a);
    case 3: return launch_pdl("ln_table_kernel", ln_table_kernel<3>, grid, block, 0, s, a);
    default: return launch_pdl("ln_table_kernel", ln_table_kernel<4>, grid, block, 0, s, a);
  }
}

}  // namespace frt

extern "C" int frt_ada_norm_quant_fp8(
    int mode, int rows, int D, float eps, frt_bf16* res, const frt_bf16* delta,
    const frt_bf16* prev_gate, long gate_row_stride, const frt_bf16* weight,
    const frt_bf16* style, long style_row_stride, const frt_bf16* x,
    const frt_bf16* temb, int chunks, const float* table, int shift_idx,
    int scale_idx, const float* act_scale, frt_e4m3* x8_out, frt_bf16* gate_out,
    float* amax_out, void* stream) {
  frt::clear_error();
  return frt::producer_call(mode, rows, D, eps, res, delta, prev_gate, gate_row_stride, weight,
                            style, style_row_stride, x, temb, chunks, table, shift_idx,
                            scale_idx, act_scale, x8_out, gate_out, amax_out, nullptr,
                            static_cast<cudaStream_t>(stream));
}
