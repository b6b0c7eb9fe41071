// gemm.cu -- a2 (+ fused a3 / a5): the packed FP8 GEMM on sm_100a tensor
// cores (tcgen05 MMA, TMEM accumulators, TMA operand loads).
//
// flashrt-structures 0.2.0, impls/qkv_pack/fp8_static.py (module docstring:
// sibling GEMMs packed into one [sum N_i, K] matrix so the small-M group pays
// one launch; `PackedLinear._run`: out = act_scale * w_scale * (x8 @ w8^T) +
// bias in bf16) and impls/adarms_stack/fp8_chain.py (`norm_project` feeds
// the FP8 wire straight into the GEMM; `_quantize` folds act_scale * w_scale
// into alpha; `down_project` consumes the merged GEGLU requant).
//
// Design (one CTA per SM, persistent over work units):
//   warp 0      one lane issues TMA loads of 128-byte-wide K slices of the A
//               and B tiles into a STAGES-deep ring (128-byte swizzle);
//   warp 1      allocates TMEM, one lane issues tcgen05.mma (M=128, N=BN,
//               K=32, e4m3 x e4m3 -> fp32) into one of two TMEM accumulators;
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane quarter, alpha, bias,
//               bf16 / RoPE + KV scatter / GEGLU + e4m3, stores to HBM; the
//               double-buffered accumulator lets it overlap the next unit's
//               main loop.
// Large M: A = x8 (tokens on TMEM lanes), B = w8, BN = 256 (or 128).
// Small M (<= 128): swap A and B so the packed weights fill the MMA rows (64
// per tile, twice the tiles of 128-row tiles) and the few tokens are the MMA
// N (64 or 128); when the tiles still leave most SMs idle, K is split over
// CTAs so the weight stream is spread across the SMs, and the CTA that
// finishes a tile last sums the fp32 partials in split order (deterministic,
// no atomics on data, no waiting between CTAs).
// Every wait on an mbarrier is bounded in time; a wait that runs out records
// FRT_ETIMEOUT, the CTA drains its in-flight copies and MMAs (again bounded),
// frees its TMEM and returns.  No TMA multicast is used anywhere.
#include <mutex>
#include <type_traits>

#include "frt_common.cuh"
#include "frt_sm100.cuh"

namespace frt {
namespace {

constexpr int BM = 128;             // MMA M of the normal orientation
constexpr int BK = 128;             // K bytes per stage: one swizzle row
constexpr int kThreads = 192;
constexpr int kPairEpiWarps = 8;    // CTA-pair kernel: two epilogue warps per TMEM lane quarter
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;
constexpr int kMaxCluster = 8;      // portable thread-block cluster size
constexpr uint64_t kWaitNs = 2000000000ull;   // 2 s per wait
constexpr uint64_t kDrainNs = 200000000ull;   // 0.2 s to drain after an abort

enum { EPI_BF16 = 0, EPI_GEGLU = 1, EPI_ROPE = 2, EPI_GELU = 3 };

#ifndef FRT_MIN_KB_PER_SPLIT
#define FRT_MIN_KB_PER_SPLIT 16  // K-blocks (of 128) per split at least
#endif

struct GemmParams {
  int M, N, K;
  int a_tiles, b_tiles, k_blocks, splits, units;
  const float* act_scale;
  const float* w_scale;
  const uint16_t* bias;
  int epi;
  void* out;
  long ldo;
  const float* out_scale;
  // split + RoPE + KV epilogue
  int Mseq, hq, hkv, hd, P, T;
  const uint16_t* rope;
  uint16_t* q_out;
  uint16_t* k_cache;
  uint16_t* v_cache;
  // split-K
  float* partials;
  unsigned* counters;
  int* status;
};

__host__ __device__ constexpr uint32_t tmem_cols_for(int n) {
  return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

__device__ __forceinline__ void record_timeout(int* status) {
  if (status) atomicExch(status, FRT_ETIMEOUT);
}

// ---------------------------------------------------------------- epilogue --

// One token row m, output columns n0 .. n0 + W - 1 (W = 8 or 16, n0 % W == 0,
// inside one head): the same arithmetic as warp_rows_epilogue at 16-byte
// granularity, in two steps.  item_plan works out, ahead of the
// accumulators, where each 8-column piece goes and loads the rope and bias
// pieces it needs; item_apply then only scales, adds, rotates and stores
// (a short dependency chain: the epilogue of a small tile runs one warp per
// scheduler, so every dependent instruction after the data arrives counts).
template <int W>
struct ItemPlan {
  uint16_t* dst[W / 8];  // nullptr: the item lies outside the output
  uint4 bias8[W / 8], rope8[W / 8];
  bool rot;
};

template <int W>
__device__ __forceinline__ void item_plan(const GemmParams& p, int m, int n0, ItemPlan<W>& it) {
#pragma unroll
  for (int g = 0; g < W / 8; ++g) {
    it.dst[g] = nullptr;
    it.bias8[g] = it.rope8[g] = make_uint4(0, 0, 0, 0);
  }
  it.rot = false;
  if (n0 >= p.N || m >= p.M) return;
  const int b = m / p.Mseq, s = m % p.Mseq;
  const int h = n0 / p.hd, d00 = n0 % p.hd;
  it.rot = p.epi == EPI_ROPE && h < p.hq + p.hkv;
#pragma unroll
  for (int g = 0; g < W / 8; ++g) {
    if (p.bias) it.bias8[g] = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + 8 * g));
    if (it.rot)
      it.rope8[g] = __ldg(reinterpret_cast<const uint4*>(p.rope + long(s) * p.hd + d00 + 8 * g));
    const int d0 = d00 + 8 * g;
    if (p.epi == EPI_BF16)
      it.dst[g] = static_cast<uint16_t*>(p.out) + long(m) * p.ldo + n0 + 8 * g;
    else if (h < p.hq)
      it.dst[g] = p.q_out + ((long(b) * p.Mseq + s) * p.hq + h) * p.hd + d0;
    else if (h < p.hq + p.hkv)
      it.dst[g] = p.k_cache + ((long(b) * p.T + p.P + s) * p.hkv + (h - p.hq)) * p.hd + d0;
    else
      it.dst[g] = p.v_cache + ((long(b) * p.T + p.P + s) * p.hkv + (h - p.hq - p.hkv)) * p.hd + d0;
  }
}

template <int W>
__device__ __forceinline__ void item_apply(const GemmParams& p, const float (&v)[W], float alpha,
                                           const ItemPlan<W>& it) {
#pragma unroll
  for (int g = 0; g < W / 8; ++g) {
    if (!it.dst[g]) continue;
    float y[8];
    if (p.bias) {
      float bb[8];
      unpack8(it.bias8[g], bb);
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = bf2f(f2bf(__fadd_rn(__fmul_rn(v[8 * g + j], alpha), bb[j])));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) y[j] = bf2f(f2bf(__fmul_rn(v[8 * g + j], alpha)));
    }
    if (it.rot) {
      float r[8];
      unpack8(it.rope8[g], r);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float c = r[2 * i], sn = r[2 * i + 1];
        const float x0 = y[2 * i], x1 = y[2 * i + 1];
        y[2 * i] = __fsub_rn(__fmul_rn(x0, c), __fmul_rn(x1, sn));
        y[2 * i + 1] = __fadd_rn(__fmul_rn(x0, sn), __fmul_rn(x1, c));
      }
    }
    *reinterpret_cast<uint4*>(it.dst[g]) = pack8_bf16(y);
  }
}

// ------------------------------------------------- staged row epilogue --
//
// The normal orientation leaves accumulator row m_base + lane of a warp's 32
// rows in each thread.  Written straight from registers, every store
// instruction of the warp would touch 32 rows (32 cache lines for 16 bytes
// each), which made the output path slower than the main loop.  Instead each
// warp stages 32 rows x 128 bytes of finished output in its own 4 KB of
// shared memory (16-byte units swizzled by row, so both the row-wise writes
// and the column-wise reads are conflict-free) and writes them back as whole
// 128-byte row segments: eight threads per row, four rows per store.  The
// RoPE rotation runs in that write-back, on the staged bf16 values (the
// unfused form rotates the same bf16-rounded values), so the rope-table
// loads are row segments too.
constexpr int kEpiStageBytes = 32 * 128;   // one warp's staging buffer

__device__ __forceinline__ void stage_put(uint8_t* buf, int row, int unit, const uint4& v) {
  *reinterpret_cast<uint4*>(buf + row * 128 + ((unit ^ (row & 7)) << 4)) = v;
}
__device__ __forceinline__ uint4 stage_get(const uint8_t* buf, int row, int unit) {
  return *reinterpret_cast<const uint4*>(buf + row * 128 + ((unit ^ (row & 7)) << 4));
}

// Write-back of the staged bf16 rows of one 64-column group.  Thread (row
// r = lane/8 + 4i, unit u = lane % 8) writes output columns n0 + 8u .. +7 of
// token row m_base + r; with the RoPE epilogue q and k heads are rotated
// with the table row of their position and q / k / v go to their buffers
// (the 8 columns of a unit lie inside one head: hd % 8 == 0).  The rope
// rows are requested (rope_rows) before the group's accumulators are read,
// so those loads overlap the TMEM loads and the arithmetic.
__device__ __forceinline__ void rope_rows(const GemmParams& p, int lane, int m_base, int n0,
                                          uint4 (&rv)[8]) {
  const int n = n0 + 8 * (lane & 7);
  const int h = n / p.hd, d0 = n - h * p.hd;
  if (p.epi != EPI_ROPE || n >= p.N || h >= p.hq + p.hkv) return;
  const int m0 = m_base + (lane >> 3);
  int s = m0 % p.Mseq;
  const uint16_t* rr = p.rope + long(s) * p.hd + d0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (m0 + 4 * i < p.M) rv[i] = __ldg(reinterpret_cast<const uint4*>(rr));
    rr += 4 * p.hd;
    s += 4;
    while (s >= p.Mseq) { s -= p.Mseq; rr -= long(p.Mseq) * p.hd; }
  }
}

// The destinations of one unit's rows step by a constant: q rows are token
// rows (b * M + s), cache rows b * T + P + s jump by T - M where s wraps.
__device__ __forceinline__ void flush_rows_bf16(const GemmParams& p, const uint8_t* buf, int lane,
                                                int m_base, int n0, int units,
                                                const uint4 (&rv)[8]) {
  __syncwarp();
  const int u = lane & 7, r0 = lane >> 3;
  const int n = n0 + 8 * u;
  if (u < units && n < p.N) {
    const int m0 = m_base + r0;
    if (p.epi == EPI_BF16) {
      uint16_t* base = static_cast<uint16_t*>(p.out) + n;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (m0 + 4 * i < p.M)
          *reinterpret_cast<uint4*>(base + long(m0 + 4 * i) * p.ldo) =
              stage_get(buf, r0 + 4 * i, u);
    } else {  // EPI_ROPE
      const int h = n / p.hd, d0 = n - h * p.hd;
      const bool rot = h < p.hq + p.hkv;
      const int b = m0 / p.Mseq;
      int s = m0 - b * p.Mseq;
      uint16_t* dst;
      long step, wrap;
      if (h < p.hq) {
        dst = p.q_out + (long(m0) * p.hq + h) * p.hd + d0;
        step = 4L * p.hq * p.hd;
        wrap = 0;
      } else {
        const int hh = rot ? h - p.hq : h - p.hq - p.hkv;
        dst = (rot ? p.k_cache : p.v_cache) + ((long(b) * p.T + p.P + s) * p.hkv + hh) * p.hd + d0;
        step = 4L * p.hkv * p.hd;
        wrap = long(p.T - p.Mseq) * p.hkv * p.hd;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (m0 + 4 * i < p.M) {
          uint4 x = stage_get(buf, r0 + 4 * i, u);
          if (rot) x = rope_rotate8(x, rv[i]);
          *reinterpret_cast<uint4*>(dst) = x;
        }
        dst += step;
        s += 4;
        while (s >= p.Mseq) { s -= p.Mseq; dst += wrap; }
      }
    }
  }
  __syncwarp();
}

// Write back `units` 16-byte units of each staged e4m3 row: row r holds
// output bytes col0 .. col0 + 16 * units - 1 of token row m_base + r.
__device__ __forceinline__ void flush_rows_u8(const GemmParams& p, const uint8_t* buf, int lane,
                                              int m_base, int col0, int units) {
  __syncwarp();
  const int u = lane & 7;
  if (u < units) {
    uint8_t* base = static_cast<uint8_t*>(p.out) + col0 + 16 * u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = (lane >> 3) + 4 * i;
      if (m_base + r < p.M)
        *reinterpret_cast<uint4*>(base + long(m_base + r) * p.ldo) = stage_get(buf, r, u);
    }
  }
  __syncwarp();
}

// 32 bias values of columns n .. n + 31 (bf16 -> fp32); zeros without bias.
__device__ __forceinline__ void load_bias32(const GemmParams& p, int n, uint4 (&b4)[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k)
    b4[k] = p.bias ? __ldg(reinterpret_cast<const uint4*>(p.bias + n) + k) : make_uint4(0, 0, 0, 0);
}

// v = bf16(acc * alpha [+ bias]) as a float, in place: the value the plain
// epilogue stores and the gated epilogues start from.  Paired fp32
// instructions (each lane rounded as the scalar operation), one bf16x2
// rounding per pair.
__device__ __forceinline__ void scale_bias32(const GemmParams& p, float (&v)[32],
                                             const uint4 (&b4)[4], uint64_t alpha2) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t w[4] = {b4[k].x, b4[k].y, b4[k].z, b4[k].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint64_t a = mul2(f2_pack(v[8 * k + 2 * i], v[8 * k + 2 * i + 1]), alpha2);
      if (p.bias) a = add2(a, bf16x2_to_f2(w[i]));
      const uint64_t y = bf16x2_to_f2(pack_bf16x2(f2_lo(a), f2_hi(a)));
      v[8 * k + 2 * i] = f2_lo(y);
      v[8 * k + 2 * i + 1] = f2_hi(y);
    }
  }
}

// 8 accumulators of columns n .. n + 7 -> their 8 bf16 outputs bf16(acc *
// alpha [+ bias]), rounded once, computed as paired fp32 operations (each
// lane rounded exactly as the scalar operation: the same bits, half the
// instructions).
__device__ __forceinline__ uint4 scale_bias_pack8(const float* v, const uint4& b4, uint64_t alpha2,
                                                  bool has_bias) {
  const uint32_t w[4] = {b4.x, b4.y, b4.z, b4.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint64_t a = mul2(f2_pack(v[2 * i], v[2 * i + 1]), alpha2);
    if (has_bias) a = add2(a, bf16x2_to_f2(w[i]));
    o[i] = pack_bf16x2(f2_lo(a), f2_hi(a));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The epilogue of one warp's 32 accumulator rows m_base .. m_base + 31 over
// the accumulator chunks cb .. ce - 1 (32 columns each); load(c, v) fills
// chunk c of this thread's row (warp-uniform), done() runs once this warp's
// last chunk is loaded (it releases the TMEM accumulator).
//   bf16 / RoPE: chunk c -> output columns col0 + 32c (RoPE: rotated);
//   GELU:        the same columns as e4m3(gelu_tanh(y) / out_scale);
//   GEGLU:       chunks c in [cb, ce) (within 0..3) are gate columns
//                col0 + 32c, chunks c + 4 the matching up columns
//                col0 + 128 + 32c; output e4m3 columns out0 + 32c =
//                e4m3(gelu_tanh(gate) * up / out_scale).
// y = bf16(acc * alpha [+ bias]) everywhere; division by out_scale is a
// multiplication by its correctly rounded reciprocal, as in the standalone
// kernels.  Each group of chunks (two for bf16, up to four for e4m3: one
// 128-byte row segment) requests its bias pieces and rope rows first.
template <class Load, class Done>
__device__ __forceinline__ void warp_rows_epilogue(const GemmParams& p, uint8_t* buf, int lane,
                                                   int m_base, int col0, int cb, int ce, int out0,
                                                   float alpha, Load load, Done done) {
  if (p.epi == EPI_GEGLU || p.epi == EPI_GELU) {
    const float inv_os = __frcp_rn(__ldg(p.out_scale));
    const uint64_t half_c = f2_pack(0.5f * inv_os, 0.5f * inv_os);
    const uint64_t alpha2 = f2_pack(alpha, alpha);
    const bool geglu = p.epi == EPI_GEGLU;
#pragma unroll 1
    for (int c0 = cb; c0 < ce; c0 += 4) {
      const int cn = ce - c0 < 4 ? ce - c0 : 4;
#pragma unroll 1
      for (int c = c0; c < c0 + cn; ++c) {
        uint4 bg[4], bu[4];
        load_bias32(p, col0 + 32 * c, bg);
        if (geglu) load_bias32(p, col0 + 128 + 32 * c, bu);
        float q[32];
        load(c, q);
        if (!geglu && c == ce - 1) done();
        scale_bias32(p, q, bg, alpha2);
        if (geglu) {
          float z[32];
          load(c + 4, z);
          if (c == ce - 1) done();
          scale_bias32(p, z, bu, alpha2);
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const uint64_t h = gelu_tanh_scaled2<true>(f2_pack(q[j], q[j + 1]),
                                                       f2_pack(z[j], z[j + 1]), half_c);
            q[j] = f2_lo(h);
            q[j + 1] = f2_hi(h);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const uint64_t h = gelu_tanh_scaled2<false>(f2_pack(q[j], q[j + 1]), 0, half_c);
            q[j] = f2_lo(h);
            q[j + 1] = f2_hi(h);
          }
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          float a8[8], b8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) { a8[j] = q[16 * k + j]; b8[j] = q[16 * k + 8 + j]; }
          const uint2 lo = pack8_e4m3(a8), hi = pack8_e4m3(b8);
          stage_put(buf, lane, 2 * (c - c0) + k, make_uint4(lo.x, lo.y, hi.x, hi.y));
        }
      }
      flush_rows_u8(p, buf, lane, m_base, (geglu ? out0 : col0) + 32 * c0, 2 * cn);
    }
    return;
  }
#pragma unroll 1
  for (int c0 = cb; c0 < ce; c0 += 2) {
    const int cn = ce - c0 < 2 ? ce - c0 : 2;
    uint4 rv[8];
    rope_rows(p, lane, m_base, col0 + 32 * c0, rv);
    uint4 b4[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (j < cn) load_bias32(p, col0 + 32 * (c0 + j), b4[j]);
    const uint64_t alpha2 = f2_pack(alpha, alpha);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      if (j < cn) {
        float v[32];
        load(c0 + j, v);
        if (c0 + j == ce - 1) done();
#pragma unroll
        for (int k = 0; k < 4; ++k)
          stage_put(buf, lane, 4 * j + k, scale_bias_pack8(v + 8 * k, b4[j][k], alpha2, p.bias));
      }
    }
    flush_rows_bf16(p, buf, lane, m_base, col0 + 32 * c0, 4 * cn, rv);
  }
}

// The single-CTA kernel's epilogue (normal orientation): each thread writes
// its own accumulator row m straight from registers, columns col0 + 32c for
// chunks c in [cb, ce) (GEGLU: gate chunks c within 0..3 with up chunks
// c + 4, output columns out0 + 32c).  That kernel runs at most one tile per
// CTA (larger tile counts go to CTA pairs), and so does the pair kernel's
// DIRECT form, so a staged write-back would only add a round trip to a
// latency-bound tile.  The same arithmetic as
// warp_rows_epilogue; each chunk's bias and rope pieces are requested
// before its accumulators are read.
template <class Load, class Done>
__device__ __forceinline__ void rows_direct_epilogue(const GemmParams& p, int m, int col0, int cb,
                                                     int ce, int out0, float alpha, Load load,
                                                     Done done) {
  const bool ok = m < p.M;
  if (p.epi == EPI_GEGLU || p.epi == EPI_GELU) {
    const bool geglu = p.epi == EPI_GEGLU;
    const float inv_os = __frcp_rn(__ldg(p.out_scale));
    const uint64_t half_c = f2_pack(0.5f * inv_os, 0.5f * inv_os);
    const uint64_t alpha2 = f2_pack(alpha, alpha);
    const int nout = ce;
#pragma unroll 1
    for (int c = cb; c < nout; ++c) {
      uint4 bg[4], bu[4];
      load_bias32(p, col0 + 32 * c, bg);
      if (geglu) load_bias32(p, col0 + 128 + 32 * c, bu);
      float q[32];
      load(c, q);
      if (!geglu && c == nout - 1) done();
      scale_bias32(p, q, bg, alpha2);
      if (geglu) {
        float z[32];
        load(c + 4, z);
        if (c == nout - 1) done();
        scale_bias32(p, z, bu, alpha2);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const uint64_t h = gelu_tanh_scaled2<true>(f2_pack(q[j], q[j + 1]),
                                                     f2_pack(z[j], z[j + 1]), half_c);
          q[j] = f2_lo(h);
          q[j + 1] = f2_hi(h);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const uint64_t h = gelu_tanh_scaled2<false>(f2_pack(q[j], q[j + 1]), 0, half_c);
          q[j] = f2_lo(h);
          q[j + 1] = f2_hi(h);
        }
      }
      if (ok) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + long(m) * p.ldo +
                                              (geglu ? out0 : col0) + 32 * c);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          float a8[8], b8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) { a8[j] = q[16 * k + j]; b8[j] = q[16 * k + 8 + j]; }
          const uint2 lo = pack8_e4m3(a8), hi = pack8_e4m3(b8);
          dst[k] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
      }
    }
    return;
  }
  const uint64_t alpha2 = f2_pack(alpha, alpha);
#pragma unroll 1
  for (int c = cb; c < ce; ++c) {
    const int n = col0 + 32 * c;
    uint4 b4[4], rv[4];
    load_bias32(p, n, b4);
    const int h = p.epi == EPI_ROPE ? n / p.hd : 0, d0 = p.epi == EPI_ROPE ? n - h * p.hd : 0;
    const bool rot = p.epi == EPI_ROPE && h < p.hq + p.hkv;
    const int s = ok && p.epi == EPI_ROPE ? m % p.Mseq : 0;
    if (rot && ok) {
      const uint4* rr = reinterpret_cast<const uint4*>(p.rope + long(s) * p.hd + d0);
#pragma unroll
      for (int k = 0; k < 4; ++k) rv[k] = __ldg(rr + k);
    }
    float v[32];
    load(c, v);
    if (c == ce - 1) done();
    if (!ok) continue;
    uint16_t* dst;
    if (p.epi == EPI_BF16) {
      dst = static_cast<uint16_t*>(p.out) + long(m) * p.ldo + n;
    } else {  // the 32 columns lie inside one head (hd % 32 == 0)
      const int b = m / p.Mseq;
      dst = h < p.hq ? p.q_out + (long(m) * p.hq + h) * p.hd + d0
          : h < p.hq + p.hkv
              ? p.k_cache + ((long(b) * p.T + p.P + s) * p.hkv + (h - p.hq)) * p.hd + d0
              : p.v_cache + ((long(b) * p.T + p.P + s) * p.hkv + (h - p.hq - p.hkv)) * p.hd + d0;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint4 x = scale_bias_pack8(v + 8 * k, b4[k], alpha2, p.bias);
      if (rot) x = rope_rotate8(x, rv[k]);
      reinterpret_cast<uint4*>(dst)[k] = x;
    }
  }
}

// TMEM lane holding accumulator row r of an MMA with M = BMT rows: all 128
// lanes for M = 128; for M = 64 the rows fill the first 16 lanes of each
// 32-lane quarter (rows 16q .. 16q+15 in lanes 32q .. 32q+15).  The epilogue
// warp of quarter q therefore owns rows 16q + lane (lane < 16) when BMT = 64.
template <int BMT>
__device__ __forceinline__ int acc_row(int q, int lane) {
  return BMT == 128 ? 32 * q + lane : 16 * q + lane;
}
template <int BMT>
__device__ __forceinline__ bool acc_row_valid(int lane) {
  return BMT == 128 || lane < 16;
}

// Swapped orientation, emitting half: the tile's (token, W-column) items,
// numbered token-major so neighbouring threads write neighbouring 16-byte
// pieces of one token row.  This thread takes items [lo, hi) with stride
// 128 over the four epilogue warps.  fetch(m_local, cw, v) gathers the
// item's W fp32 accumulators (output columns W*cw .. W*cw+W-1 of token
// m_local); the item's rope and bias loads are issued before it.
template <int BMT, int BN, int W, class Fetch>
__device__ __forceinline__ void emit_swap_items(const GemmParams& p, int ta, int tb, float alpha,
                                                int lo, int hi, Fetch fetch) {
  constexpr int CW = BMT / W;
  const int t = int(threadIdx.x) - 64;  // 0 .. 127 over the four epilogue warps
#pragma unroll 1
  for (int it = lo + t; it < hi; it += 128) {
    const int m_local = it / CW, cw = it % CW;
    const int n0 = ta * BMT + W * cw;
    const int m = tb * BN + m_local;
    if (n0 >= p.N || m >= p.M) continue;
    ItemPlan<W> ip;
    item_plan<W>(p, m, n0, ip);
    float v[W];
    fetch(m_local, cw, v);
    item_apply<W>(p, v, alpha, ip);
  }
}

// Run the epilogue of one tile.  load(c, v) fills v with accumulator chunk c
// (32 columns of this thread's TMEM lane); it is called warp-uniformly.
// done() runs once every chunk has been loaded (it releases the TMEM
// accumulator when the chunks come from TMEM).
// Normal orientation: each thread's row through rows_direct_epilogue.
// Swapped orientation: the chunks are staged in
// the shared-memory tile T (fp32 [BMT output columns][BN tokens], row
// stride BN + 4) and read back transposed, token-major, so neighbouring
// threads write neighbouring 16-byte pieces of one token row.
template <bool SWAP, int BMT, int BN, class Load, class Done>
__device__ __forceinline__ void tile_epilogue(const GemmParams& p, int ta, int tb, int q, int lane,
                                              float alpha, float* T, Load load, Done done) {
  if (!SWAP) {
    int c_last = BN / 32 - 1;
    while (c_last > 0 && tb * BN + 32 * c_last >= p.N) --c_last;
    rows_direct_epilogue(p, ta * BMT + 32 * q + lane, tb * BN, 0,
                         p.epi == EPI_GEGLU ? 4 : c_last + 1, tb * 128, alpha, load, done);
    return;
  }
  constexpr int TS = BMT + 4;
  const int row = acc_row<BMT>(q, lane);
  const bool valid = acc_row_valid<BMT>(lane);
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    float v[32];
    load(c, v);
    if (valid) {
#pragma unroll
      for (int j = 0; j < 32; ++j) T[(32 * c + j) * TS + row] = v[j];
    }
  }
  done();
  named_bar_sync(2, 128);
  emit_swap_items<BMT, BN, 8>(p, ta, tb, alpha, 0, BN * (BMT / 8),
                              [&](int m_local, int c8, float (&v)[8]) {
    const float4* src = reinterpret_cast<const float4*>(T + m_local * TS + 8 * c8);
    const float4 a = src[0], b = src[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  });
  named_bar_sync(2, 128);
}

// Swapped orientation, staging half: the accumulator of this thread's TMEM
// lane (an output column) goes to the token-major tile T
// ([BN tokens][BMT + 4] fp32) in this CTA's shared memory.
template <int BMT, int BN, class Load>
__device__ __forceinline__ void stage_swap_tile(float* T, int q, int lane, Load load) {
  constexpr int TS = BMT + 4;
  const int row = acc_row<BMT>(q, lane);
  const bool valid = acc_row_valid<BMT>(lane);
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    float v[32];
    load(c, v);
    if (valid) {
#pragma unroll
      for (int j = 0; j < 32; ++j) T[(32 * c + j) * TS + row] = v[j];
    }
  }
}

// ------------------------------------------------------------------ kernel --

template <bool SWAP, int BMT, int BN>
__host__ __device__ constexpr int t_tile_bytes() {
  return SWAP ? BN * (BMT + 4) * 4 : 0;
}

template <bool SWAP, int BMT, int BN, int STAGES>
__host__ __device__ constexpr int smem_total() {
  return STAGES * (BMT * BK + BN * BK) + t_tile_bytes<SWAP, BMT, BN>() + 1024 + 512;
}

// CLUSTER: the p.splits K-splits of a tile run as one thread-block cluster
// (rank = split, one unit per CTA); each CTA stages its fp32 partial in its
// shared memory.  The leader's (rank 0's) last MMA commit also arrives on
// the other ranks' `go` barriers (commit multicast), so they learn its
// operand ring is free the moment its MMAs complete; each then bulk-copies its
// staged partial into slot rank-1 of the leader's ring, counted as
// transaction bytes on the leader's barrier red_full, and leaves once the
// leader confirms receipt.  The leader sums the partials in rank order from
// its own shared memory and runs the whole tile's epilogue, with the rope
// and bias operands loaded while the main loop ran -- no global partials,
// no atomics, no full-cluster barrier on the output path.
template <bool SWAP, int BMT, int BN, int STAGES, bool CLUSTER>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const GemmParams p) {
  static_assert(SWAP || BMT == 128, "the normal orientation uses 128-row tiles");
  static_assert(!CLUSTER || SWAP, "cluster K-splits serve the swapped orientation");
  constexpr int A_BYTES = BMT * BK;
  constexpr int B_BYTES = BN * BK;
  constexpr uint32_t TMEM_COLS = tmem_cols_for(2 * BN);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  float* T = reinterpret_cast<float*>(sB + STAGES * B_BYTES);
  uint64_t* full =
      reinterpret_cast<uint64_t*>(sB + STAGES * B_BYTES + t_tile_bytes<SWAP, BMT, BN>());
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* red_full = drain + 1;  // CLUSTER leader: the other ranks' partials
  uint64_t* go = drain + 2;        // CLUSTER other ranks: the leader's ring is free
  uint64_t* done = drain + 3;      // CLUSTER other ranks: the leader has the partial
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* last_flag = abort_flag + 1;
  volatile int* epi_ok = abort_flag + 2;  // [4], one per epilogue warp

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the next kernel in the stream may start its prologue now; it waits for
  // this grid's completion before touching memory
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    if (CLUSTER) {
      mbar_init(red_full, 1);
      mbar_init(go, 1);
      mbar_init(done, 1);
    }
    *abort_flag = 0;
    *last_flag = 0;
    fence_barrier_init();
    if (CLUSTER && cluster_ctarank() == 0 && p.splits > 1)
      mbar_arrive_expect_tx(red_full, uint32_t(p.splits - 1) * t_tile_bytes<SWAP, BMT, BN>());
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  __syncwarp();  // warp 0's lanes wait for lane 0's barrier set-up
  tc_fence_before();
  __syncthreads();
  if (CLUSTER) cluster_arrive_relaxed();  // this CTA's barriers exist
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      // The packed weights are not written by the kernel this one may
      // overlap: the first unit's weight slices are requested before waiting
      // on the kernel that produces the activations, so they stream in while
      // it finishes.
      const CUtensorMap* wmap = SWAP ? &tmA : &tmB;
      const CUtensorMap* xmap = SWAP ? &tmB : &tmA;
      const int u0 = blockIdx.x;
      int n_pre = 0;
      if (u0 < p.units) {
        const int tile = u0 / p.splits, split = u0 % p.splits;
        const int ta = tile % p.a_tiles, tb = tile / p.a_tiles;
        const int kb0 = int(long(split) * p.k_blocks / p.splits);
        const int kb1 = int(long(split + 1) * p.k_blocks / p.splits);
        n_pre = kb1 - kb0 < STAGES ? kb1 - kb0 : STAGES;
        for (int i = 0; i < n_pre; ++i) {
          mbar_arrive_expect_tx(&full[i], A_BYTES + B_BYTES);
          if (SWAP) tma_load_2d(sA + i * A_BYTES, wmap, &full[i], (kb0 + i) * BK, ta * BMT);
          else tma_load_2d(sB + i * B_BYTES, wmap, &full[i], (kb0 + i) * BK, tb * BN);
        }
      }
      pdl_wait();
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = u0; u < p.units && ok; u += gridDim.x) {
        const int tile = u / p.splits, split = u % p.splits;
        const int ta = tile % p.a_tiles, tb = tile / p.a_tiles;
        const int kb0 = int(long(split) * p.k_blocks / p.splits);
        const int kb1 = int(long(split + 1) * p.k_blocks / p.splits);
        for (int kb = kb0; kb < kb1; ++kb) {
          const bool pre = (u == u0) && (kb - kb0 < n_pre);
          if (!pre) {
            if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, kWaitNs, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], A_BYTES + B_BYTES);
            if (SWAP) tma_load_2d(sA + stage * A_BYTES, wmap, &full[stage], kb * BK, ta * BMT);
            else tma_load_2d(sB + stage * B_BYTES, wmap, &full[stage], kb * BK, tb * BN);
          }
          if (!(SWAP && CLUSTER && pre)) {
            if (SWAP) tma_load_2d(sB + stage * B_BYTES, xmap, &full[stage], kb * BK, tb * BN);
            else tma_load_2d(sA + stage * A_BYTES, xmap, &full[stage], kb * BK, ta * BMT);
          }
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        record_timeout(p.status);
        *abort_flag = 1;
        // drain: wait (bounded) for the copies still in flight, newest first
        int st = stage;
        uint32_t ph = phase;
        for (int i = 0; i < issued && i < STAGES; ++i) {
          if (--st < 0) { st = STAGES - 1; ph ^= 1u; }
          mbar_wait_bounded(&full[st], ph, kDrainNs, nullptr);
        }
      }
    }
    // the other 31 lanes wait here for lane 0, so the warp reaches the block
    // barrier below converged (an aligned barrier must not be met by part of
    // a warp while the rest is still working)
    __syncwarp();
    if (CLUSTER) cluster_wait();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    // (cluster: the other ranks' barriers exist before the commit below
    // arrives on them)
    if (CLUSTER) cluster_wait();
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(BMT, BN);
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++local) {
        const int split = u % p.splits;
        const int kb0 = int(long(split) * p.k_blocks / p.splits);
        const int kb1 = int(long(split + 1) * p.k_blocks / p.splits);
        const int ab = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[ab], aph ^ 1u, kWaitNs, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dcol = tmem_base + uint32_t(ab * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, kWaitNs, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = sdesc_k_sw128(a_base + stage * A_BYTES);
          const uint64_t bd = sdesc_k_sw128(b_base + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            umma_e4m3(dcol, ad + 2 * k, bd + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[ab]);
        // cluster leader: its ring is free once these MMAs complete; the
        // same completion tells the other ranks to send their partials
        if (CLUSTER && p.splits > 1 && cluster_ctarank() == 0)
          umma_commit_mc(go, uint16_t(((1u << p.splits) - 1u) & ~1u));
      }
      if (!ok) {
        record_timeout(p.status);
        *abort_flag = 1;
        umma_commit(drain);  // completes when every MMA issued so far is done
        mbar_wait_bounded(drain, 0, kDrainNs, nullptr);
      }
    }
    __syncwarp();  // converge before the block barrier and the TMEM release
  } else {
    // ----------------------------------------------------------- epilogue --
    // The rope table is bind-time data: pull this CTA's first-unit rows into
    // L2 before waiting on the previous kernel, so the epilogue finds them.
    if (p.epi == EPI_ROPE && blockIdx.x < unsigned(p.units)) {
      const int tile0 = int(blockIdx.x) / p.splits;
      const int tok_tile = SWAP ? tile0 / p.a_tiles : tile0 % p.a_tiles;
      const int tok_rows = SWAP ? BN : BMT;
      const long row_bytes = long(p.hd) * 2;
      const int t = int(threadIdx.x) - 64;
      for (int r = t; r < tok_rows; r += 128) {
        const int m = tok_tile * tok_rows + r;
        if (m >= p.M) break;
        const char* base = reinterpret_cast<const char*>(p.rope + long(m % p.Mseq) * p.hd);
        for (long off = 0; off < row_bytes; off += 128) prefetch_l2(base + off);
      }
    }
    pdl_wait();
    if (SWAP && CLUSTER && lane == 0 && blockIdx.x < unsigned(p.units)) {
      // the activation boxes of the stages prefetched with weights, spread
      // over the four epilogue warps (idle until the accumulator is full):
      // the stages fill in about the time of one box instead of one after
      // another behind the producer thread's issue
      const int u0 = blockIdx.x;
      const int tile = u0 / p.splits, split = u0 % p.splits;
      const int tb = tile / p.a_tiles;
      const int kb0 = int(long(split) * p.k_blocks / p.splits);
      const int kb1 = int(long(split + 1) * p.k_blocks / p.splits);
      const int n_pre = kb1 - kb0 < STAGES ? kb1 - kb0 : STAGES;
      for (int i = warp - 2; i < n_pre; i += 4)
        tma_load_2d(sB + i * B_BYTES, &tmB, &full[i], (kb0 + i) * BK, tb * BN);
    }
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const float alpha = __fmul_rn(__ldg(p.act_scale), __ldg(p.w_scale));
    const int row = acc_row<BMT>(q, lane);
    const bool valid = acc_row_valid<BMT>(lane);
    // CLUSTER leader: the rope and bias pieces of its items, loaded while
    // the main loop runs (they are read-only here and written, if at all,
    // by kernels that completed before the dependency wait above)
    constexpr int LW = 16;                          // columns per leader item
    constexpr int LNI = CLUSTER ? BN * (BMT / LW) / 128 : 1;  // items per thread
    ItemPlan<LW> lplan[LNI];
    const uint32_t crank = CLUSTER ? cluster_ctarank() : 0u;
    if constexpr (CLUSTER) if (crank == 0 && blockIdx.x < unsigned(p.units)) {
      const int tile = int(blockIdx.x) / p.splits;
      const int ta = tile % p.a_tiles, tb = tile / p.a_tiles;
#pragma unroll
      for (int i = 0; i < LNI; ++i) {
        const int it = int(threadIdx.x) - 64 + 128 * i;
        item_plan<LW>(p, tb * BN + it / (BMT / LW), ta * BMT + LW * (it % (BMT / LW)), lplan[i]);
      }
    }
    bool staged = false, cwaited = false;
    int local = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++local) {
      const int tile = u / p.splits, split = u % p.splits;
      const int ta = tile % p.a_tiles, tb = tile / p.a_tiles;
      const int ab = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      // All four epilogue warps agree on whether the accumulator arrived, so
      // none of them can be left alone at a named barrier.
      const bool got = __all_sync(0xffffffffu,
                                  mbar_wait_bounded(&tfull[ab], aph, kWaitNs, abort_flag));
      if (lane == 0) epi_ok[q] = got ? 1 : 0;
      named_bar_sync(1, 128);
      const bool all_ok = epi_ok[0] && epi_ok[1] && epi_ok[2] && epi_ok[3];
      named_bar_sync(1, 128);
      if (!all_ok) {
        if (lane == 0) record_timeout(p.status);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + uint32_t(ab * BN) + (uint32_t(32 * q) << 16);
      if constexpr (CLUSTER) {
        // one unit per CTA: stage this rank's partial (the leader's MMA
        // completion has already told the other ranks its ring is free)
        cluster_wait();
        cwaited = true;
        stage_swap_tile<BMT, BN>(T, q, lane,
                                 [&](int c, float (&v)[32]) { tmem_ld32(tbase + 32 * c, v); });
        staged = true;
        break;
      }
      auto release_tmem = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[ab]);
      };
      if (p.splits == 1) {
        tile_epilogue<SWAP, BMT, BN>(
            p, ta, tb, q, lane, alpha, T,
            [&](int c, float (&v)[32]) { tmem_ld32(tbase + 32 * c, v); }, release_tmem);
      } else {
        // spill this split's fp32 partial, accumulator-row major
        float* part = p.partials + (long(tile) * p.splits + split) * (BMT * BN) + long(row) * BN;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tbase + 32 * c, v);
          if (valid) {
            float4* d4 = reinterpret_cast<float4*>(part + 32 * c);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              d4[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
          }
        }
        release_tmem();
        __threadfence();
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) {
          const unsigned old = atomicAdd(&p.counters[tile], 1u);
          *last_flag = (old == unsigned(p.splits - 1)) ? 1 : 0;
        }
        named_bar_sync(1, 128);
        if (*last_flag) {
          __threadfence();
          const float* base = p.partials + long(tile) * p.splits * (BMT * BN) + long(row) * BN;
          tile_epilogue<SWAP, BMT, BN>(
              p, ta, tb, q, lane, alpha, T,
              [&](int c, float (&v)[32]) {
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = 0.0f;
                if (!valid) return;
                // the splits in order, eight 16-byte loads in flight per step
#pragma unroll 1
                for (int s = 0; s < p.splits; ++s) {
                  const float4* s0 =
                      reinterpret_cast<const float4*>(base + long(s) * (BMT * BN) + 32 * c);
                  float4 f[8];
#pragma unroll
                  for (int k = 0; k < 8; ++k) f[k] = __ldcg(s0 + k);
#pragma unroll
                  for (int k = 0; k < 8; ++k) {
                    v[4 * k] = __fadd_rn(v[4 * k], f[k].x);
                    v[4 * k + 1] = __fadd_rn(v[4 * k + 1], f[k].y);
                    v[4 * k + 2] = __fadd_rn(v[4 * k + 2], f[k].z);
                    v[4 * k + 3] = __fadd_rn(v[4 * k + 3], f[k].w);
                  }
                }
              },
              [] {});
          if (threadIdx.x == 64) p.counters[tile] = 0u;
        }
        named_bar_sync(1, 128);
      }
    }
    if constexpr (CLUSTER) {
      if (!cwaited) cluster_wait();
      constexpr uint32_t TB = uint32_t(t_tile_bytes<SWAP, BMT, BN>());
      const bool fits = uint32_t(p.splits - 1) * TB <= uint32_t(STAGES * (A_BYTES + B_BYTES));
      if (staged && !fits) {
        if (threadIdx.x == 64) record_timeout(p.status);  // the host never plans this
      } else if (staged && crank != 0) {
        // hand the staged partial to the leader, then wait for its receipt
        // (this CTA's shared memory must outlive the copy)
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (threadIdx.x == 64) {
          if (mbar_wait_bounded_cluster(go, 0, kWaitNs)) {
            bulk_copy_to_peer(map_cluster(smem_u32(smem) + (crank - 1u) * TB, 0), T, TB,
                              map_cluster(smem_u32(red_full), 0));
            if (!mbar_wait_bounded_cluster(done, 0, kWaitNs)) record_timeout(p.status);
          } else {
            record_timeout(p.status);
          }
        }
        __syncwarp();
      } else if (staged) {
        // leader: own partial complete, then the others' in its ring
        named_bar_sync(1, 128);
        const bool got = mbar_wait_bounded_cluster(red_full, 0, kWaitNs);
        if (threadIdx.x == 64) {
          if (got) {
            for (int j = 1; j < p.splits; ++j)
              mbar_arrive_relaxed_cluster(map_cluster(smem_u32(done), uint32_t(j)));
          } else {
            record_timeout(p.status);
          }
        }
        if (got) {
          constexpr int TS = BMT + 4, CW = BMT / LW;
          const float* slots = reinterpret_cast<const float*>(smem);
          const int nsl = p.splits - 1;
#pragma unroll
          for (int i = 0; i < LNI; ++i) {
            const int it = int(threadIdx.x) - 64 + 128 * i;
            const int off = (it / CW) * TS + LW * (it % CW);
            float v[LW];
#pragma unroll
            for (int j = 0; j < LW; ++j) v[j] = 0.0f;
            auto add = [&](const float* src) {
              const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
              for (int k = 0; k < LW / 4; ++k) {
                const float4 f = s4[k];
                v[4 * k] = __fadd_rn(v[4 * k], f.x);
                v[4 * k + 1] = __fadd_rn(v[4 * k + 1], f.y);
                v[4 * k + 2] = __fadd_rn(v[4 * k + 2], f.z);
                v[4 * k + 3] = __fadd_rn(v[4 * k + 3], f.w);
              }
            };
            add(T + off);  // rank 0, then ranks 1 .. splits-1
            for (int sl = 0; sl < nsl; ++sl) add(slots + sl * int(TB / 4) + off);
            item_apply<LW>(p, v, alpha, lplan[i]);
          }
        }
      }
    }
  }


  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------- CTA-pair kernel --
//
// Normal orientation, tiles of 256 rows x BN columns per CTA pair (a
// cluster of 2): each CTA loads its 128 rows of x8 and BN/2 rows of w8 per
// K-block, the even CTA issues tcgen05.mma.cta_group::2 (M = 256, N = BN)
// over both CTAs' shared memory, and each CTA's epilogue drains its own 128
// accumulator rows from its own TMEM.  Per K-block an SM moves 16 KB +
// BN*64 B instead of 16 KB + BN*128 B for the same MMA work, so the same
// shared-memory ring hides more latency.
//   full[s]   (even CTA) 2 arrivals: each CTA's producer arms its bytes;
//             both CTAs' TMA loads complete on it
//   empty[s]  (each CTA) released by the even CTA's multicast commit
//   tfull[b]  (each CTA) accumulator b ready, multicast commit
//   tempty[b] (even CTA) 16 arrivals: the eight epilogue warps of each CTA
//             (two per TMEM lane quarter, each draining half the columns)
// DIRECT (plans with at most one tile per pair, filling most pairs): the
// epilogue writes each thread's row straight from registers instead of
// staging it.
// All waits are bounded; a final cluster barrier keeps both CTAs (their
// shared memory and TMEM) alive until the pair is done.
template <int BN, int STAGES, bool DIRECT>
__global__ void __launch_bounds__(kPairThreads, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmParams p) {
  constexpr int A_BYTES = 128 * BK;
  constexpr int B_BYTES = (BN / 2) * BK;
  constexpr uint32_t TMEM_COLS = tmem_cols_for(2 * BN);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* ebuf_base = sB + STAGES * B_BYTES;  // the epilogue warps' row staging
  uint64_t* full = reinterpret_cast<uint64_t*>(ebuf_base + kPairEpiWarps * kEpiStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_ok = abort_flag + 2;  // [kPairEpiWarps]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;
  const int pair = int(blockIdx.x >> 1), npairs = int(gridDim.x >> 1);
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kPairEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t full_lead = map_cluster(smem_u32(full), 0);
  const uint32_t tempty_lead = map_cluster(smem_u32(tempty), 0);

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      const int u0 = pair;
      int n_pre = 0;
      if (u0 < p.units) {  // weights first, before the dependency wait
        const int tn = u0 / p.a_tiles;
        n_pre = p.k_blocks < STAGES ? p.k_blocks : STAGES;
        for (int i = 0; i < n_pre; ++i) {
          mbar_arrive_expect_tx_cluster(full_lead + 8u * i, A_BYTES + B_BYTES);
          tma_load_2d_pair(sB + i * B_BYTES, &tmB, full_lead + 8u * i, i * BK,
                           tn * BN + int(rank) * (BN / 2));
        }
      }
      pdl_wait();
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = u0; u < p.units && ok; u += npairs) {
        const int tm = u % p.a_tiles, tn = u / p.a_tiles;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          const bool pre = (u == u0) && (kb < n_pre);
          if (!pre) {
            if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, kWaitNs, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx_cluster(full_lead + 8u * stage, A_BYTES + B_BYTES);
            tma_load_2d_pair(sB + stage * B_BYTES, &tmB, full_lead + 8u * stage, kb * BK,
                             tn * BN + int(rank) * (BN / 2));
          }
          tma_load_2d_pair(sA + stage * A_BYTES, &tmA, full_lead + 8u * stage, kb * BK,
                           tm * 256 + int(rank) * 128);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        record_timeout(p.status);
        *abort_flag = 1;
        if (lead) {  // the even CTA's barriers count both CTAs' copies
          int st = stage;
          uint32_t ph = phase;
          for (int i = 0; i < issued && i < STAGES; ++i) {
            if (--st < 0) { st = STAGES - 1; ph ^= 1u; }
            mbar_wait_bounded(&full[st], ph, kDrainNs, nullptr);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------ MMA issuer (even CTA) --
    if (lane == 0 && lead) {
      constexpr uint32_t idesc = idesc_e4m3_f32(256, BN);
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair; u < p.units && ok; u += npairs, ++local) {
        const int ab = local & 1;
        const uint32_t aph = (local >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[ab], aph ^ 1u, kWaitNs, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dcol = tmem_base + uint32_t(ab * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, kWaitNs, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = sdesc_k_sw128(a_base + stage * A_BYTES);
          const uint64_t bd = sdesc_k_sw128(b_base + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            umma_pair_e4m3(dcol, ad + 2 * k, bd + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          umma_pair_commit(&empty[stage], 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_pair_commit(&tfull[ab], 0x3);
      }
      if (!ok) {
        record_timeout(p.status);
        *abort_flag = 1;
        umma_pair_commit(drain, 0x1);
        mbar_wait_bounded(drain, 0, kDrainNs, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- epilogue --
    pdl_wait();
    const int ew = warp - 2;               // 0 .. kPairEpiWarps - 1
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int half = ew >> 2;              // which half of the tile's chunks it drains
    uint8_t* ebuf = ebuf_base + ew * kEpiStageBytes;
    // chunks [cb, ce) of this warp: the two warps of a lane quarter split
    // the tile's columns (GEGLU: its four gate chunks, each with its up chunk)
    constexpr int NCH = BN / 32;
    const int nch = p.epi == EPI_GEGLU ? 4 : NCH;
    const int cb = half ? (nch + 1) / 2 : 0, ce = half ? nch : (nch + 1) / 2;
    const float alpha = __fmul_rn(__ldg(p.act_scale), __ldg(p.w_scale));
    int local = 0;
    for (int u = pair; u < p.units; u += npairs, ++local) {
      const int tm = u % p.a_tiles, tn = u / p.a_tiles;
      const int ab = local & 1;
      const uint32_t aph = (local >> 1) & 1;
      const bool got = __all_sync(0xffffffffu,
                                  mbar_wait_bounded(&tfull[ab], aph, kWaitNs, abort_flag));
      if (lane == 0) epi_ok[ew] = got ? 1 : 0;
      named_bar_sync(1, 32 * kPairEpiWarps);
      bool all_ok = true;
#pragma unroll
      for (int i = 0; i < kPairEpiWarps; ++i) all_ok = all_ok && epi_ok[i];
      named_bar_sync(1, 32 * kPairEpiWarps);
      if (!all_ok) {
        if (lane == 0) record_timeout(p.status);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + uint32_t(ab * BN) + (uint32_t(32 * q) << 16);
      auto load = [&](int c, float (&v)[32]) { tmem_ld32(tbase + 32 * c, v); };
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_lead + 8u * ab);
      };
      if constexpr (DIRECT)
        rows_direct_epilogue(p, tm * 256 + int(rank) * 128 + 32 * q + lane, tn * BN, cb, ce,
                             tn * 128, alpha, load, release);
      else
        warp_rows_epilogue(p, ebuf, lane, tm * 256 + int(rank) * 128 + 32 * q, tn * BN, cb, ce,
                           tn * 128, alpha, load, release);
    }
  }

  cluster_sync_all();  // the pair is done with both CTAs' memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------- wide CTA-pair kernel --
//
// Normal orientation, tiles of 256 rows x 512 columns per CTA pair: per
// K-step the even CTA issues two tcgen05.mma.cta_group::2 (M = 256, N =
// 256), one per 256-column half of the tile, into the two halves of the
// whole TMEM (512 columns x 128 lanes per CTA).  Per K-block an SM loads 16
// KB of x8 and 2 x 16 KB of weights (48 KB) for 8.4 M MACs, against 32 KB
// for 4.2 M MACs in gemm_pair_kernel: a quarter fewer operand bytes per MAC,
// which is what bounds the pair kernel's main loop (the shared-memory fill).
// The accumulator takes the whole TMEM, so it is single-buffered: the
// epilogue (eight warps, two per TMEM lane quarter, one 256-column half
// each) drains it while the producer keeps filling the 4-stage ring with the
// next tile's operands, and the MMAs of the next tile start once every
// epilogue warp of both CTAs has read its columns.
//   full[s]   (even CTA) 2 arrivals: each CTA's producer arms its bytes
//   empty[s]  (each CTA) released by the even CTA's multicast commit
//   tfull     (each CTA) the accumulator is complete, multicast commit
//   tempty    (even CTA) 16 arrivals: eight epilogue warps per CTA
// Half h of the tile holds weight rows tn*512 + h*256 .. +255 (each CTA the
// 128 rows rank*128 .. of that half), so the column mapping is that of two
// adjacent 256-column tiles.  All waits are bounded; a final cluster barrier
// keeps both CTAs (their shared memory and TMEM) alive until the pair is done.
constexpr int kWideEpiWarps = 8;
constexpr int kWideThreads = 64 + 32 * kWideEpiWarps;

template <int STAGES>
__global__ void __launch_bounds__(kWideThreads, 1)
gemm_pair_wide_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  constexpr int BN = 256;                      // one MMA's N; the tile is 2 x BN
  constexpr int A_BYTES = 128 * BK;
  constexpr int B_HALF = (BN / 2) * BK;        // this CTA's rows of one half
  constexpr int B_BYTES = 2 * B_HALF;
  constexpr uint32_t TMEM_COLS = 512;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* ebuf_base = sB + STAGES * B_BYTES;  // the epilogue warps' row staging
  uint64_t* full = reinterpret_cast<uint64_t*>(ebuf_base + kWideEpiWarps * kEpiStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_ok = abort_flag + 2;  // [kWideEpiWarps]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool lead = rank == 0;
  const int pair = int(blockIdx.x >> 1), npairs = int(gridDim.x >> 1);
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, 2 * kWideEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t full_lead = map_cluster(smem_u32(full), 0);
  const uint32_t tempty_lead = map_cluster(smem_u32(tempty), 0);

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0) {
      const int u0 = pair;
      const int brow = int(rank) * (BN / 2);
      int n_pre = 0;
      if (u0 < p.units) {  // weights first, before the dependency wait
        const int tn = u0 / p.a_tiles;
        n_pre = p.k_blocks < STAGES ? p.k_blocks : STAGES;
        for (int i = 0; i < n_pre; ++i) {
          mbar_arrive_expect_tx_cluster(full_lead + 8u * i, A_BYTES + B_BYTES);
          for (int h = 0; h < 2; ++h)
            tma_load_2d_pair(sB + i * B_BYTES + h * B_HALF, &tmB, full_lead + 8u * i, i * BK,
                             tn * 2 * BN + h * BN + brow);
        }
      }
      pdl_wait();
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = u0; u < p.units && ok; u += npairs) {
        const int tm = u % p.a_tiles, tn = u / p.a_tiles;
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          const bool pre = (u == u0) && (kb < n_pre);
          if (!pre) {
            if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, kWaitNs, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx_cluster(full_lead + 8u * stage, A_BYTES + B_BYTES);
            for (int h = 0; h < 2; ++h)
              tma_load_2d_pair(sB + stage * B_BYTES + h * B_HALF, &tmB, full_lead + 8u * stage,
                               kb * BK, tn * 2 * BN + h * BN + brow);
          }
          tma_load_2d_pair(sA + stage * A_BYTES, &tmA, full_lead + 8u * stage, kb * BK,
                           tm * 256 + int(rank) * 128);
          ++issued;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        record_timeout(p.status);
        *abort_flag = 1;
        if (lead) {  // the even CTA's barriers count both CTAs' copies
          int st = stage;
          uint32_t ph = phase;
          for (int i = 0; i < issued && i < STAGES; ++i) {
            if (--st < 0) { st = STAGES - 1; ph ^= 1u; }
            mbar_wait_bounded(&full[st], ph, kDrainNs, nullptr);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------ MMA issuer (even CTA) --
    if (lane == 0 && lead) {
      constexpr uint32_t idesc = idesc_e4m3_f32(256, BN);
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      int stage = 0, local = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair; u < p.units && ok; u += npairs, ++local) {
        if (!mbar_wait_bounded(tempty, (local & 1) ^ 1u, kWaitNs, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, kWaitNs, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = sdesc_k_sw128(a_base + stage * A_BYTES);
          const uint64_t bd0 = sdesc_k_sw128(b_base + stage * B_BYTES);
          const uint64_t bd1 = sdesc_k_sw128(b_base + stage * B_BYTES + B_HALF);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
            umma_pair_e4m3(tmem_base, ad + 2 * k, bd0 + 2 * k, idesc, acc);
            umma_pair_e4m3(tmem_base + BN, ad + 2 * k, bd1 + 2 * k, idesc, acc);
          }
          umma_pair_commit(&empty[stage], 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_pair_commit(tfull, 0x3);
      }
      if (!ok) {
        record_timeout(p.status);
        *abort_flag = 1;
        umma_pair_commit(drain, 0x1);
        mbar_wait_bounded(drain, 0, kDrainNs, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ----------------------------------------------------------- epilogue --
    pdl_wait();
    const int ew = warp - 2;               // 0 .. 7
    const int q = warp & 3;                // TMEM lane quarter this warp may access
    const int h = ew >> 2;                 // the 256-column half it drains
    uint8_t* ebuf = ebuf_base + ew * kEpiStageBytes;
    const float alpha = __fmul_rn(__ldg(p.act_scale), __ldg(p.w_scale));
    int local = 0;
    for (int u = pair; u < p.units; u += npairs, ++local) {
      const int tm = u % p.a_tiles, tn = u / p.a_tiles;
      const bool got = __all_sync(0xffffffffu,
                                  mbar_wait_bounded(tfull, local & 1, kWaitNs, abort_flag));
      if (lane == 0) epi_ok[ew] = got ? 1 : 0;
      named_bar_sync(1, 32 * kWideEpiWarps);
      bool all_ok = true;
#pragma unroll
      for (int i = 0; i < kWideEpiWarps; ++i) all_ok = all_ok && epi_ok[i];
      named_bar_sync(1, 32 * kWideEpiWarps);
      if (!all_ok) {
        if (lane == 0) record_timeout(p.status);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + uint32_t(h * BN) + (uint32_t(32 * q) << 16);
      auto load = [&](int c, float (&v)[32]) { tmem_ld32(tbase + 32 * c, v); };
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_lead);
      };
      // the half's first output column; with the GEGLU epilogue it holds
      // gate block (tn*2 + h) in columns 0..127 and the matching up block in
      // 128..255 (the gate/up block layout)
      const int n0 = tn * 2 * BN + h * BN;
      warp_rows_epilogue(p, ebuf, lane, tm * 256 + int(rank) * 128 + 32 * q, n0, 0,
                         p.epi == EPI_GEGLU ? 4 : BN / 32, (tn * 2 + h) * 128, alpha, load,
                         release);
    }
  }

  cluster_sync_all();  // the pair is done with both CTAs' memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// --------------------------------------------- CTA-pair kernel, K in halves --
//
// One tile per cluster of 4 CTAs: two CTA pairs (cluster ranks 0-1 and 2-3)
// run the same 256 x BN tile over the two halves of K, each pair as in
// gemm_pair_kernel (cta_group::2 MMAs issued by its even CTA).  When its MMAs
// are done, each CTA of the second pair stages its fp32 accumulator rows in
// its own (now idle) operand ring and bulk-copies them into the ring of the
// CTA holding the same rows in the first pair (rank - 2), which adds them to
// its own accumulator chunk by chunk and runs the tile's epilogue.  For
// shapes whose tiles leave half the SMs idle over a long K (the MLP's down
// projection): twice the SMs pull operands, and the partial sums stay on chip.
//   full[s]   (pair's even CTA) 2 arrivals, both CTAs' TMA bytes
//   empty[s]  (each CTA) the pair's MMA commit, multicast to the pair
//   tfull     (each CTA) the accumulator is complete
//   go        (second pair) the receiving CTA's ring is free
//   red_full  (first pair) the partial rows have landed (transaction bytes)
//   done      (second pair) the receiver has them: the ring may be released
// Every wait is bounded; a final cluster barrier keeps all four CTAs alive
// until the cluster is done.
template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
gemm_pair_split_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, const GemmParams p) {
  constexpr int A_BYTES = 128 * BK;
  constexpr int B_BYTES = (BN / 2) * BK;
  constexpr int RS = BN + 4;                       // staged row stride (floats)
  constexpr uint32_t PART = uint32_t(128 * RS * 4);  // one CTA's staged rows
  static_assert(PART <= uint32_t(STAGES * (A_BYTES + B_BYTES)), "the ring holds the partial");
  constexpr uint32_t TMEM_COLS = tmem_cols_for(BN);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* ebuf_base = sB + STAGES * B_BYTES;  // the epilogue warps' row staging
  uint64_t* full = reinterpret_cast<uint64_t*>(ebuf_base + 4 * kEpiStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* drain = tfull + 1;
  uint64_t* go = drain + 1;
  uint64_t* red_full = drain + 2;
  uint64_t* done = drain + 3;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_ok = abort_flag + 2;  // [4]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int half = int(rank >> 1);          // which half of K this pair runs
  const bool lead = (rank & 1u) == 0;       // the pair's MMA issuer
  const uint32_t lead_rank = rank & ~1u;
  const uint16_t pair_mask = uint16_t(0x3u << (2 * half));
  const int tile = int(blockIdx.x >> 2);
  const bool has_tile = tile < p.units;
  const int tm = tile % p.a_tiles, tn = tile / p.a_tiles;
  const int kb0 = half * p.k_blocks / 2, kb1 = (half + 1) * p.k_blocks / 2;
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    mbar_init(go, 1);
    mbar_init(red_full, 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    if (half == 0) mbar_arrive_expect_tx(red_full, PART);
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // every CTA's barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t full_lead = map_cluster(smem_u32(full), lead_rank);

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    if (lane == 0 && has_tile) {
      const int nk = kb1 - kb0;
      const int n_pre = nk < STAGES ? nk : STAGES;
      for (int i = 0; i < n_pre; ++i) {  // weights first, before the dependency wait
        mbar_arrive_expect_tx_cluster(full_lead + 8u * i, A_BYTES + B_BYTES);
        tma_load_2d_pair(sB + i * B_BYTES, &tmB, full_lead + 8u * i, (kb0 + i) * BK,
                         tn * BN + int(rank & 1u) * (BN / 2));
      }
      pdl_wait();
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int kb = kb0 + i;
        if (i >= n_pre) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, kWaitNs, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx_cluster(full_lead + 8u * stage, A_BYTES + B_BYTES);
          tma_load_2d_pair(sB + stage * B_BYTES, &tmB, full_lead + 8u * stage, kb * BK,
                           tn * BN + int(rank & 1u) * (BN / 2));
        }
        tma_load_2d_pair(sA + stage * A_BYTES, &tmA, full_lead + 8u * stage, kb * BK,
                         tm * 256 + int(rank & 1u) * 128);
        ++issued;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) {
        record_timeout(p.status);
        *abort_flag = 1;
        if (lead) {
          int st = stage;
          uint32_t ph = phase;
          for (int i = 0; i < issued && i < STAGES; ++i) {
            if (--st < 0) { st = STAGES - 1; ph ^= 1u; }
            mbar_wait_bounded(&full[st], ph, kDrainNs, nullptr);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------------- MMA issuer (even CTA) --
    if (lane == 0 && lead && has_tile) {
      constexpr uint32_t idesc = idesc_e4m3_f32(256, BN);
      const uint32_t a_base = smem_u32(sA), b_base = smem_u32(sB);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < kb1 - kb0; ++i) {
        if (!mbar_wait_bounded(&full[stage], phase, kWaitNs, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = sdesc_k_sw128(a_base + stage * A_BYTES);
        const uint64_t bd = sdesc_k_sw128(b_base + stage * B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 32; ++k)
          umma_pair_e4m3(tmem_base, ad + 2 * k, bd + 2 * k, idesc, (i > 0 || k > 0) ? 1u : 0u);
        umma_pair_commit(&empty[stage], pair_mask);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (ok) {
        umma_pair_commit(tfull, pair_mask);
      } else {
        record_timeout(p.status);
        *abort_flag = 1;
        umma_pair_commit(drain, uint16_t(1u << rank));
        mbar_wait_bounded(drain, 0, kDrainNs, nullptr);
      }
    }
    __syncwarp();
  } else if (has_tile) {
    // ----------------------------------------------------------- epilogue --
    pdl_wait();
    const int q = warp & 3;
    const int row = 32 * q + lane;
    uint8_t* ebuf = ebuf_base + (warp - 2) * kEpiStageBytes;
    const float alpha = __fmul_rn(__ldg(p.act_scale), __ldg(p.w_scale));
    const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(tfull, 0, kWaitNs, abort_flag));
    if (lane == 0) epi_ok[q] = got ? 1 : 0;
    named_bar_sync(1, 128);
    const bool all_ok = epi_ok[0] && epi_ok[1] && epi_ok[2] && epi_ok[3];
    tc_fence_after();
    float* part = reinterpret_cast<float*>(smem);  // the idle ring: staged rows
    if (!all_ok) {
      if (threadIdx.x == 64) record_timeout(p.status);
    } else if (half == 1) {
      // hand this CTA's accumulator rows to the CTA with the same rows in
      // the first pair, then wait until it has them
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem_base + 32 * c + (uint32_t(32 * q) << 16), v);
        float4* d4 = reinterpret_cast<float4*>(part + row * RS + 32 * c);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          d4[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (threadIdx.x == 64) {
        if (mbar_wait_bounded_cluster(go, 0, kWaitNs)) {
          bulk_copy_to_peer(map_cluster(smem_u32(smem), rank - 2u), part, PART,
                            map_cluster(smem_u32(red_full), rank - 2u));
          if (!mbar_wait_bounded_cluster(done, 0, kWaitNs)) record_timeout(p.status);
        } else {
          record_timeout(p.status);
        }
      }
      __syncwarp();
    } else {
      // this CTA's MMAs are done: its ring may receive the other half's rows
      // (bare signals: what they order -- the MMAs' reads of the ring, the
      // bulk copy's writes -- is ordered by the barriers those complete on)
      if (threadIdx.x == 64) mbar_arrive_relaxed_cluster(map_cluster(smem_u32(go), rank + 2u));
      const bool in = mbar_wait_bounded_cluster(red_full, 0, kWaitNs);
      if (threadIdx.x == 64) {
        if (in) mbar_arrive_relaxed_cluster(map_cluster(smem_u32(done), rank + 2u));
        else record_timeout(p.status);
      }
      if (in) {
        const float* pr = part + row * RS;
        auto load = [&](int c, float (&v)[32]) {
          tmem_ld32(tmem_base + 32 * c + (uint32_t(32 * q) << 16), v);
          const float4* s4 = reinterpret_cast<const float4*>(pr + 32 * c);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float4 f = s4[k];
            v[4 * k] = __fadd_rn(v[4 * k], f.x);
            v[4 * k + 1] = __fadd_rn(v[4 * k + 1], f.y);
            v[4 * k + 2] = __fadd_rn(v[4 * k + 2], f.z);
            v[4 * k + 3] = __fadd_rn(v[4 * k + 3], f.w);
          }
        };
        warp_rows_epilogue(p, ebuf, lane, tm * 256 + int(rank & 1u) * 128 + 32 * q, tn * BN, 0,
                           p.epi == EPI_GEGLU ? 4 : BN / 32, tn * 128, alpha, load, [] {});
      }
    }
  }

  cluster_sync_all();  // the cluster is done with every CTA's memory
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// -------------------------------------------------------------------- host --

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Row-major [rows, K] e4m3 tensor, box = 128 bytes of K x box_rows rows,
// 128-byte swizzle, out-of-bounds elements read as zero.
int make_map(CUtensorMap* m, const void* ptr, long rows, int K, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FRT_ECUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  const cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(K)};
  const cuuint32_t box[2] = {cuuint32_t(BK), cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FRT_ECUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return FRT_OK;
}

struct Plan {
  bool swap, cluster, pair, split2;
  int bmt, bn, a_tiles, b_tiles, k_blocks, splits, units, grid;
  size_t counters_bytes, ws_bytes;
};

#ifndef FRT_MAX_CLUSTER_SPLITS  // more ranks shorten the main loop but lengthen the gather
#define FRT_MAX_CLUSTER_SPLITS 4
#endif
#ifndef FRT_MIN_KB_PER_CLUSTER_SPLIT
#define FRT_MIN_KB_PER_CLUSTER_SPLIT 2  // K-blocks per split of a cluster tile
#endif

Plan make_plan(int M, int N, int K, int epi) {
  Plan pl{};
  pl.k_blocks = (K + BK - 1) / BK;
  pl.bmt = 128;
  // the e4m3 epilogues write token rows: the normal orientation serves them
  if (epi != EPI_GEGLU && epi != EPI_GELU && M <= 128) {
    pl.swap = true;
    pl.bmt = 64;
    pl.bn = M <= 64 ? 64 : 128;
  }
  else {
    pl.swap = false;
    pl.bn = (N % 256 == 0) ? 256 : 128;
    // narrower tiles before splitting K when 256-wide tiles underfill the SMs
    // (a GEGLU tile keeps its gate and up halves together: always 256 wide)
    const long t256 = ((M + 127L) / 128) * ((N + 255L) / 256);
    if (epi != EPI_GEGLU && pl.bn == 256 && t256 < num_sms()) pl.bn = 128;
    // CTA pairs (256-row tiles, half the B tile per SM): the tile width and
    // the schedule (pairs or single CTAs) with the lowest estimated cost,
    // waves x bytes a CTA moves per K-block (16 KB of x8 plus its weight
    // rows), which is what bounds both the L2-fed main loop and, for short
    // K, the number of rounds of prologue and epilogue
    const int sms = num_sms(), npairs = sms / 2;
    const long tiles1 = ((M + 127L) / 128) * ((N + pl.bn - 1L) / pl.bn);
    const long kb = pl.k_blocks;
    const long cost1 = ((tiles1 + sms - 1) / sms) * (16384L + pl.bn * 128L) * kb;
    const long mt2 = (M + 255L) / 256;
    if (M >= 256) {
      // 512: the wide pair tile (two 256-column MMAs into the whole TMEM)
      static const int kPairBn[] = {512, 256, 192, 160, 128};
      int best = 0;
      bool best_split = false;
      long best_cost = cost1;
      for (int bn2 : kPairBn) {
        if (N % bn2 != 0 || (epi == EPI_GEGLU && bn2 != 256 && bn2 != 512)) continue;
        const long units2 = mt2 * (N / bn2);
        if (units2 < 16) continue;
        // the wide tile's accumulator fills the TMEM, so its epilogue does
        // not overlap the next tile's main loop: measured at about 20
        // K-blocks of main-loop time per tile
        const long kb_eff = bn2 == 512 ? kb + 20 : kb;
        const long cost2 = ((units2 + npairs - 1) / npairs) * (16384L + bn2 * 64L) * kb_eff;
        if (cost2 < best_cost || (epi == EPI_GEGLU && !best)) {
          best = bn2;
          best_cost = cost2;
          best_split = false;
        }
        // K in halves over two pairs per tile (one tile per cluster of 4,
        // one wave), for tiles that leave half the SMs idle over a long K;
        // the on-chip hand-over of the partial costs about 8 K-blocks
        if ((bn2 == 256 || bn2 == 128) && kb >= 32 && units2 * 4 <= sms) {
          const long cost3 = (16384L + bn2 * 64L) * (kb / 2 + 8);
          if (cost3 < best_cost) {
            best = bn2;
            best_cost = cost3;
            best_split = true;
          }
        }
      }
      if (best) {
        const long units2 = mt2 * (N / best);
        pl.pair = true;
        pl.split2 = best_split;
        pl.bn = best;
        pl.a_tiles = int(mt2);
        pl.b_tiles = int(N / best);
        pl.splits = 1;
        pl.units = int(units2);
        pl.grid = best_split ? int(4 * units2) : int(2 * (units2 < npairs ? units2 : npairs));
        return pl;
      }
    }
  }
  const long a_rows = pl.swap ? N : M, b_rows = pl.swap ? M : N;
  pl.a_tiles = int((a_rows + pl.bmt - 1) / pl.bmt);
  pl.b_tiles = int((b_rows + pl.bn - 1) / pl.bn);
  const int tiles = pl.a_tiles * pl.b_tiles;
  const int sms = num_sms();
  pl.splits = 1;
  if (pl.swap) {
    // few weight tiles: split K over a cluster per tile so the weight stream
    // is pulled by (almost) every SM; the cluster reduces on chip
    int s_max = 1;
    if (tiles * 2 <= sms) {
      s_max = sms / tiles;
      const int by_k = pl.k_blocks / FRT_MIN_KB_PER_CLUSTER_SPLIT;
      if (s_max > by_k) s_max = by_k;
      if (s_max > FRT_MAX_CLUSTER_SPLITS) s_max = FRT_MAX_CLUSTER_SPLITS;
      if (s_max < 1) s_max = 1;
    }
    pl.cluster = s_max > 1;
    pl.splits = s_max;
    pl.units = tiles * pl.splits;
    pl.grid = pl.cluster ? pl.units : (tiles < sms ? tiles : sms);
    return pl;
  }
  // split K only when the tiles leave most SMs idle and each split keeps at
  // least FRT_MIN_KB_PER_SPLIT K-blocks of work
  if (tiles * 2 <= sms) {
    int s = sms / tiles;
    const int by_k = pl.k_blocks / FRT_MIN_KB_PER_SPLIT;
    if (s > by_k) s = by_k;
    if (s > 16) s = 16;
    pl.splits = s < 1 ? 1 : s;
  }
  pl.units = tiles * pl.splits;
  pl.grid = pl.units < sms ? pl.units : sms;
  if (pl.splits > 1) {
    pl.counters_bytes = (size_t(tiles) * sizeof(unsigned) + 255) & ~size_t(255);
    pl.ws_bytes = pl.counters_bytes + size_t(tiles) * pl.splits * pl.bmt * pl.bn * sizeof(float);
  }
  return pl;
}

template <bool SWAP, int BMT, int BN, int STAGES, bool CLUSTER>
int prepare_kernel() {
  constexpr int smem = smem_total<SWAP, BMT, BN, STAGES>();
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = gemm_kernel<SWAP, BMT, BN, STAGES, CLUSTER>;
  if (first_use(reinterpret_cast<const void*>(kern))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return fail(FRT_ECUDA, "cudaFuncSetAttribute(max dynamic smem %d)", smem);
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
  }
  return FRT_OK;
}

template <bool SWAP, int BMT, int BN, int STAGES>
int launch_t(const Plan& pl, const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
             cudaStream_t s) {
  constexpr int smem = smem_total<SWAP, BMT, BN, STAGES>();
  int rc = prepare_kernel<SWAP, BMT, BN, STAGES, false>();
  if (rc) return rc;
  return launch_pdl("gemm_kernel", gemm_kernel<SWAP, BMT, BN, STAGES, false>, dim3(pl.grid),
                    dim3(kThreads), size_t(smem), s, ta, tb, p);
}

// Most clusters of `size` CTAs of this kernel the device can hold at once.
template <int BMT, int BN, int STAGES>
int max_active_clusters(int size, int grid) {
  constexpr int smem = smem_total<true, BMT, BN, STAGES>();
  static int cache[64][kMaxCluster + 1];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && cache[dev][size] > 0) return cache[dev][size];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = size;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_kernel<true, BMT, BN, STAGES, true>, &cfg) !=
      cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  if (dev < 64 && n > 0) cache[dev][size] = n;
  return n;
}

// Swapped orientation: a cluster per tile when the plan splits K and the
// device can hold every tile's cluster at once (else fewer splits).
template <int BMT, int BN, int STAGES>
int launch_swap(Plan pl, const CUtensorMap& ta, const CUtensorMap& tb, GemmParams p,
                cudaStream_t s) {
  constexpr int smem = smem_total<true, BMT, BN, STAGES>();
  if (pl.cluster) {
    int rc = prepare_kernel<true, BMT, BN, STAGES, true>();
    if (rc) return rc;
    const int tiles = pl.a_tiles * pl.b_tiles;
    // the leader's operand ring receives the other ranks' staged partials
    constexpr int kMaxRanks = 1 + STAGES * (BMT * BK + BN * BK) / t_tile_bytes<true, BMT, BN>();
    int size = pl.splits < kMaxRanks ? pl.splits : kMaxRanks;
    while (size > 1 && max_active_clusters<BMT, BN, STAGES>(size, tiles * size) < tiles) --size;
    if (size > 1) {
      p.splits = size;
      p.units = tiles * size;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(p.units);
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = s;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = size;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      cudaError_t e =
          cudaLaunchKernelEx(&cfg, gemm_kernel<true, BMT, BN, STAGES, true>, ta, tb, p);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(FRT_ECUDA, "gemm_kernel (cluster %d): %s", size, cudaGetErrorString(e));
      }
      return FRT_OK;
    }
    // no cluster size fits: one CTA per tile, no K split
    p.splits = 1;
    p.units = tiles;
    pl.grid = tiles < num_sms() ? tiles : num_sms();
  }
  return launch_t<true, BMT, BN, STAGES>(pl, ta, tb, p, s);
}

template <int BN, int STAGES>
int launch_pair(const Plan& pl, const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                cudaStream_t s) {
  constexpr int smem =
      STAGES * (128 * BK + (BN / 2) * BK) + kPairEpiWarps * kEpiStageBytes + 1024 + 256;
  static_assert(smem <= 232448, "shared memory budget");
  // At most one tile per pair, on at least half the pairs: the direct
  // (unstaged) epilogue.  Measured on the 18-layer stack's q/k/v GEMM (N 640,
  // 160-wide pair tiles): 64 tiles 10.7 -> 9.3 us direct; 16 tiles 6.2 us
  // staged against 7.2 direct.
  const bool direct = pl.units <= pl.grid / 2 && 4 * pl.units >= num_sms();
  auto kern = direct ? gemm_pair_kernel<BN, STAGES, true> : gemm_pair_kernel<BN, STAGES, false>;
  if (first_use(reinterpret_cast<const void*>(kern))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return fail(FRT_ECUDA, "cudaFuncSetAttribute(max dynamic smem %d)", smem);
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FRT_ECUDA, "gemm_pair_kernel: %s", cudaGetErrorString(e));
  }
  return FRT_OK;
}

template <int STAGES>
int launch_pair_wide(const Plan& pl, const CUtensorMap& ta, const CUtensorMap& tb,
                     const GemmParams& p, cudaStream_t s) {
  constexpr int smem = STAGES * (128 * BK + 256 * BK) + kWideEpiWarps * kEpiStageBytes + 1024 + 256;
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = gemm_pair_wide_kernel<STAGES>;
  if (first_use(reinterpret_cast<const void*>(kern))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return fail(FRT_ECUDA, "cudaFuncSetAttribute(max dynamic smem %d)", smem);
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kWideThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FRT_ECUDA, "gemm_pair_wide_kernel: %s", cudaGetErrorString(e));
  }
  return FRT_OK;
}

template <int BN, int STAGES>
int launch_pair_split(const Plan& pl, const CUtensorMap& ta, const CUtensorMap& tb,
                      const GemmParams& p, cudaStream_t s) {
  constexpr int smem = STAGES * (128 * BK + (BN / 2) * BK) + 4 * kEpiStageBytes + 1024 + 256;
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = gemm_pair_split_kernel<BN, STAGES>;
  if (first_use(reinterpret_cast<const void*>(kern))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return fail(FRT_ECUDA, "cudaFuncSetAttribute(max dynamic smem %d)", smem);
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 4;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FRT_ECUDA, "gemm_pair_split_kernel: %s", cudaGetErrorString(e));
  }
  return FRT_OK;
}

int run_gemm(const Plan& pl, GemmParams& p, const void* x8, const void* w8, void* workspace,
             size_t workspace_bytes, cudaStream_t s) {
  if (pl.ws_bytes > 0) {
    FRT_REQUIRE(workspace, FRT_EINVAL, "this shape splits K: a workspace of %zu bytes is required",
                pl.ws_bytes);
    FRT_REQUIRE(workspace_bytes >= pl.ws_bytes, FRT_ERANGE,
                "workspace of %zu bytes is smaller than the %zu this shape needs", workspace_bytes,
                pl.ws_bytes);
    FRT_REQUIRE(aligned(workspace, 256), FRT_EALIGN, "workspace must be 256-byte aligned");
    p.counters = static_cast<unsigned*>(workspace);
    p.partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + pl.counters_bytes);
  }
  p.a_tiles = pl.a_tiles; p.b_tiles = pl.b_tiles; p.k_blocks = pl.k_blocks;
  p.splits = pl.splits; p.units = pl.units;
  p.status = device_status_ptr();
  CUtensorMap ta, tb;
  int rc;
  if (pl.pair) {  // each CTA loads 128 rows of x8 and BN/2 rows of w8
    if ((rc = make_map(&ta, x8, p.M, p.K, 128))) return rc;
    // weight box: this CTA's half of one MMA's 256 (or bn) columns
    if ((rc = make_map(&tb, w8, p.N, p.K, (pl.bn > 256 ? 256 : pl.bn) / 2))) return rc;
    if (pl.split2) {
      if (pl.bn == 256) return launch_pair_split<256, 6>(pl, ta, tb, p, s);
      return launch_pair_split<128, 8>(pl, ta, tb, p, s);
    }
    if (pl.bn == 512) return launch_pair_wide<4>(pl, ta, tb, p, s);
    if (pl.bn == 256) return launch_pair<256, 6>(pl, ta, tb, p, s);
    if (pl.bn == 192) return launch_pair<192, 6>(pl, ta, tb, p, s);
    if (pl.bn == 160) return launch_pair<160, 7>(pl, ta, tb, p, s);
    return launch_pair<128, 8>(pl, ta, tb, p, s);
  }
  if (!pl.swap) {
    if ((rc = make_map(&ta, x8, p.M, p.K, BM))) return rc;
    if ((rc = make_map(&tb, w8, p.N, p.K, pl.bn))) return rc;
  } else {
    if ((rc = make_map(&ta, w8, p.N, p.K, pl.bmt))) return rc;
    if ((rc = make_map(&tb, x8, p.M, p.K, pl.bn))) return rc;
  }
  if (!pl.swap && pl.bn == 256) return launch_t<false, 128, 256, 4>(pl, ta, tb, p, s);
  if (!pl.swap) return launch_t<false, 128, 128, 6>(pl, ta, tb, p, s);
  if (pl.bn == 64) return launch_swap<64, 64, 12>(pl, ta, tb, p, s);
  return launch_swap<64, 128, 7>(pl, ta, tb, p, s);
}

// The C ABI's epilogue code -> the kernels' epilogue.
int epi_of(int epilogue) {
  return epilogue == FRT_EPI_GEGLU_E4M3   ? EPI_GEGLU
         : epilogue == FRT_EPI_GELU_E4M3 ? EPI_GELU
                                         : EPI_BF16;
}

int validate_common(int M, int N, int K, const void* x8, const void* w8, const float* act_scale,
                    const float* w_scale) {
  FRT_REQUIRE(M >= 0, FRT_ESHAPE, "M must be >= 0, got %d", M);
  FRT_REQUIRE(N > 0 && N % 32 == 0, FRT_ESHAPE, "N must be a positive multiple of 32, got %d", N);
  FRT_REQUIRE(K > 0 && K % 16 == 0, FRT_ESHAPE, "K must be a positive multiple of 16, got %d", K);
  FRT_REQUIRE(x8 && w8 && act_scale && w_scale, FRT_EINVAL,
              "x8, w8, act_scale and w_scale are required");
  FRT_REQUIRE(aligned(x8, 16) && aligned(w8, 16), FRT_EALIGN, "x8 and w8 must be 16-byte aligned");
  return FRT_OK;
}

// Every host-side check of frt_packed_fp8_gemm's arguments (shared with the
// no-allocation entry, which must reject a call before it touches the GPU).
int validate_gemm(int M, int N, int K, const void* x8, const void* w8, const float* act_scale,
                  const float* w_scale, const void* bias, int epilogue, const void* out, long ldo,
                  const float* out_scale) {
  int rc = validate_common(M, N, K, x8, w8, act_scale, w_scale);
  if (rc) return rc;
  FRT_REQUIRE(epilogue == FRT_EPI_BF16 || epilogue == FRT_EPI_GEGLU_E4M3 ||
                  epilogue == FRT_EPI_GELU_E4M3,
              FRT_EINVAL, "unknown epilogue %d", epilogue);
  FRT_REQUIRE(out, FRT_EINVAL, "out is required");
  FRT_REQUIRE(!bias || aligned(bias, 16), FRT_EALIGN, "bias must be 16-byte aligned");
  FRT_REQUIRE(aligned(out, 16), FRT_EALIGN, "out must be 16-byte aligned");
  if (epilogue == FRT_EPI_BF16) {
    FRT_REQUIRE(ldo >= N && ldo % 8 == 0, FRT_EALIGN, "ldo must be >= N and a multiple of 8");
  } else if (epilogue == FRT_EPI_GELU_E4M3) {
    FRT_REQUIRE(out_scale, FRT_EINVAL, "the GELU epilogue needs out_scale");
    FRT_REQUIRE(ldo >= N && ldo % 16 == 0, FRT_EALIGN,
                "ldo must be >= N and a multiple of 16 bytes");
  } else {
    FRT_REQUIRE(N % 256 == 0, FRT_ESHAPE, "the GEGLU epilogue needs N %% 256 == 0, got %d", N);
    FRT_REQUIRE(out_scale, FRT_EINVAL, "the GEGLU epilogue needs out_scale");
    FRT_REQUIRE(ldo >= N / 2 && ldo % 16 == 0, FRT_EALIGN,
                "ldo must be >= N/2 and a multiple of 16 bytes");
  }
  return FRT_OK;
}

}  // namespace
}  // namespace frt

extern "C" size_t frt_gemm_workspace_size(int M, int N, int K, int epilogue) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return frt::make_plan(M, N, K, frt::epi_of(epilogue))
      .ws_bytes;
}

extern "C" int frt_gemm_plan_info(int M, int N, int K, int epilogue, int* info, int n) {
  frt::clear_error();
  FRT_REQUIRE(info && n >= FRT_PLAN_INFO_LEN, FRT_EINVAL,
              "info must hold FRT_PLAN_INFO_LEN (%d) ints", FRT_PLAN_INFO_LEN);
  FRT_REQUIRE(M >= 0 && N > 0 && K > 0, FRT_ESHAPE, "M must be >= 0 and N, K positive");
  FRT_REQUIRE(epilogue >= FRT_EPI_BF16 && epilogue <= FRT_EPI_GELU_E4M3, FRT_EINVAL,
              "unknown epilogue %d", epilogue);
  if (M == 0) {  // nothing is launched
    for (int i = 0; i < FRT_PLAN_INFO_LEN; ++i) info[i] = 0;
    return FRT_OK;
  }
  const frt::Plan pl = frt::make_plan(M, N, K, frt::epi_of(epilogue));
  const int v[FRT_PLAN_INFO_LEN] = {pl.swap,  pl.pair,   pl.split2, pl.cluster, pl.bmt,
                                    pl.bn,    pl.splits, pl.units,  pl.grid,    pl.k_blocks};
  for (int i = 0; i < FRT_PLAN_INFO_LEN; ++i) info[i] = v[i];
  return FRT_OK;
}

extern "C" int frt_packed_fp8_gemm(int M, int N, int K, const frt_e4m3* x8, const frt_e4m3* w8,
                                   const float* act_scale, const float* w_scale,
                                   const frt_bf16* bias, int epilogue, void* out, long ldo,
                                   const float* out_scale, void* workspace,
                                   size_t workspace_bytes, void* stream) {
  frt::clear_error();
  int rc = frt::validate_gemm(M, N, K, x8, w8, act_scale, w_scale, bias, epilogue, out, ldo,
                              out_scale);
  if (rc) return rc;
  if (M == 0) return FRT_OK;
  const int epi = frt::epi_of(epilogue);
  frt::Plan pl = frt::make_plan(M, N, K, epi);
  frt::GemmParams p{};
  p.M = M; p.N = N; p.K = K;
  p.act_scale = act_scale; p.w_scale = w_scale; p.bias = bias;
  p.epi = epi; p.out = out; p.ldo = ldo; p.out_scale = out_scale;
  p.Mseq = 1;
  return frt::run_gemm(pl, p, x8, w8, workspace, workspace_bytes,
                       static_cast<cudaStream_t>(stream));
}

extern "C" int frt_packed_fp8_gemm_rope_kvcache(
    int B, int M, int K, int hq, int hkv, int hd, int P, int T, const frt_e4m3* x8,
    const frt_e4m3* w8, const float* act_scale, const float* w_scale, const frt_bf16* bias,
    const frt_bf16* rope, frt_bf16* q_out, frt_bf16* k_cache, frt_bf16* v_cache, void* workspace,
    size_t workspace_bytes, void* stream) {
  using frt::aligned;
  frt::clear_error();
  FRT_REQUIRE(B >= 0 && M >= 0 && hq >= 0 && hkv >= 1, FRT_ESHAPE, "bad B/M/heads");
  FRT_REQUIRE(hd >= 32 && hd % 32 == 0, FRT_ESHAPE,
              "the fused epilogue needs hd %% 32 == 0, got %d", hd);
  FRT_REQUIRE(P >= 0 && P + M <= T, FRT_ERANGE, "P + M = %d exceeds the cache capacity T = %d",
              P + M, T);
  const int N = (hq + 2 * hkv) * hd;
  const long rows = long(B) * M;
  FRT_REQUIRE(rows <= 0x7fffffffL, FRT_ESHAPE, "B*M too large");
  int rc = frt::validate_common(int(rows), N, K, x8, w8, act_scale, w_scale);
  if (rc) return rc;
  FRT_REQUIRE(rope && k_cache && v_cache && (q_out || hq == 0), FRT_EINVAL,
              "rope, q_out, k_cache and v_cache are required");
  FRT_REQUIRE(!bias || aligned(bias, 16), FRT_EALIGN, "bias must be 16-byte aligned");
  FRT_REQUIRE(aligned(rope, 16) && aligned(k_cache, 16) && aligned(v_cache, 16) &&
                  (!q_out || aligned(q_out, 16)),
              FRT_EALIGN, "rope, q_out and the caches must be 16-byte aligned");
  if (rows == 0) return FRT_OK;
  frt::Plan pl = frt::make_plan(int(rows), N, K, frt::EPI_ROPE);
  frt::GemmParams p{};
  p.M = int(rows); p.N = N; p.K = K;
  p.act_scale = act_scale; p.w_scale = w_scale; p.bias = bias;
  p.epi = frt::EPI_ROPE;
  p.Mseq = M; p.hq = hq; p.hkv = hkv; p.hd = hd; p.P = P; p.T = T;
  p.rope = rope; p.q_out = q_out; p.k_cache = k_cache; p.v_cache = v_cache;
  return frt::run_gemm(pl, p, x8, w8, workspace, workspace_bytes,
                       static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------- no-allocation variant --
//
// Some callers cannot allocate device memory for the split-K workspace:
// plug-ins whose host engine owns every byte of device memory and forbids
// allocation from inside the plug-in, real-time loops that must not enter
// the CUDA allocator (cudaMalloc can synchronise the device), and code that
// runs while a stream is being captured, where a fresh allocation cannot be
// recorded.  frt_packed_fp8_gemm_noalloc serves them with a workspace that
// lives in this file: a static device array of kNoAllocScratchBytes, which
// every GPU that loads the library holds until the process exits.
namespace frt {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  In host code
// the array's name only stands in for the symbol; the address the kernels
// need comes from cudaGetSymbolAddress, looked up on every call (cheap, no
// allocation), so no address outlives the context it belongs to (a device
// reset or a new primary context gives the next call the new address).
int noalloc_scratch(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) {
    cudaGetLastError();
    return fail(FRT_ECUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
  }
  *out = p;
  return FRT_OK;
}

}  // namespace
}  // namespace frt

extern "C" int frt_packed_fp8_gemm_noalloc(int M, int N, int K, const frt_e4m3* x8,
                                           const frt_e4m3* w8, const float* act_scale,
                                           const float* w_scale, const frt_bf16* bias,
                                           int epilogue, void* out, long ldo,
                                           const float* out_scale, void* stream) {
  frt::clear_error();
  // every argument check first: a rejected call must not touch the shared
  // scratch (another call may be using it on the GPU)
  int rc = frt::validate_gemm(M, N, K, x8, w8, act_scale, w_scale, bias, epilogue, out, ldo,
                              out_scale);
  if (rc) return rc;
  if (M == 0) return FRT_OK;
  const frt::Plan pl = frt::make_plan(M, N, K, frt::epi_of(epilogue));
  FRT_REQUIRE(pl.ws_bytes <= frt::kNoAllocScratchBytes, FRT_ERANGE,
              "this shape needs %zu bytes of split-K workspace; the static scratch of "
              "frt_packed_fp8_gemm_noalloc holds %zu (use frt_packed_fp8_gemm with a "
              "caller workspace)",
              pl.ws_bytes, frt::kNoAllocScratchBytes);
  if (pl.ws_bytes == 0)
    return frt_packed_fp8_gemm(M, N, K, x8, w8, act_scale, w_scale, bias, epilogue, out, ldo,
                               out_scale, nullptr, 0, stream);
  void* ws = nullptr;
  rc = frt::noalloc_scratch(&ws);
  if (rc) return rc;
  // the split counters at the head of the workspace must start at zero; a
  // completed call leaves them zero, an interrupted one might not
  if (cudaMemsetAsync(ws, 0, pl.counters_bytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return frt::fail(FRT_ECUDA, "clearing the static scratch counters");
  return frt_packed_fp8_gemm(M, N, K, x8, w8, act_scale, w_scale, bias, epilogue, out, ldo,
                             out_scale, ws, pl.ws_bytes, stream);
}
