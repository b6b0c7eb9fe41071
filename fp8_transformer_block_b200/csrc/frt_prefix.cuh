// frt_prefix.cuh -- the prefix copy into the chain's caches, as a device
// routine shared by the split kernel and the producer launch that carries it.
//
// flashrt-structures 0.2.0, impls/adarms_stack/fp8_chain.py `_make_run`, the
// `ad:prefix` range: the host cache holds K and V as [B, hkv, T_src, hd]; rows
// p < P go to the chain's caches [B, T, hkv, hd]; keys are gathered through
// kperm (kperm[2i] = i, kperm[2i+1] = hd/2 + i) so the host's rotate-half
// layout lands in the adjacent-pair layout; values are copied as they are.
#pragma once

#include "frt_common.cuh"

namespace frt {

struct PrefixArgs {
  int B, hkv, hd, P, T, T_src, interleave;
  const uint16_t* pk;
  const uint16_t* pv;
  uint16_t* k_cache;
  uint16_t* v_cache;
  long units;  // 2 * B * P * hkv * hd / 8 sixteen-byte units
};

// Unit u (one 8-element chunk of one key or value row): where it lands in
// the chain's cache, and the source data it needs (a key chunk gathers two
// half chunks of the host row).
struct PrefixUnit {
  uint16_t* dst;
  uint2 lo, hi;   // key gather halves, or the value chunk's two halves
  bool gather;
};

__device__ __forceinline__ PrefixUnit prefix_load(const PrefixArgs& a, long u) {
  const int hd8 = a.hd / 8;
  const int which = int(u & 1);
  u >>= 1;
  const int c = int(u % hd8);
  u /= hd8;
  const int h = int(u % a.hkv);
  u /= a.hkv;
  const int p = int(u % a.P);
  const int b = int(u / a.P);
  const long src_row = ((long(b) * a.hkv + h) * a.T_src + p) * a.hd;
  const long dst = ((long(b) * a.T + p) * a.hkv + h) * a.hd + 8 * c;
  PrefixUnit r;
  r.gather = which == 0 && a.interleave;
  r.dst = (which ? a.v_cache : a.k_cache) + dst;
  if (!r.gather) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>((which ? a.pv : a.pk) + src_row + 8 * c));
    r.lo = make_uint2(v.x, v.y);
    r.hi = make_uint2(v.z, v.w);
  } else {
    // destination slots 8c..8c+7 take sources 4c..4c+3 (even slots) and
    // hd/2 + 4c .. +3 (odd slots)
    r.lo = __ldg(reinterpret_cast<const uint2*>(a.pk + src_row + 4 * c));
    r.hi = __ldg(reinterpret_cast<const uint2*>(a.pk + src_row + a.hd / 2 + 4 * c));
  }
  return r;
}

__device__ __forceinline__ void prefix_store(const PrefixUnit& r) {
  if (!r.gather) {
    *reinterpret_cast<uint4*>(r.dst) = make_uint4(r.lo.x, r.lo.y, r.hi.x, r.hi.y);
    return;
  }
  const uint32_t l[2] = {r.lo.x, r.lo.y}, m[2] = {r.hi.x, r.hi.y};
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    o[2 * k] = (l[k] & 0xFFFFu) | (m[k] << 16);
    o[2 * k + 1] = (l[k] >> 16) | (m[k] & 0xFFFF0000u);
  }
  *reinterpret_cast<uint4*>(r.dst) = make_uint4(o[0], o[1], o[2], o[3]);
}

// Copy unit u.
__device__ __forceinline__ void prefix_unit(const PrefixArgs& a, long u) {
  prefix_store(prefix_load(a, u));
}

// Copy units first, first + stride, ... (< a.units): every load of up to
// kPrefixBatch units is issued before the first store, so a thread with
// several units pays one memory round trip per batch, not one per unit.
constexpr int kPrefixBatch = 8;
__device__ __forceinline__ void prefix_units_strided(const PrefixArgs& a, long first, long stride) {
  for (long u0 = first; u0 < a.units; u0 += stride * kPrefixBatch) {
    PrefixUnit r[kPrefixBatch];
#pragma unroll
    for (int i = 0; i < kPrefixBatch; ++i)
      if (u0 + i * stride < a.units) r[i] = prefix_load(a, u0 + i * stride);
#pragma unroll
    for (int i = 0; i < kPrefixBatch; ++i)
      if (u0 + i * stride < a.units) prefix_store(r[i]);
  }
}

}  // namespace frt
