// rope.cu -- a3 / a4: the rotary table, the split + adjacent-pair RoPE + KV
// write, and the prefix copy into the chain's caches.
//
// flashrt-structures 0.2.0, impls/adarms_stack/fp8_chain.py: `_build_rope`
// (bf16 table with cos in even and sin in odd slots, taken from the first,
// half-duplicated half of the host's rotary output), `_make_run` (the split
// kernel writes q_out and the suffix K/V rows P.. of the layer's caches; the
// `ad:prefix` range gathers the host's prefix keys through `kperm` and copies
// the values) and `_alloc` (q [1,S,nh,hd], caches [1,T,kv,hd]).
//
// All three are HBM-bound streams: 16-byte loads and stores, one 8-element
// chunk per thread step, grid-stride loops sized to the SM count.
#include "frt_internal.cuh"

namespace frt {
namespace {

__global__ void rope_table_kernel(int M, int hd, int P, double theta, uint16_t* out) {
  const int half = hd / 2;
  const long total = long(M) * half;
  for (long g = blockIdx.x * long(blockDim.x) + threadIdx.x; g < total;
       g += long(gridDim.x) * blockDim.x) {
    const int s = int(g / half), i = int(g % half);
    const double inv_freq = pow(theta, -double(2 * i) / double(hd));
    const double ang = double(P + s) * inv_freq;
    double sn, cs;
    sincos(ang, &sn, &cs);
    out[long(s) * hd + 2 * i] = __bfloat16_as_ushort(__double2bfloat16(cs));
    out[long(s) * hd + 2 * i + 1] = __bfloat16_as_ushort(__double2bfloat16(sn));
  }
}

struct SplitArgs {
  int B, M, hq, hkv, hd, P, T;
  const uint16_t* qkv;
  const uint16_t* rope;
  uint16_t* q_out;
  uint16_t* k_cache;
  uint16_t* v_cache;
  long suffix_units;
  PrefixArgs pre;  // pre.units == 0: no prefix copy
};

// Rotate 4 adjacent pairs of x (8 bf16) with 4 (cos, sin) pairs of r.
__device__ __forceinline__ uint4 rotate8(const uint4& xv, const uint4& rv) {
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

__global__ void split_rope_kernel(SplitArgs a) {
  const int hd8 = a.hd / 8;
  const int heads = a.hq + 2 * a.hkv;
  const long N8 = long(heads) * hd8;
  const long total = a.suffix_units + a.pre.units;
  pdl_trigger();
  pdl_wait();
  for (long g = blockIdx.x * long(blockDim.x) + threadIdx.x; g < total;
       g += long(gridDim.x) * blockDim.x) {
    if (g < a.suffix_units) {
      const long r = g / N8;
      const int c8 = int(g % N8);
      const int b = int(r / a.M), s = int(r % a.M);
      const int h = c8 / hd8, d0 = (c8 % hd8) * 8;
      const uint4 xv = __ldg(reinterpret_cast<const uint4*>(a.qkv + r * N8 * 8 + long(c8) * 8));
      if (h < a.hq + a.hkv) {
        const uint4 rv = __ldg(reinterpret_cast<const uint4*>(a.rope + long(s) * a.hd + d0));
        const uint4 o = rotate8(xv, rv);
        uint16_t* dst = h < a.hq
            ? a.q_out + ((long(b) * a.M + s) * a.hq + h) * a.hd + d0
            : a.k_cache + ((long(b) * a.T + a.P + s) * a.hkv + (h - a.hq)) * a.hd + d0;
        *reinterpret_cast<uint4*>(dst) = o;
      } else {
        const int hv = h - a.hq - a.hkv;
        *reinterpret_cast<uint4*>(a.v_cache + ((long(b) * a.T + a.P + s) * a.hkv + hv) * a.hd + d0) = xv;
      }
    } else {
      prefix_unit(a.pre, g - a.suffix_units);
    }
  }
}

int launch_split(const SplitArgs& a, cudaStream_t s) {
  const long total = a.suffix_units + a.pre.units;
  if (total == 0) return FRT_OK;
  const long blocks_needed = (total + 255) / 256;
  const int grid = int(blocks_needed < num_sms() * 16L ? blocks_needed : num_sms() * 16L);
  return launch_pdl("split_rope_kernel", split_rope_kernel, dim3(grid), dim3(256), 0, s, a);
}

}  // namespace
}  // namespace frt

extern "C" int frt_build_rope_table(int M, int hd, int P, double theta, frt_bf16* rope_out,
                                    void* stream) {
  frt::clear_error();
  FRT_REQUIRE(M >= 0 && P >= 0, FRT_ESHAPE, "M and P must be >= 0");
  FRT_REQUIRE(hd >= 2 && hd % 2 == 0, FRT_ESHAPE, "hd must be even, got %d", hd);
  FRT_REQUIRE(theta > 0.0, FRT_EINVAL, "theta must be > 0");
  FRT_REQUIRE(rope_out, FRT_EINVAL, "rope_out is required");
  if (M == 0) return FRT_OK;
  const long total = long(M) * (hd / 2);
  const int grid = int((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
  frt::rope_table_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(M, hd, P, theta,
                                                                              rope_out);
  return frt::check_launch("frt_build_rope_table");
}

namespace frt {

int prefix_args(int B, int hkv, int hd, int P, int T, int T_src, const uint16_t* pk,
                const uint16_t* pv, int interleave, uint16_t* k_cache, uint16_t* v_cache,
                PrefixArgs* a) {
  FRT_REQUIRE(B >= 0 && hkv >= 1, FRT_ESHAPE, "bad B/hkv");
  FRT_REQUIRE(hd >= 8 && hd % 8 == 0, FRT_ESHAPE, "hd must be a multiple of 8, got %d", hd);
  FRT_REQUIRE(pk && pv, FRT_EINVAL, "prefix_k and prefix_v are both required");
  FRT_REQUIRE(k_cache && v_cache, FRT_EINVAL, "k_cache and v_cache are required");
  FRT_REQUIRE(P >= 0 && P <= T && P <= T_src, FRT_ERANGE,
              "prefix rows P=%d must fit the cache (T=%d) and the source (T_src=%d)", P, T, T_src);
  FRT_REQUIRE(aligned(pk, 16) && aligned(pv, 16) && aligned(k_cache, 16) && aligned(v_cache, 16),
              FRT_EALIGN, "prefix tensors and caches must be 16-byte aligned");
  a->B = B; a->hkv = hkv; a->hd = hd; a->P = P; a->T = T; a->T_src = T_src;
  a->interleave = interleave != 0;
  a->pk = pk; a->pv = pv; a->k_cache = k_cache; a->v_cache = v_cache;
  a->units = 2L * B * P * hkv * (hd / 8);
  return FRT_OK;
}

}  // namespace frt

extern "C" int frt_split_rope_kvcache(int B, int M, int hq, int hkv, int hd, int P, int T,
                                      const frt_bf16* qkv, const frt_bf16* rope, frt_bf16* q_out,
                                      frt_bf16* k_cache, frt_bf16* v_cache,
                                      const frt_bf16* prefix_k, const frt_bf16* prefix_v,
                                      int prefix_T_src, int prefix_interleave, void* stream) {
  using frt::aligned;
  frt::clear_error();
  FRT_REQUIRE(B >= 0 && M >= 0 && hq >= 0 && hkv >= 1, FRT_ESHAPE, "bad B/M/heads");
  FRT_REQUIRE(hd >= 8 && hd % 8 == 0, FRT_ESHAPE, "hd must be a multiple of 8, got %d", hd);
  FRT_REQUIRE(P >= 0 && P + M <= T, FRT_ERANGE, "P + M = %d exceeds the cache capacity T = %d",
              P + M, T);
  FRT_REQUIRE(k_cache && v_cache, FRT_EINVAL, "k_cache and v_cache are required");
  FRT_REQUIRE(aligned(k_cache, 16) && aligned(v_cache, 16), FRT_EALIGN, "caches must be 16-byte aligned");
  if (M > 0 && B > 0) {
    FRT_REQUIRE(qkv && rope && (q_out || hq == 0), FRT_EINVAL, "qkv, rope and q_out are required");
    FRT_REQUIRE(aligned(qkv, 16) && aligned(rope, 16) && (!q_out || aligned(q_out, 16)),
                FRT_EALIGN, "qkv, rope and q_out must be 16-byte aligned");
  }
  frt::SplitArgs a{};
  a.B = B; a.M = M; a.hq = hq; a.hkv = hkv; a.hd = hd; a.P = P; a.T = T;
  a.qkv = qkv; a.rope = rope; a.q_out = q_out; a.k_cache = k_cache; a.v_cache = v_cache;
  a.suffix_units = long(B) * M * (hq + 2 * hkv) * (hd / 8);
  if (prefix_k) {
    int rc = frt::prefix_args(B, hkv, hd, P, T, prefix_T_src, prefix_k, prefix_v,
                              prefix_interleave, k_cache, v_cache, &a.pre);
    if (rc) return rc;
  }
  return frt::launch_split(a, static_cast<cudaStream_t>(stream));
}

extern "C" int frt_prefix_copy_kv(int B, int hkv, int hd, int P, int T, int T_src,
                                  const frt_bf16* prefix_k, const frt_bf16* prefix_v, int interleave,
                                  frt_bf16* k_cache, frt_bf16* v_cache, void* stream) {
  frt::clear_error();
  frt::SplitArgs a{};
  int rc = frt::prefix_args(B, hkv, hd, P, T, T_src, prefix_k, prefix_v, interleave, k_cache,
                            v_cache, &a.pre);
  if (rc) return rc;
  a.hkv = hkv; a.hd = hd;
  return frt::launch_split(a, static_cast<cudaStream_t>(stream));
}
