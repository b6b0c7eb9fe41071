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
// All three are HBM-bound streams of 16-byte loads and stores: the split
// kernel one block per token and column slice with every load of a thread
// issued before its first store, the prefix copy a grid-stride loop sized to
// the SM count.
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
};

// Units (16 bytes: 8 columns of one row's q, k or v) per thread per step of
// the split kernel: their loads are all issued before the first store.
constexpr int kSplitUnroll = 4;
constexpr int kSplitThreads = 128;

// Split + RoPE + KV write.  Block (x, s, b) takes token s of batch b (no
// index division for the row) and units x*T*U + t + T*k (k < U) of its
// N/8: the row's q/k/v pieces and their rope-table pieces are requested
// first, then rotated and stored.
__global__ void __launch_bounds__(kSplitThreads)
split_rope_kernel(SplitArgs a) {
  const int s = int(blockIdx.y), b = int(blockIdx.z);
  const int hd8 = a.hd / 8;
  const int N8 = (a.hq + 2 * a.hkv) * hd8;
  const long r = long(b) * a.M + s;
  const uint16_t* src = a.qkv + r * N8 * 8;
  const uint16_t* rrow = a.rope + long(s) * a.hd;
  const long krow = (long(b) * a.T + a.P + s) * a.hkv;   // cache row (in heads)
  const long qrow = r * a.hq;                            // q_out row (in heads)
  pdl_trigger();
  pdl_wait();
  const int c_base = int(blockIdx.x) * kSplitThreads * kSplitUnroll + int(threadIdx.x);
  uint4 xv[kSplitUnroll], rv[kSplitUnroll];
#pragma unroll
  for (int k = 0; k < kSplitUnroll; ++k) {
    const int c8 = c_base + k * kSplitThreads;
    if (c8 < N8) {
      const int h = c8 / hd8, d0 = (c8 - h * hd8) * 8;
      xv[k] = __ldg(reinterpret_cast<const uint4*>(src + c8 * 8));
      if (h < a.hq + a.hkv) rv[k] = __ldg(reinterpret_cast<const uint4*>(rrow + d0));
    }
  }
#pragma unroll
  for (int k = 0; k < kSplitUnroll; ++k) {
    const int c8 = c_base + k * kSplitThreads;
    if (c8 < N8) {
      const int h = c8 / hd8, d0 = (c8 - h * hd8) * 8;
      uint16_t* dst;
      uint4 o = xv[k];
      if (h < a.hq) {
        dst = a.q_out + (qrow + h) * a.hd + d0;
        o = rope_rotate8(o, rv[k]);
      } else if (h < a.hq + a.hkv) {
        dst = a.k_cache + (krow + (h - a.hq)) * a.hd + d0;
        o = rope_rotate8(o, rv[k]);
      } else {
        dst = a.v_cache + (krow + (h - a.hq - a.hkv)) * a.hd + d0;
      }
      *reinterpret_cast<uint4*>(dst) = o;
    }
  }
}

int launch_split(const SplitArgs& a, cudaStream_t s) {
  if (long(a.B) * a.M == 0) return FRT_OK;
  const int N8 = (a.hq + 2 * a.hkv) * (a.hd / 8);
  const int gx = (N8 + kSplitThreads * kSplitUnroll - 1) / (kSplitThreads * kSplitUnroll);
  return launch_pdl("split_rope_kernel", split_rope_kernel, dim3(gx, a.M, a.B),
                    dim3(kSplitThreads), 0, s, a);
}

// The prefix copy alone: 16-byte units over a grid sized to the SM count,
// each thread's loads issued before its stores.
__global__ void prefix_copy_kernel(PrefixArgs a) {
  pdl_trigger();
  pdl_wait();
  prefix_units_strided(a, blockIdx.x * long(blockDim.x) + threadIdx.x, long(gridDim.x) * blockDim.x);
}

int launch_prefix(const PrefixArgs& a, cudaStream_t s) {
  if (a.units == 0) return FRT_OK;
  const long blocks_needed = (a.units + 255) / 256;
  const int grid = int(blocks_needed < num_sms() * 8L ? blocks_needed : num_sms() * 8L);
  return launch_pdl("prefix_copy_kernel", prefix_copy_kernel, dim3(grid), dim3(256), 0, s, a);
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
  FRT_REQUIRE(M <= 65535 && B <= 65535, FRT_ESHAPE,
              "the split kernel takes at most 65535 tokens and batches, got M=%d B=%d", M, B);
  frt::SplitArgs a{};
  a.B = B; a.M = M; a.hq = hq; a.hkv = hkv; a.hd = hd; a.P = P; a.T = T;
  a.qkv = qkv; a.rope = rope; a.q_out = q_out; a.k_cache = k_cache; a.v_cache = v_cache;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (prefix_k) {
    frt::PrefixArgs pre{};
    int rc = frt::prefix_args(B, hkv, hd, P, T, prefix_T_src, prefix_k, prefix_v,
                              prefix_interleave, k_cache, v_cache, &pre);
    if (rc) return rc;
    rc = frt::launch_prefix(pre, st);
    if (rc) return rc;
  }
  return frt::launch_split(a, st);
}

extern "C" int frt_prefix_copy_kv(int B, int hkv, int hd, int P, int T, int T_src,
                                  const frt_bf16* prefix_k, const frt_bf16* prefix_v, int interleave,
                                  frt_bf16* k_cache, frt_bf16* v_cache, void* stream) {
  frt::clear_error();
  frt::PrefixArgs pre{};
  int rc = frt::prefix_args(B, hkv, hd, P, T, T_src, prefix_k, prefix_v, interleave, k_cache,
                            v_cache, &pre);
  if (rc) return rc;
  return frt::launch_prefix(pre, static_cast<cudaStream_t>(stream));
}
