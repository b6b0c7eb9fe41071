// style.cu -- the modulation projection on device: one stacked dense
// projection of the conditioning row gives every norm of the stack its
// (scale, shift, gate) rows (impls/adarms_stack/fp8_chain.py `_style_stack`;
// the binder there bakes it once per probed step, this computes it for the
// live conditioning at run time).
//
//   st[r, n] = sum_k cond[r, k] * w[n, k] + bias[n]      (fp32 accumulate)
//   style[r, n] = bf16(st[r, n]);  fin[r, n - fin_col0] = st[r, n]
//
// A matrix-vector product over bf16 weights [N, K] that are read exactly
// once: the kernel is bound by HBM.  A task is 8 output columns: the warp
// splits K over its lanes in 16-byte chunks (one 512-byte row segment per
// warp load), keeps fp32 partial sums in registers and reduces them across
// the warp once.  The grid is persistent (as many CTAs as are resident at
// once), each warp walking a strided list of tasks; its lanes stage their
// chunks through a shared-memory ring with asynchronous copies two steps
// ahead of the multiplies, across task boundaries too, so HBM sees a steady
// stream (12 KB per warp in flight) rather than one burst per wave, at no
// cost in registers.  The weights are bind-time data: the first steps are
// requested before the programmatic dependency wait.

#include "frt_common.cuh"

namespace frt {
namespace {

constexpr int kStyleCols = 8;    // output columns per warp
constexpr int kStyleWarps = 8;   // warps per CTA

struct StyleArgs {
  int rows, K, N, C;  // C = K / 8 chunks of 16 bytes
  const float* cond;
  long ld_cond;
  const uint16_t* w;
  long ldw;
  const float* bias;
  uint16_t* style;
  long ld_style;
  float* fin;
  long ld_fin;
  int fin_col0;
};

// 16-byte asynchronous copy global -> shared, L1 bypassed (read once),
// 256-byte L2 fetches; completion tracked per thread by commit groups.
__device__ __forceinline__ void cp_async16(void* smem, const uint16_t* g) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(d), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// R conditioning rows per CTA row-group (grid.y walks the groups).  A
// persistent grid: warp g of G takes tasks g, g + G, ... (8 columns each);
// a task is ceil(C / 32) steps, lane l handling chunk l + 32 i at step i.
// Each lane copies its own chunks of the task's 8 weight rows into its own
// slots of a DEPTH-step shared-memory ring, DEPTH - 1 steps ahead of the
// step it multiplies (across task boundaries too), and reads back only what
// it copied itself: a commit-group wait per step, no barrier, no spin.
template <int R, int DEPTH>
__global__ void __launch_bounds__(kStyleWarps * 32) style_project_kernel(StyleArgs a) {
  constexpr int CW = kStyleCols;
  extern __shared__ uint4 style_ring[];  // [warps][DEPTH][CW][32]
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint4* ring = style_ring + warp * (DEPTH * CW * 32);
  const long tasks = (long(a.N) + CW - 1) / CW;
  const long G = long(gridDim.x) * kStyleWarps;
  long t = long(blockIdx.x) * kStyleWarps + warp;
  const int spt = (a.C + 31) / 32;  // steps per task, warp-uniform
  const int r0 = blockIdx.y * R;
  const float* cp[R];
#pragma unroll
  for (int r = 0; r < R; ++r) cp[r] = a.cond + long(r0 + r < a.rows ? r0 + r : a.rows - 1) * a.ld_cond;

  // the copies of step (tp, ip) into ring slot `slot`; the last task's rows
  // past N re-read row N - 1 (loads in bounds, sums dropped).  An empty
  // group is committed past the end, so the group count stays in step.
  long tp = t;
  int ip = 0;
  auto issue = [&](int slot) {
    if (tp < tasks) {
      const int c = lane + 32 * ip;
      if (c < a.C) {
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const long n = tp * CW + j < a.N ? tp * CW + j : a.N - 1;
          cp_async16(ring + (slot * CW + j) * 32 + lane, a.w + n * a.ldw + 8 * c);
        }
      }
      if (++ip == spt) {
        ip = 0;
        tp += G;
      }
    }
    cp_async_commit();
  };

  float acc[CW][R];
#pragma unroll
  for (int j = 0; j < CW; ++j)
#pragma unroll
    for (int r = 0; r < R; ++r) acc[j][r] = 0.0f;

#pragma unroll
  for (int s = 0; s < DEPTH - 1; ++s) issue(s);
  pdl_wait();
  int i = 0, slot = 0;
  while (t < tasks) {
    issue(slot == 0 ? DEPTH - 1 : slot - 1);
    cp_async_wait<DEPTH - 1>();  // this lane's copies of the current step landed
    const int c = lane + 32 * i;
    if (c < a.C) {
      float cv[R][8];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float4 lo = __ldg(reinterpret_cast<const float4*>(cp[r] + 8 * c));
        const float4 hi = __ldg(reinterpret_cast<const float4*>(cp[r] + 8 * c) + 1);
        cv[r][0] = lo.x; cv[r][1] = lo.y; cv[r][2] = lo.z; cv[r][3] = lo.w;
        cv[r][4] = hi.x; cv[r][5] = hi.y; cv[r][6] = hi.z; cv[r][7] = hi.w;
      }
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        float wv[8];
        unpack8(ring[(slot * CW + j) * 32 + lane], wv);
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[j][r] = fmaf(cv[r][e], wv[e], acc[j][r]);
      }
    }
    if (++i == spt) {  // the task's last step: reduce across the warp and store
#pragma unroll
      for (int j = 0; j < CW; ++j)
#pragma unroll
        for (int r = 0; r < R; ++r) acc[j][r] = warp_sum(acc[j][r]);
      // every lane holds every sum; lane j * R + r stores column j, row r
#pragma unroll
      for (int j = 0; j < CW; ++j) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const long n = t * CW + j;
          if (lane == j * R + r && n < a.N && r0 + r < a.rows) {
            float v = acc[j][r];
            if (a.bias) v = __fadd_rn(v, __ldg(a.bias + n));
            const long row = r0 + r;
            a.style[row * a.ld_style + n] = f2bf(v);
            if (a.fin && n >= a.fin_col0) a.fin[row * a.ld_fin + (n - a.fin_col0)] = v;
          }
          acc[j][r] = 0.0f;
        }
      }
      i = 0;
      t += G;
    }
    slot = slot + 1 == DEPTH ? 0 : slot + 1;
  }
  cp_async_wait<0>();
}

constexpr int kStyleDepth = 3;
constexpr size_t kStyleSmem = size_t(kStyleWarps) * kStyleDepth * kStyleCols * 32 * 16;

}  // namespace

// Resident CTAs per SM of the R-row kernel (its registers and ring decide),
// per device; the shared-memory limit is raised once per kernel and device.
template <int R>
int style_blocks_per_sm() {
  static int cache[64];
  int dev = 0;
  cudaGetDevice(&dev);
  auto kern = style_project_kernel<R, kStyleDepth>;
  if (first_use(reinterpret_cast<const void*>(kern))) {
    // (this claims the kernel's first use, so the carveout the launch helper
    // sets on first use is set here too)
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kStyleSmem)) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
  }
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kStyleWarps * 32, kStyleSmem) !=
          cudaSuccess ||
      n < 1) {
    cudaGetLastError();
    n = 1;
  }
  if (dev < 64) cache[dev] = n;
  return n;
}

}  // namespace frt

extern "C" int frt_style_project(int rows, int K, int N, const float* cond, long ld_cond,
                                 const frt_bf16* w, long ldw, const float* bias,
                                 frt_bf16* style_out, long ld_style, float* fin_out,
                                 long ld_fin, int fin_col0, void* stream) {
  using frt::aligned;
  frt::clear_error();
  FRT_REQUIRE(rows >= 0 && rows <= 65535, FRT_ESHAPE, "rows must be in [0, 65535], got %d", rows);
  FRT_REQUIRE(K >= 8 && K <= 65536 && K % 8 == 0, FRT_ESHAPE,
              "K must be a multiple of 8 in [8, 65536], got %d", K);
  FRT_REQUIRE(N >= 1, FRT_ESHAPE, "N must be positive, got %d", N);
  FRT_REQUIRE(cond && w && style_out, FRT_EINVAL, "cond, w and style_out are required");
  FRT_REQUIRE(ld_cond >= K && ld_cond % 4 == 0, FRT_EALIGN,
              "ld_cond must be a multiple of 4 that is >= K");
  FRT_REQUIRE(ldw >= K && ldw % 8 == 0, FRT_EALIGN, "ldw must be a multiple of 8 that is >= K");
  FRT_REQUIRE(ld_style >= N, FRT_ESHAPE, "ld_style must be >= N");
  FRT_REQUIRE(aligned(cond, 16) && aligned(w, 16) && aligned(style_out, 2) &&
                  (!bias || aligned(bias, 4)),
              FRT_EALIGN, "cond and w must be 16-byte aligned");
  if (fin_out) {
    FRT_REQUIRE(fin_col0 >= 0 && fin_col0 <= N, FRT_ERANGE, "fin_col0 must be in [0, N]");
    FRT_REQUIRE(ld_fin >= N - fin_col0, FRT_ESHAPE, "ld_fin must be >= N - fin_col0");
    FRT_REQUIRE(aligned(fin_out, 4), FRT_EALIGN, "fin_out must be 4-byte aligned");
  }
  if (rows == 0) return FRT_OK;
  frt::StyleArgs a{rows, K, N, K / 8, cond, ld_cond,
                   reinterpret_cast<const uint16_t*>(w), ldw, bias,
                   reinterpret_cast<uint16_t*>(style_out), ld_style, fin_out, ld_fin,
                   fin_out ? fin_col0 : N};
  const long tasks = (long(N) + frt::kStyleCols - 1) / frt::kStyleCols;
  const long want = (tasks + frt::kStyleWarps - 1) / frt::kStyleWarps;
  const dim3 block(frt::kStyleWarps * 32);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto go = [&](auto kern, int per_sm, unsigned groups) {
    if (per_sm < 1)
      return frt::fail(FRT_ECUDA, "style_project_kernel: cannot raise its shared-memory limit");
    // persistent: as many CTAs as fit on the SMs at once (row groups
    // share them), never more than there are tasks
    const long cap = long(per_sm) * frt::num_sms();
    long gx = groups > 1 ? (cap + groups - 1) / groups : cap;
    gx = gx < 1 ? 1 : (gx < want ? gx : want);
    return frt::launch_pdl("style_project_kernel", kern, dim3(unsigned(gx), groups), block,
                           frt::kStyleSmem, s, a);
  };
  constexpr int D = frt::kStyleDepth;
  if (rows == 1) return go(frt::style_project_kernel<1, D>, frt::style_blocks_per_sm<1>(), 1u);
  if (rows == 2) return go(frt::style_project_kernel<2, D>, frt::style_blocks_per_sm<2>(), 1u);
  return go(frt::style_project_kernel<4, D>, frt::style_blocks_per_sm<4>(),
            unsigned((rows + 3) / 4));
}
