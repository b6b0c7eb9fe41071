/*
 * frt.h -- C ABI of libfrt, the sm_100a (B200) fused static-FP8
 * attention-input chain.
 *
 * The chain (flashrt-structures 0.2.0, impls/adarms_stack/fp8_chain.py,
 * module docstring and `_make_run`; impls/modnorm_qkv_chain/fp8_ptok_table.py,
 * `PerTokenModChainBlock.forward`):
 *   1. producer: gated residual add + adaptive RMS or LayerNorm with
 *      shift/scale(/gate) modulation + static-scale e4m3 quantize, one pass;
 *   2. one FP8 GEMM over sibling weights packed into one [sum N_i, K] matrix
 *      with one joint per-tensor scale (impls/qkv_pack/fp8_static.py,
 *      module docstring and `_pack_weights`), plus bias;
 *   3. split + adjacent-pair RoPE + KV-cache write behind a copied prefix.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers unless marked "host".  The caller
 *     owns all memory; the library allocates nothing.  Tensors are dense,
 *     row-major, with the shapes given.  bf16 tensors are passed as
 *     frt_bf16 (the 16-bit pattern), e4m3fn tensors as frt_e4m3 (the code).
 *   - Scales (act_scale, w_scale, out_scale) are device fp32 [1] tensors,
 *     never host floats, so calls can be captured into CUDA graphs.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work
 *     is enqueued asynchronously; nothing synchronises with the host.
 *   - Arguments are validated on the host before any launch.  A rejected
 *     call launches nothing and returns a negative FRT_E* code; the reason
 *     is available from frt_last_error() on the calling thread.  FRT_ECUDA
 *     reports a CUDA error seen at launch.
 *   - Device-side waits (mbarrier pipelines) are bounded in time.  A wait
 *     that runs out records FRT_ETIMEOUT in the library's device status
 *     word, makes the kernel drain and return, and frt_device_status()
 *     reports it later.
 */
#ifndef FRT_H_
#define FRT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t frt_bf16; /* bfloat16 bit pattern */
typedef uint8_t frt_e4m3;  /* float8 e4m3fn code   */

enum {
  FRT_OK = 0,
  FRT_EINVAL = -1,   /* null pointer, bad enum, bad scalar                 */
  FRT_ESHAPE = -2,   /* dimension outside what the kernel supports         */
  FRT_EALIGN = -3,   /* pointer or stride not aligned as required          */
  FRT_ERANGE = -4,   /* P + M > T, workspace too small, row capacity       */
  FRT_ECUDA = -5,    /* CUDA reported an error at launch                   */
  FRT_ETIMEOUT = -6  /* a bounded device-side wait ran out                 */
};

/* Reason for the last failing call on this thread ("" if none). */
const char* frt_last_error(void);

/* ABI version of this header (major * 100 + minor). */
int frt_version(void);

/* Read (and with reset != 0, clear) the device status word of the current
 * device.  Synchronises `stream` first.  Returns FRT_OK, FRT_ETIMEOUT (some
 * bounded wait ran out since the last reset) or FRT_ECUDA. */
int frt_device_status(int reset, void* stream);

/* ----------------------------------------------------------------------- */
/* a1 / a1'  Producer.                                                      */
/* ----------------------------------------------------------------------- */
enum { FRT_NORM_ADARMS = 0, FRT_NORM_LAYERNORM_TABLE = 1 };

/*
 * frt_ada_norm_quant_fp8 -- one pass over `rows` rows of width D.
 *
 * mode FRT_NORM_ADARMS (fp8_chain.py, `norm_project` -> the norm kernel's
 * call, and the fp32 tail of `_make_run`, which fixes the formula):
 *   h = res + prev_gate * delta;  res <- bf16(h)            (in place)
 *   y = bf16(h) / sqrt(mean(bf16(h)^2) + eps) * w * (1 + scale) + shift
 *   x8 = e4m3(clamp(y / act_scale, +-448));  gate_out = gate
 *   res, delta: [rows, D].  prev_gate: [1 or rows, D], row stride
 *   gate_row_stride elements (0 = one row broadcast).  weight: [D] or NULL
 *   (= ones).  style: [1 or rows, 3D] = (scale, shift, gate) chunks, row
 *   stride style_row_stride (0 = broadcast).  gate_out: [rows, D] or NULL.
 *   x, temb, table, chunks, shift_idx, scale_idx are ignored.
 *
 * mode FRT_NORM_LAYERNORM_TABLE (fp8_ptok_table.py, module docstring and
 * `PerTokenModChainBlock.forward`: table add + chunk selection + no-affine
 * LayerNorm + modulation + static quantize):
 *   shift = table[shift_idx] + temb[r, shift_idx];  scale likewise
 *   y = (x - mean(x)) / sqrt(var(x) + eps) * (1 + scale) + shift  (biased var)
 *   x: [rows, D]; temb: [rows, chunks, D] bf16; table: [chunks, D] fp32.
 *   res, delta, prev_gate, weight, style, gate_out are ignored.
 *
 * act_scale: device fp32 [1].  x8_out: [rows, D] e4m3.  amax_out: NULL or a
 * device fp32 [1] the caller zeroed; the kernel raises it to max |y| (the
 * static calibration of fp8_chain.py `bind_adarms_fp8_chain`).
 * Requires 8 <= D <= 16384, D % 8 == 0, 16-byte aligned bf16 pointers and
 * row strides that are multiples of 8, x8_out 8-byte aligned.  rows == 0 is
 * a no-op.  All arithmetic fp32; the row statistics use IEEE-rounded
 * division and square root; the quantizer multiplies y by the fp32
 * reciprocal of act_scale.
 */
int frt_ada_norm_quant_fp8(int mode, int rows, int D, float eps,
                           frt_bf16* res, const frt_bf16* delta,
                           const frt_bf16* prev_gate, long gate_row_stride,
                           const frt_bf16* weight, const frt_bf16* style,
                           long style_row_stride, const frt_bf16* x,
                           const frt_bf16* temb, int chunks,
                           const float* table, int shift_idx, int scale_idx,
                           const float* act_scale, frt_e4m3* x8_out,
                           frt_bf16* gate_out, float* amax_out, void* stream);

/* ----------------------------------------------------------------------- */
/* a0  Joint per-tensor weight pack (bind time).                            */
/* ----------------------------------------------------------------------- */
enum {
  FRT_PACK_CONCAT = 0,     /* rows in sibling order (torch.cat along N)    */
  FRT_PACK_QK_INTERLEAVE = 1, /* siblings (q, k, v): in each q and k head,
                                 row i -> 2i, row hd/2+i -> 2i+1; v as is   */
  FRT_PACK_GATE_UP_BLOCKS = 2 /* siblings (gate, up), equal n, n % 128 == 0:
                                 128-row gate block then the matching up
                                 block, repeated (for the fused GEGLU)      */
};

/*
 * frt_pack_weights_fp8 (qkv_pack/fp8_static.py `_pack_weights`;
 * fp8_chain.py `_quantize` with `_interleave_rows`):
 *   w_scale = max(amax(|w_all|) / 448, 1e-8);  w8 = e4m3(clamp(w / w_scale))
 * w: HOST array of n_siblings DEVICE pointers, sibling i is [n_rows[i], K]
 * bf16 (n_rows is a HOST array).  bias: NULL or a HOST array of device
 * pointers, entries NULL for siblings without bias (zeros are packed).
 * w8_out: [N, K] e4m3, N = sum n_rows.  w_scale_out: device fp32 [1].
 * bias_out: [N] bf16 or NULL.  layout: FRT_PACK_*; hd is the head size for
 * FRT_PACK_QK_INTERLEAVE.  1 <= n_siblings <= 4, K % 16 == 0.
 * Bit-exact: true fp32 division, round to nearest even.
 */
int frt_pack_weights_fp8(int n_siblings, const frt_bf16* const* w,
                         const int* n_rows, int K, const frt_bf16* const* bias,
                         int layout, int hd, frt_e4m3* w8_out,
                         float* w_scale_out, frt_bf16* bias_out, void* stream);

/* ----------------------------------------------------------------------- */
/* a2 (+ a5)  Packed FP8 GEMM on tcgen05 tensor cores.                      */
/* ----------------------------------------------------------------------- */
enum { FRT_EPI_BF16 = 0, FRT_EPI_GEGLU_E4M3 = 1, FRT_EPI_GELU_E4M3 = 2 };

/*
 * Bytes of workspace frt_packed_fp8_gemm / _rope_kvcache need for this
 * shape (0 if the chosen schedule does not split K).  The workspace must be
 * zero-filled once before its first use; every completed call leaves its
 * counters at zero again.  Calls that share a workspace must not overlap.
 */
size_t frt_gemm_workspace_size(int M, int N, int K, int epilogue);

/*
 * The schedule frt_packed_fp8_gemm (and the rope/KV form, which plans like
 * FRT_EPI_BF16) picks for this shape on the current device (148 SMs when no
 * device is visible), host-side only, for tests and tuning.  info[0 ..
 * FRT_PLAN_INFO_LEN - 1] receives: swapped orientation (weights on the MMA M
 * side), CTA pairs, K in halves over two pairs, K split in a cluster, the
 * weight (swapped) or activation tile rows, the other tile side, K splits,
 * work units, grid CTAs, 128-byte K-blocks.  A cluster launch may still use
 * fewer splits when the device cannot hold every tile's cluster at once.
 * M == 0 (nothing launched) gives all zeros.  FRT_EINVAL for a short or NULL info or an unknown epilogue, FRT_ESHAPE
 * for M < 0, N <= 0 or K <= 0.
 */
enum { FRT_PLAN_INFO_LEN = 10 };
int frt_gemm_plan_info(int M, int N, int K, int epilogue, int* info, int n);

/*
 * frt_packed_fp8_gemm (qkv_pack/fp8_static.py `PackedLinear._run`;
 * fp8_chain.py `norm_project` / `down_project`):
 *   acc[m, n] = sum_k x8[m, k] * w8[n, k]            (fp32 accumulate)
 *   FRT_EPI_BF16:  out[m, n] = bf16(acc * (act_scale * w_scale) + bias[n])
 *                  out: [M, ldo] bf16, ldo >= N.
 *   FRT_EPI_GEGLU_E4M3 (fp8_chain.py `down_project`, the merged GEGLU +
 *   requant kernel): w8 packed with FRT_PACK_GATE_UP_BLOCKS; with
 *   g, u = bf16(acc * alpha + bias) of matching gate/up columns,
 *                  out[m, j] = e4m3(gelu_tanh(g) * u * (1 / out_scale))
 *                  out: [M, ldo] e4m3, ldo >= N / 2; N % 256 == 0.
 *   FRT_EPI_GELU_E4M3 (fp8_ptok_table.py, the DiT FFN's fp8_gelu_mlp
 *   middle step): with y = bf16(acc * alpha + bias),
 *                  out[m, n] = e4m3(gelu_tanh(y) * (1 / out_scale))
 *                  out: [M, ldo] e4m3, ldo >= N.
 * x8: [M, K] e4m3; w8: [N, K] e4m3; bias: [N] bf16 or NULL.
 * Requires K % 16 == 0, N % 32 == 0, 16-byte aligned x8/w8/out/bias, ldo %
 * 16 == 0 (bytes of a row).  M == 0 is a no-op.  workspace: see
 * frt_gemm_workspace_size (may be NULL when that is 0).
 * The kernel starts loading w8 while the kernel before it on the stream
 * finishes (programmatic dependent launch): w8 must not be written by the
 * immediately preceding kernel on the stream (frt_pack_weights_fp8 ends with
 * a fence launch, so weights it packed are always safe).
 */
int frt_packed_fp8_gemm(int M, int N, int K, const frt_e4m3* x8,
                        const frt_e4m3* w8, const float* act_scale,
                        const float* w_scale, const frt_bf16* bias,
                        int epilogue, void* out, long ldo,
                        const float* out_scale, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * frt_packed_fp8_gemm_noalloc -- frt_packed_fp8_gemm for callers that cannot
 * allocate device memory (a plug-in whose host engine owns all device
 * memory, a real-time loop that must not enter the CUDA allocator, code
 * running while a stream is captured).  The pages have no counterpart; this
 * is a convenience of this library.  Same arguments and results as
 * frt_packed_fp8_gemm without the workspace: shapes whose split-K schedule
 * needs a workspace use a static device array of 8 MiB that the library
 * holds on every GPU that loads it, until the process exits.  Shapes that
 * need more are rejected with FRT_ERANGE (nothing is launched).  The call
 * allocates nothing.  Every argument is checked on the host first, exactly
 * as frt_packed_fp8_gemm checks them; a rejected call returns its code
 * without enqueueing anything.  Each call looks up the array's device
 * address in the current context (cudaGetSymbolAddress: no allocation, no
 * launch), so a call after cudaDeviceReset finds the array of the new
 * context; make the first call on a device outside any stream capture (it
 * may load the library's device code).  Every call shares
 * the one array and zeroes its split counters first (a stream-ordered
 * memset): calls that may overlap on the GPU (other streams, other
 * threads) race on it and must be serialised by the caller.
 */
int frt_packed_fp8_gemm_noalloc(int M, int N, int K, const frt_e4m3* x8,
                                const frt_e4m3* w8, const float* act_scale,
                                const float* w_scale, const frt_bf16* bias,
                                int epilogue, void* out, long ldo,
                                const float* out_scale, void* stream);

/*
 * frt_packed_fp8_gemm_rope_kvcache -- the packed q/k/v GEMM with the split +
 * RoPE + KV write fused into its epilogue (qkv_pack/fp8_static.py joint
 * slots: q and k are one contiguous run consumed together; attention_core
 * `alias_suffix`: the producer writes the suffix in place).  Same result,
 * bit for bit, as frt_packed_fp8_gemm (bf16) followed by
 * frt_split_rope_kvcache on the bf16 output.  N = (hq + 2*hkv) * hd; rows
 * are b * M + s for b < B; see frt_split_rope_kvcache for the outputs.
 * hd % 32 == 0.  The prefix is not copied here (frt_prefix_copy_kv).
 */
int frt_packed_fp8_gemm_rope_kvcache(
    int B, int M, int K, int hq, int hkv, int hd, int P, int T,
    const frt_e4m3* x8, const frt_e4m3* w8, const float* act_scale,
    const float* w_scale, const frt_bf16* bias, const frt_bf16* rope,
    frt_bf16* q_out, frt_bf16* k_cache, frt_bf16* v_cache, void* workspace,
    size_t workspace_bytes, void* stream);

/* ----------------------------------------------------------------------- */
/* a3 / a4  RoPE table, split + RoPE + KV write, prefix copy.               */
/* ----------------------------------------------------------------------- */

/*
 * frt_build_rope_table (fp8_chain.py `_build_rope`): for s < M, i < hd/2,
 *   rope[s, 2i] = bf16(cos((P + s) * theta^(-2i/hd))), rope[s, 2i+1] = sin
 * evaluated in fp64 and rounded once to bf16.  rope_out: [M, hd] bf16.
 */
int frt_build_rope_table(int M, int hd, int P, double theta,
                         frt_bf16* rope_out, void* stream);

/*
 * frt_split_rope_kvcache (fp8_chain.py `_make_run`, the split kernel call;
 * buffers as in `_alloc`): qkv [B*M, (hq + 2*hkv)*hd] bf16, row b*M + s.
 * For q and k heads every adjacent pair (x0, x1) with c = rope[s, 2i],
 * sn = rope[s, 2i+1] becomes (x0*c - x1*sn, x0*sn + x1*c) (fp32, rounded to
 * bf16).  q_out: [B, M, hq, hd]; k_cache, v_cache: [B, T, hkv, hd], written
 * at rows P + s (v copied).  If prefix_k is non-NULL the call also copies
 * the prefix (frt_prefix_copy_kv, launched first).  Requires P + M <= T,
 * M <= 65535 and B <= 65535,
 * hd % 8 == 0, 16-byte aligned pointers.
 */
int frt_split_rope_kvcache(int B, int M, int hq, int hkv, int hd, int P,
                           int T, const frt_bf16* qkv, const frt_bf16* rope,
                           frt_bf16* q_out, frt_bf16* k_cache,
                           frt_bf16* v_cache, const frt_bf16* prefix_k,
                           const frt_bf16* prefix_v, int prefix_T_src,
                           int prefix_interleave, void* stream);

/*
 * frt_prefix_copy_kv (fp8_chain.py `_make_run`, the `ad:prefix` range):
 * prefix_k, prefix_v: host-cache layout [B, hkv, T_src, hd] bf16 (device
 * memory).  Rows p < P go to k_cache / v_cache [B, T, hkv, hd].  With
 * interleave != 0 the key's head dimension is gathered through
 * kperm[2i] = i, kperm[2i+1] = hd/2 + i (rotate-half -> adjacent pairs);
 * v is copied as is.  Bit-exact copy.  P <= T_src, P <= T, hd % 8 == 0.
 */
int frt_prefix_copy_kv(int B, int hkv, int hd, int P, int T, int T_src,
                       const frt_bf16* prefix_k, const frt_bf16* prefix_v,
                       int interleave, frt_bf16* k_cache, frt_bf16* v_cache,
                       void* stream);

/* ----------------------------------------------------------------------- */
/* a5  GEGLU + static requant (standalone form).                            */
/* ----------------------------------------------------------------------- */

/*
 * frt_geglu_quant_fp8 (fp8_chain.py `down_project`; tanh-GELU required by
 * `bind_adarms_fp8_chain`): gu [M, 2H] bf16 (gate in columns [0, H), up in
 * [H, 2H)), row stride ld_gu elements;
 *   hid8[m, j] = e4m3(gelu_tanh(g) * u * (1 / out_scale)) (fp32 reciprocal),
 *   gelu_tanh(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
 * hid8: [M, H].  amax_out: NULL or zeroed device fp32 [1] raised to
 * max |gelu_tanh(g) * u| (calibration).  H % 8 == 0.
 */
int frt_geglu_quant_fp8(int M, int H, const frt_bf16* gu, long ld_gu,
                        const float* out_scale, frt_e4m3* hid8,
                        float* amax_out, void* stream);

/*
 * frt_gelu_quant_fp8 (fp8_ptok_table.py, the DiT FFN's fp8_gelu_mlp middle
 * step, unfused form): hid8[m, j] = e4m3(gelu_tanh(u[m, j]) / out_scale),
 * computed as a multiply by the fp32 reciprocal like the GEGLU kernel.
 * u: bf16 [M, ld_u] (16-byte aligned, ld_u >= H, multiple of 8); hid8:
 * [M, H] e4m3 (8-byte aligned); amax_out (nullable, caller-zeroed) gets
 * max |gelu_tanh(u)|.  H % 8 == 0.
 */
int frt_gelu_quant_fp8(int M, int H, const frt_bf16* u, long ld_u,
                       const float* out_scale, frt_e4m3* hid8, float* amax_out,
                       void* stream);

/* ----------------------------------------------------------------------- */
/* The attention-input chain layer: producer -> packed GEMM (+ RoPE + KV).  */
/* ----------------------------------------------------------------------- */
enum {
  FRT_CHAIN_FUSED_ROPE = 0, /* GEMM epilogue does split + RoPE + KV write */
  FRT_CHAIN_UNFUSED = 1     /* GEMM -> qkv (bf16) -> split kernel          */
};

typedef struct frt_chain_desc {
  int B, M, D;            /* rows = B * M, model width D = K of the GEMM   */
  int hq, hkv, hd;        /* heads; N = (hq + 2*hkv) * hd                  */
  int P, T;               /* prefix rows already in the cache; capacity    */
  float eps;
  int norm_mode;          /* FRT_NORM_*                                    */
  int flags;              /* FRT_CHAIN_*                                   */
  /* producer, FRT_NORM_ADARMS */
  frt_bf16* res; const frt_bf16* delta; const frt_bf16* prev_gate;
  long gate_row_stride; const frt_bf16* norm_weight; const frt_bf16* style;
  long style_row_stride; frt_bf16* gate_out;
  /* producer, FRT_NORM_LAYERNORM_TABLE */
  const frt_bf16* x; const frt_bf16* temb; int chunks; const float* table;
  int shift_idx, scale_idx;
  const float* act_scale; /* device [1] */
  frt_e4m3* x8;           /* [B*M, D] caller-owned staging of the wire     */
  /* packed projection */
  const frt_e4m3* w8; const float* w_scale; const frt_bf16* bias;
  /* RoPE + cache */
  const frt_bf16* rope;   /* [M, hd] */
  frt_bf16* q_out; frt_bf16* k_cache; frt_bf16* v_cache;
  /* optional prefix copy (NULL prefix_k = none) */
  const frt_bf16* prefix_k; const frt_bf16* prefix_v; int prefix_T_src;
  int prefix_interleave;
  frt_bf16* qkv;          /* [B*M, N], needed only with FRT_CHAIN_UNFUSED  */
  void* workspace; size_t workspace_bytes;
} frt_chain_desc;

/* Workspace bytes frt_chain_layer needs for this descriptor. */
size_t frt_chain_workspace_size(const frt_chain_desc* d);

/*
 * frt_chain_layer (fp8_chain.py `_make_run`, one layer's attention half:
 * norm_project(slot 2l, "qkv") then the split kernel; fp8_ptok_table.py:
 * producer then the Q/K/V wire projections): launches the producer, then
 * the packed GEMM with the fused split + RoPE + KV epilogue (or, with
 * FRT_CHAIN_UNFUSED, the GEMM into d->qkv and the split kernel), plus the
 * prefix copy when d->prefix_k is set.  All launches on `stream`.
 */
int frt_chain_layer(const frt_chain_desc* d, void* stream);

/* ----------------------------------------------------------------------- */
/* The FFN half of the AdaRMS layer (fp8_chain.py `_make_run`:               */
/* norm_project(styles, 2l + 1, dn, g1, e, "gu", gu, g2), then               */
/* `down_project`).                                                          */
/* ----------------------------------------------------------------------- */

typedef struct frt_ffn_desc {
  int rows, D, H;         /* tokens, model width, FFN hidden width         */
  float eps;
  /* AdaRMS producer at the FFN site (see frt_ada_norm_quant_fp8, mode 0)   */
  frt_bf16* res;          /* [rows, D] residual, updated in place          */
  const frt_bf16* delta;  /* [rows, D] the output projection's result      */
  const frt_bf16* prev_gate; long gate_row_stride; /* the attention norm's gate */
  const frt_bf16* norm_weight;                      /* nullable = ones      */
  const frt_bf16* style; long style_row_stride;     /* this norm's (scale, shift, gate) */
  frt_bf16* gate_out;     /* nullable: [rows, D], this norm's gate         */
  const float* act_scale; /* device [1]: static scale of the producer      */
  frt_e4m3* x8;           /* [rows, D] staging                             */
  /* gate/up projection with the GEGLU requant epilogue                     */
  const frt_e4m3* w8_gu;  /* [2H, D], FRT_PACK_GATE_UP_BLOCKS layout       */
  const float* w_scale_gu;
  const frt_bf16* bias_gu;    /* nullable, [2H] in the same layout         */
  const float* hid_scale; /* device [1]: static scale of the GEGLU output  */
  frt_e4m3* hid8;         /* [rows, H] staging                             */
  /* down projection                                                         */
  const frt_e4m3* w8_dn;  /* [D, H] */
  const float* w_scale_dn;
  const frt_bf16* bias_dn;    /* nullable, [D] */
  frt_bf16* out;          /* [rows, D] bf16: the next layer's delta        */
  void* workspace; size_t workspace_bytes;  /* both GEMMs, used in turn   */
} frt_ffn_desc;

/* Workspace bytes frt_ffn_layer needs (the larger of its two GEMMs'). */
size_t frt_ffn_workspace_size(const frt_ffn_desc* d);

/*
 * frt_ffn_layer: the producer at the FFN site (res += prev_gate * delta,
 * AdaRMS, static quantize into x8, gate out), the packed gate/up GEMM with
 * the GEGLU + static requant epilogue into hid8, and the down projection
 * into out: three launches on `stream`, each starting while its
 * predecessor drains.  Shapes: D and H multiples of 16, 2H a multiple of
 * 256; errors as the underlying entry points report them.
 */
int frt_ffn_layer(const frt_ffn_desc* d, void* stream);

/* ----------------------------------------------------------------------- */
/* Output side of the AdaRMS layer (fp8_chain.py `out_project`, "ad:tail").  */
/* ----------------------------------------------------------------------- */

/*
 * frt_quantize_fp8_static (fp8_chain.py `out_project`: the attention output
 * quantized with the site's static scale, t_sc_o, before the o_proj GEMM):
 *   x8[r, j] = e4m3_rne_sat(x[r, j] / act_scale[0])   (IEEE fp32 division)
 * x: bf16 [rows, ldx] (device, 16-byte aligned, ldx >= D,
 * ldx % 8 == 0); act_scale: device fp32 [1]; x8_out: [rows, D] e4m3, 8-byte
 * aligned.  amax_out (nullable, device fp32 [1], caller-zeroed) receives
 * max |x| via atomic max.  D % 8 == 0.  rows == 0 is a no-op.
 */
int frt_quantize_fp8_static(int rows, int D, const frt_bf16* x, long ldx,
                            const float* act_scale, frt_e4m3* x8_out,
                            float* amax_out, void* stream);

/*
 * frt_ada_rms_tail (fp8_chain.py `_make_run`, the "ad:tail" range after
 * the layer loop), per row r, fp32 throughout:
 *   h_j   = res[r, j] + gate[r|0, j] * delta[r, j]     (not rounded to bf16)
 *   out_j = bf16((h_j / sqrt(mean_j h^2 + eps)) * (1 + fin[j]) + fin[fin_row_stride + j])
 * res, delta, out: bf16 [rows, D]; gate: bf16 rows gate_row_stride apart
 * (0 = one broadcast row); fin: device fp32, the last norm's scale row and,
 * fin_row_stride elements later, its shift row (one row each, broadcast
 * over tokens).  All 16-byte aligned; D % 8 == 0, 8 <= D <= 8192.
 */
int frt_ada_rms_tail(int rows, int D, float eps, const frt_bf16* res,
                     const frt_bf16* delta, const frt_bf16* gate,
                     long gate_row_stride, const float* fin, long fin_row_stride,
                     frt_bf16* out, void* stream);

/*
 * frt_style_project (fp8_chain.py `_style_stack`: one stacked dense
 * projection serves every norm's (scale, shift, gate); the binder there
 * evaluates it with addmm in fp32 once per probed step and casts the rows
 * to bf16, keeping the final norm's rows in fp32).  This computes it on the
 * device for the live conditioning.  For each row r < rows and column n < N,
 * fp32 throughout:
 *   st[r, n]  = sum_k cond[r, k] * w[n, k] + bias[n]    (bias last)
 *   style_out[r * ld_style + n] = bf16(st[r, n])        (round to nearest even)
 *   fin_out[r * ld_fin + n - fin_col0] = st[r, n]       for n >= fin_col0
 * cond: device fp32 [rows, K], rows ld_cond elements apart (16-byte aligned,
 * ld_cond % 4 == 0).  w: device bf16 [N, K], rows ldw elements apart
 * (16-byte aligned, ldw % 8 == 0): the norms' dense weights concatenated
 * along their outputs, so norm i's scale, shift and gate are columns
 * 3*D*i + {0, D, 2*D} (+ j) and the style rows of norm i start at column
 * 3*D*i of style_out.  bias: device fp32 [N] or NULL.  fin_out: device fp32
 * or NULL (skipped); with a stacked layout, fin_col0 = 3*D*(n_norms - 1)
 * gives the final norm's (scale, shift, gate) rows D apart, the form
 * frt_ada_rms_tail reads.  K % 8 == 0, 8 <= K <= 65536, N >= 1,
 * 0 <= rows <= 65535 (0 is a no-op).  The sum's order differs from index
 * order (lanes split K); each result is within (K + 2) * 2^-24 *
 * (sum_k |cond * w| + |bias|) of the exact value.  w and bias are read
 * before the launch waits on the kernel ahead of it in the stream (they are
 * bind-time data): no kernel still running may write them.
 */
int frt_style_project(int rows, int K, int N, const float* cond, long ld_cond,
                      const frt_bf16* w, long ldw, const float* bias,
                      frt_bf16* style_out, long ld_style, float* fin_out,
                      long ld_fin, int fin_col0, void* stream);

/* ----------------------------------------------------------------------- */
/* Self-test of the bounded device wait.                                    */
/* ----------------------------------------------------------------------- */

/*
 * Launches one CTA that waits on an mbarrier nobody arrives on, bounded by
 * `timeout_us` microseconds, then returns.  Synchronises `stream` and
 * returns FRT_ETIMEOUT when the bound ran out (the expected outcome), so a
 * test can check that bounded waits end and report.  Clears the status.
 */
int frt_selftest_bounded_wait(int timeout_us, void* stream);

/*
 * Evaluates the device GELU the GEGLU and GELU epilogues use:
 * y[i] = gelu_tanh(x[i]) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
 * in fp32, for n device floats (x, y 4-byte aligned, n >= 0), so a test can
 * hold it to an error bound against a higher-precision evaluation.
 * Asynchronous on `stream`.
 */
int frt_selftest_gelu(const float* x, float* y, long n, void* stream);

/* ----------------------------------------------------------------------- */
/* The library's own peak probes (no counterpart on the pages).             */
/* ----------------------------------------------------------------------- */

/* Operand values of the FP8 probe (the tensor pipe's rate depends on them:
 * its power draw sets the clock under the board's power limit). */
enum {
  FRT_PEAK_OPERANDS_GAUSSIAN = 0,  /* e4m3 codes of N(0, 100^2): random signs and
                                      mantissas, amax near 448, like statically
                                      quantised activations and weights */
  FRT_PEAK_OPERANDS_LOW_TOGGLE = 1 /* non-negative codes with bit 4 cleared */
};

/*
 * Dense FP8 tensor-core loop: `ctas` CTAs (one per SM is the intended use)
 * each issue 4 * iters tcgen05.mma.kind::f8f6f4 (M 128, N 256, K 32,
 * e4m3 x e4m3 -> fp32 in TMEM) back to back from operands already in shared
 * memory, filled on the device with the codes `operands` names: 2 * 128 *
 * 256 * 128 * iters flops per CTA and no memory traffic.  The caller times
 * the launch on `stream` (asynchronous).  FRT_EINVAL for ctas outside
 * [1, 4096], iters < 1 or an unknown `operands`.
 */
int frt_peak_fp8_mma(int ctas, int iters, int operands, void* stream);

/*
 * Device-to-device copy of `bytes` (16-byte aligned pointers, a multiple
 * of 16) with streaming loads and stores: 2 * bytes of DRAM traffic when
 * the buffers are far larger than L2.  Asynchronous on `stream`.
 */
int frt_peak_copy(const void* src, void* dst, size_t bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FRT_H_ */
