// chain.cu -- frt_chain_layer: one layer's attention-input chain.
//
// flashrt-structures 0.2.0, impls/adarms_stack/fp8_chain.py `_make_run`: per
// layer, `norm_project(styles, 2l, delta, gate, e, "qkv", ...)` (the fused
// producer into the merged-QKV FP8 GEMM) followed by the split + RoPE kernel
// that writes q and the suffix K/V behind the prefix copied in the
// `ad:prefix` range; impls/modnorm_qkv_chain/fp8_ptok_table.py: the
// per-token-table producer feeding the Q/K/V wire projections.
//
// Launch sequence on one stream, no host synchronisation, every kernel with
// programmatic dependent launch (each starts while its predecessor drains):
//   FRT_CHAIN_FUSED_ROPE: producer (its extra blocks copy the prefix) ->
//     packed GEMM with the split + RoPE + KV write in its epilogue;
//   FRT_CHAIN_UNFUSED: producer -> packed GEMM -> qkv -> prefix copy (when
//     there is a prefix) -> split kernel.
#include "frt_internal.cuh"

extern "C" size_t frt_chain_workspace_size(const frt_chain_desc* d) {
  if (!d) return 0;
  const long N = long(d->hq + 2 * d->hkv) * d->hd;
  const long rows = long(d->B) * d->M;
  if (rows <= 0 || N <= 0 || rows > 0x7fffffffL) return 0;
  return frt_gemm_workspace_size(int(rows), int(N), d->D, FRT_EPI_BF16);
}

extern "C" int frt_chain_layer(const frt_chain_desc* d, void* stream) {
  frt::clear_error();
  FRT_REQUIRE(d, FRT_EINVAL, "descriptor is NULL");
  FRT_REQUIRE(d->flags == FRT_CHAIN_FUSED_ROPE || d->flags == FRT_CHAIN_UNFUSED, FRT_EINVAL,
              "unknown flags %d", d->flags);
  FRT_REQUIRE(d->B >= 0 && d->M >= 0, FRT_ESHAPE, "B and M must be >= 0");
  FRT_REQUIRE(d->x8, FRT_EINVAL, "x8 staging buffer is required");
  const long rows_l = long(d->B) * d->M;
  FRT_REQUIRE(rows_l <= 0x7fffffffL, FRT_ESHAPE, "B*M too large");
  const int rows = int(rows_l);
  const int N = (d->hq + 2 * d->hkv) * d->hd;
  FRT_REQUIRE(d->P >= 0 && d->P + d->M <= d->T, FRT_ERANGE,
              "P + M = %d exceeds the cache capacity T = %d", d->P + d->M, d->T);
  int rc;
  frt::PrefixArgs pre{};
  const bool fuse_prefix = d->flags == FRT_CHAIN_FUSED_ROPE && d->prefix_k;
  if (fuse_prefix) {
    rc = frt::prefix_args(d->B, d->hkv, d->hd, d->P, d->T, d->prefix_T_src, d->prefix_k,
                          d->prefix_v, d->prefix_interleave, d->k_cache, d->v_cache, &pre);
    if (rc) return rc;
  }
  rc = frt::producer_call(d->norm_mode, rows, d->D, d->eps, d->res, d->delta, d->prev_gate,
                          d->gate_row_stride, d->norm_weight, d->style, d->style_row_stride, d->x,
                          d->temb, d->chunks, d->table, d->shift_idx, d->scale_idx, d->act_scale,
                          d->x8, d->gate_out, nullptr, fuse_prefix ? &pre : nullptr,
                          static_cast<cudaStream_t>(stream));
  if (rc) return rc;
  if (d->flags == FRT_CHAIN_FUSED_ROPE) {
    return frt_packed_fp8_gemm_rope_kvcache(d->B, d->M, d->D, d->hq, d->hkv, d->hd, d->P, d->T,
                                            d->x8, d->w8, d->act_scale, d->w_scale, d->bias,
                                            d->rope, d->q_out, d->k_cache, d->v_cache,
                                            d->workspace, d->workspace_bytes, stream);
  }
  FRT_REQUIRE(d->qkv, FRT_EINVAL, "FRT_CHAIN_UNFUSED needs the qkv buffer");
  rc = frt_packed_fp8_gemm(rows, N, d->D, d->x8, d->w8, d->act_scale, d->w_scale, d->bias,
                           FRT_EPI_BF16, d->qkv, N, nullptr, d->workspace, d->workspace_bytes,
                           stream);
  if (rc) return rc;
  return frt_split_rope_kvcache(d->B, d->M, d->hq, d->hkv, d->hd, d->P, d->T, d->qkv, d->rope,
                                d->q_out, d->k_cache, d->v_cache, d->prefix_k, d->prefix_v,
                                d->prefix_T_src, d->prefix_interleave, stream);
}

// ---------------------------------------------------------------- FFN half --
//
// fp8_chain.py `_make_run`, the second half of the layer loop:
// norm_project(styles, 2l + 1, dn, g1, e, "gu", gu, g2) -- the AdaRMS
// producer at the FFN site feeding the packed gate/up GEMM -- then
// `down_project`: the merged GEGLU + static requant (here the gate/up GEMM's
// epilogue) and the FP8 down projection.  Three launches, each with
// programmatic dependent launch.

extern "C" size_t frt_ffn_workspace_size(const frt_ffn_desc* d) {
  if (!d || d->rows <= 0 || d->D <= 0 || d->H <= 0) return 0;
  const size_t a = frt_gemm_workspace_size(d->rows, 2 * d->H, d->D, FRT_EPI_GEGLU_E4M3);
  const size_t b = frt_gemm_workspace_size(d->rows, d->D, d->H, FRT_EPI_BF16);
  return a > b ? a : b;
}

extern "C" int frt_ffn_layer(const frt_ffn_desc* d, void* stream) {
  frt::clear_error();
  FRT_REQUIRE(d, FRT_EINVAL, "descriptor is NULL");
  FRT_REQUIRE(d->rows >= 0 && d->D > 0 && d->H > 0, FRT_ESHAPE, "bad rows/D/H");
  FRT_REQUIRE(d->x8 && d->hid8 && d->out, FRT_EINVAL, "x8, hid8 and out are required");
  if (d->rows == 0) return FRT_OK;
  int rc = frt::producer_call(FRT_NORM_ADARMS, d->rows, d->D, d->eps, d->res, d->delta,
                              d->prev_gate, d->gate_row_stride, d->norm_weight, d->style,
                              d->style_row_stride, nullptr, nullptr, 0, nullptr, 0, 0,
                              d->act_scale, d->x8, d->gate_out, nullptr, nullptr,
                              static_cast<cudaStream_t>(stream));
  if (rc) return rc;
  rc = frt_packed_fp8_gemm(d->rows, 2 * d->H, d->D, d->x8, d->w8_gu, d->act_scale, d->w_scale_gu,
                           d->bias_gu, FRT_EPI_GEGLU_E4M3, d->hid8, d->H, d->hid_scale,
                           d->workspace, d->workspace_bytes, stream);
  if (rc) return rc;
  return frt_packed_fp8_gemm(d->rows, d->D, d->H, d->hid8, d->w8_dn, d->hid_scale,
                             d->w_scale_dn, d->bias_dn, FRT_EPI_BF16, d->out, d->D, nullptr,
                             d->workspace, d->workspace_bytes, stream);
}
