// frt_internal.cuh -- host-side entry points shared between translation units
// of the library (not part of the C ABI).
#pragma once

#include "frt_common.cuh"
#include "frt_prefix.cuh"

namespace frt {

// The producer (frt_ada_norm_quant_fp8's arguments) launched together with
// the prefix copy in one grid when `pre` is non-null: the extra blocks copy
// the prefix rows while the row blocks run the producer.
int producer_call(int mode, int rows, int D, float eps, uint16_t* res, const uint16_t* delta,
                  const uint16_t* prev_gate, long gate_row_stride, const uint16_t* weight,
                  const uint16_t* style, long style_row_stride, const uint16_t* x,
                  const uint16_t* temb, int chunks, const float* table, int shift_idx,
                  int scale_idx, const float* act_scale, uint8_t* x8_out, uint16_t* gate_out,
                  float* amax_out, const PrefixArgs* pre, cudaStream_t stream);

// Validate the prefix-copy arguments and fill `a`.
int prefix_args(int B, int hkv, int hd, int P, int T, int T_src, const uint16_t* pk,
                const uint16_t* pv, int interleave, uint16_t* k_cache, uint16_t* v_cache,
                PrefixArgs* a);

}  // namespace frt
